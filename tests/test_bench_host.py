"""Host-side parts of bench.py that need no GPU: the reference arm (the fp64
oracle timed on this host) prints one JSON line with the bench's keys, ranks
other than 0 stay silent, and the DRAM traffic of the dominant kernel is
looked up by stage, workload, shard count and kernel-source digest."""
import json
import os
import subprocess
import sys

import bench
from tensor_transformer_mlp_bias_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, extra_env=None):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          timeout=300, cwd=ROOT, env=env)


def test_reference_arm_prints_one_line_with_the_bench_keys():
    r = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in j, k
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == bench.UNIT
    assert j["n_gpus"] == 1 and j["steps"] == 2 and j["warmup"] == 3 and j["higher_is_better"] is True
    assert j["value"] > 0 and j["ms_per_step"] > 0
    wl = inputs.WORKLOADS["tiny"]
    assert j["config"]["T"] == wl.T and j["config"]["h"] == wl.h and j["config"]["f"] == wl.f
    assert j["config"]["flops_per_step"] == wl.flops
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1 and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_is_at_least_three_steps():
    r = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr
    assert json.loads(r.stdout.strip().splitlines()[-1])["warmup"] == 3


def test_traffic_lookup(monkeypatch):
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    rows = [ln.split() for ln in open(path).read().splitlines() if ln.strip() and not ln.startswith("#")]
    assert rows
    for stage, wl_name, t, digest, nbytes in rows:
        assert stage in bench.STAGES and wl_name in inputs.WORKLOADS and t.startswith("t=")
        assert len(digest) == 12 and float(nbytes) > 0
    stage, wl_name, t, digest, nbytes = rows[0]
    wl, tt = inputs.WORKLOADS[wl_name], int(t[2:])
    # the sources the summary was taken on
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    assert bench.traffic_for(stage, wl, tt) == float(nbytes)
    assert bench.traffic_for(stage, wl, tt + 1) is None
    other = next(n for n in inputs.WORKLOADS if n != wl_name)
    assert bench.traffic_for(stage, inputs.WORKLOADS[other], tt) is None
    # any change to the kernel sources drops the figure
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "f" * 12 if digest != "f" * 12 else "0" * 12)
    assert bench.traffic_for(stage, wl, tt) is None


def test_kernel_source_digest_covers_the_kernel_files():
    d = bench.kernel_source_digest()
    assert len(d) == 12 and int(d, 16) >= 0
