"""bench.py's JSON line on the GPU: one short run of the tiny workload in a
subprocess, checked key by key against the contract its consumers
read (metric, value, ms_per_step, steps, warmup, roofline, e2e with the
bytes it copies, clocks, gpu_launches) and for internal consistency (value
against ms_per_step and the workload's FLOPs, frac against achieved and peak,
the launch count against the steps)."""
import json
import os
import subprocess
import sys

import pytest

import bench
from tensor_transformer_mlp_bias_b200 import inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_keeps_the_contract():
    steps, warmup = 3, 3
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--steps", str(steps),
                        "--warmup", str(warmup), "--no-cpu-baseline", "--e2e-steps", "2", "--mode", "fp8"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    wl = inputs.WORKLOADS["tiny"]
    T, h, f = wl.T, wl.h, wl.f
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
              "precision_mode"):
        assert k in j, k
    assert j["metric"] == bench.METRIC and j["unit"] == bench.UNIT
    # the fp16 + e4m3 mode (the auto choice on the four larger workloads), labelled as such
    assert j["precision_mode"]["timed"] == "fp8" and j["dtype"] == "bf16+fp16+e4m3"
    assert j["n_gpus"] == 1 and j["steps"] == steps and j["warmup"] == warmup and j["scaling"] == "weak"
    assert j["config"]["flops_per_step"] == wl.flops and j["config"]["T"] == T
    assert abs(j["config"]["tensor_flops_per_step"] - 7 * 2.0 * T * h * f) < 1.0
    # value is the workload's FLOPs over the device time per step
    assert abs(j["value"] - wl.flops / (j["ms_per_step"] * 1e-3) / 1e12) <= 1e-6 * j["value"]
    assert set(j["stage_ms"]) == set(bench.FP8_STAGES)
    ro = j["roofline"]
    assert ro["bound"] == "tensor" and ro["unit"] == "TFLOP/s" and ro["stage"] in bench.FP8_STAGE_PRODUCTS
    assert abs(ro["frac"] - ro["achieved"] / ro["peak"]) < 1e-9 and 0.0 < ro["frac"] <= 1.0
    assert abs(ro["algorithmic_flops_per_launch"] - 2.0 * T * h * f) < 1.0
    assert ro["executed_tensor_products"] in (1, 1.5)
    e2e = j["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == "TFLOP/s"
    # every input copied in (X, A, a, B, b, dY) and every output copied out (Y, dX, dA, da, dB, db), bf16
    assert e2e["h2d_bytes_per_step"] == 2 * (2 * T * h + 2 * h * f + f + h)
    assert e2e["d2h_bytes_per_step"] == 2 * (2 * T * h + 2 * h * f + f + h)
    # the library's own kernels, a whole number per step
    assert j["gpu_launches"] >= 6 * steps and j["gpu_launches"] % steps == 0
    assert isinstance(j["clocks"]["reasons"], list)
    # the bf16 modes beside it: the library's default, and fast (its parity test passes on tiny)
    assert j["accurate"]["value"] > 0 and j["fast"]["value"] > 0 and "fp8" not in j
    assert j["steady"]["seconds"] >= bench.STEADY_SECONDS * 0.9
    assert j["recompute"]["value"] > 0 and j["graph"]["value"] > 0
