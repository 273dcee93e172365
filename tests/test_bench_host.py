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
        assert stage.replace("fp8.", "", 1) in bench.STAGES and wl_name in inputs.WORKLOADS and t.startswith("t=")
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


# ------------------------------------------------------------------ roofline arithmetic
PEAKS = {"bf16_tflops": 1713.1, "bf16_tflops_sustained": 1430.5, "hbm_gbs": 6425.6}
H4096 = dict(T=4096, h=4096, f=16384)


def _stages(dom_ms, dom="fc1_backward_weight"):
    ms = {s: 0.4 for s in bench.STAGES}
    ms[dom] = dom_ms
    return ms


def test_roofline_counts_algorithmic_flops_of_one_gemm():
    # the dA stage at 0.6944 ms, full clock: one GEMM of 2*T*h*f = 5.498e11 FLOPs
    clocks = {"sm_mhz": 1957.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    r = bench.roofline_entry(_stages(0.6944), bench.MODES["fast"], clocks=clocks, peaks=PEAKS, peak_src="measured",
                             **H4096)
    assert r["stage"] == "fc1_backward_weight"
    assert abs(r["algorithmic_flops_per_launch"] - 2 * 4096 * 4096 * 16384) < 1
    assert abs(r["achieved"] - 791.7) < 1.0
    # the power-cap bit alone does not switch the peak: the clock was at its maximum
    assert r["peak"] == 1713.1 and abs(r["frac"] - 0.462) < 0.002
    # both halves of the pair run: the executed tensor rate counts two products
    assert r["executed_tensor_products"] == 2 and abs(r["executed_tflops"] - 2 * r["achieved"]) < 1e-6


def test_roofline_takes_the_sustained_peak_only_when_the_clock_sagged():
    low = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    r = bench.roofline_entry(_stages(0.8), 0, clocks=low, peaks=PEAKS, peak_src="measured", **H4096)
    assert r["peak"] == 1430.5
    near = {"sm_mhz": 1920.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.roofline_entry(_stages(0.8), 0, clocks=near, peaks=PEAKS, peak_src="measured",
                                **H4096)["peak"] == 1713.1
    unsampled = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
    assert bench.roofline_entry(_stages(0.8), 0, clocks=unsampled, peaks=PEAKS, peak_src="measured",
                                **H4096)["peak"] == 1713.1


def test_roofline_fraction_stays_below_one_while_the_executed_rate_does():
    """achieved counts one GEMM, the kernel runs one or two products: as long
    as the executed tensor rate is within the peak, frac <= 1."""
    for mode in (0, 3):
        for clocks in ({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0}):
            for dom_ms in (0.66, 0.7, 0.8, 1.2):
                r = bench.roofline_entry(_stages(dom_ms), mode, clocks=clocks, peaks=PEAKS, peak_src="measured",
                                         **H4096)
                if r["executed_frac_of_peak"] <= 1.0:
                    assert r["frac"] <= 1.0, r


def test_stage_products_follow_the_mode():
    acc, fast = bench.stage_products(bench.MODES["accurate"]), bench.stage_products(bench.MODES["fast"])
    assert sum(acc.values()) == 10 and sum(fast.values()) == 8
    assert acc["fc2_forward"] == acc["fc1_backward_data"] == 2 and fast["fc2_forward"] == fast["fc1_backward_data"] == 1


def test_auto_mode_picks_the_fastest_mode_whose_parity_test_passes():
    # the fp16 + e4m3 mode meets the bar on all five workloads (tests/test_fp8.py)
    for name in ("gpt2-medium", "h4096", "8.3b-class", "175b-class"):
        assert bench.pick_mode("auto", name) == "fp8"
    assert bench.pick_mode("auto", "tiny") == "fast"  # launch-bound: the fp8 mode's extra launches cost more
    assert bench.pick_mode("accurate", "h4096") == "accurate"
    assert bench.pick_mode("fast", "h4096") == "fast"
    # without it, fast only where the fast mode's parity test passes
    saved = bench.FP8_MODE_PARITY
    try:
        bench.FP8_MODE_PARITY = ()
        assert bench.pick_mode("auto", "h4096") == "fast"
        assert bench.pick_mode("auto", "8.3b-class") == "accurate"
    finally:
        bench.FP8_MODE_PARITY = saved


def test_fp8_mode_products_and_roofline():
    p = bench.stage_products(bench.MODES["fp8"])
    assert sum(p.values()) == 7 and p["fc1_backward_weight"] == 1.5
    ms = {s: 0.4 for s in bench.FP8_STAGES}
    ms["fp8_prepare_backward"] = 9.0   # an HBM-bound preparation stage is never the tensor roofline's kernel
    ms["fc1_backward_weight"] = 0.526
    r = bench.roofline_entry(ms, bench.MODES["fp8"], 4096, 4096, 16384, {"sm_mhz": 1965, "sm_max_mhz": 1965},
                             PEAKS, "measured")
    assert r["stage"] == "fc1_backward_weight" and r["executed_tensor_products"] == 1.5
    assert abs(r["achieved"] - 2 * 4096 * 4096 * 16384 / 0.526e-3 / 1e12) < 1e-6
    assert abs(r["executed_tflops"] - 1.5 * r["achieved"]) < 1e-6 and r["frac"] <= 1.0


def test_clock_summary_keeps_only_samples_inside_the_window():
    import datetime
    txt = "\n".join([
        "2026/12/03 05:28:00.100, 0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 05:28:00.200, 0, 1500, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 05:28:00.300, 0, 1400, 1965, 950.5, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 05:28:00.400, 0, 1965, 1965, 200.5, 0x0, Not Active, Not Active, Not Active, Not Active"])
    t0, t1 = datetime.datetime(2026, 12, 3, 5, 28, 0, 150000), datetime.datetime(2026, 12, 3, 5, 28, 0, 350000)
    c = bench.summarize_clocks(txt, t0, t1)
    assert c["samples"] == 2 and c["sm_mhz"] == 1450.0 and c["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks(txt)["samples"] == 4
    assert bench.summarize_clocks("")["reasons"] == ["unsampled"]
