"""The benchmark's host arithmetic, without a GPU: kernel counts per layer
step and the algorithmic bytes and flops behind every roofline fraction.

The expected values are the per-unit figures written out from the stage
definitions (weights read once, kept rows in and out once, routing arrays
once), independent of bench.py's own expressions."""
import pytest

import bench
import synth


@pytest.mark.parametrize("name,C,launches", [
    ("tiny_switch", 32, 3 + 1 + 2 + 1),    # fp32 router, top-k, assign; dispatch; 2 FMA GEMMs; combine
    ("switch_base", 80, 2 + 1 + 1 + 0),    # fused router+top-1, assign; dispatch; fused FFN+combine
    ("xmoe_top2", 512, 2 + 1 + 2 + 1),     # SM-pair GEMMs (d_model < 2048: two launches); combine
    ("pangu_rre", 640, 2 + 1 + 1 + 0),     # RRE choice, assign; gate 1, combine inside GEMM 2
    ("skewed_switch", 256, 2 + 1 + 2 + 0),
])
def test_kernel_launches(name, C, launches):
    assert bench.kernel_launches(synth.WORKLOADS[name], C) == launches


def test_stage_work_switch_base():
    w = synth.WORKLOADS["switch_base"]
    T, d, f, E = 8192, 768, 3072, 128
    n_kept, tok_any, s = 8100, 8100, 2
    st = bench.stage_work(w, 80, s, n_kept, tok_any)
    # expert FFN: W1 and W2 once, kept rows in and out once; 4 d f flops per kept row
    assert st["expert_ffn"] == (2 * E * d * f * s + 2 * n_kept * d * s, 4.0 * n_kept * d * f)
    assert 2 * E * d * f * s == 1_207_959_552  # the 1.2 GB of Switch-Base expert weights
    # router: x and W_r in, a 4-byte index and a 4-byte gate out per token; 2 d E flops per token
    assert st["router"] == (T * d * s + E * d * s + 8 * T, 2.0 * T * d * E)
    # dispatch of a top-1 layer whose combine is fused: every token's row is read or zeroed
    # once, every kept row written once, 9 bytes of routing arrays per choice
    assert st["dispatch"][0] == (tok_any + n_kept) * d * s + (T - tok_any) * d * s + 9 * T
    assert st["combine"] == (0, 0.0)


def test_stage_work_top2_and_geglu():
    w = synth.WORKLOADS["xmoe_top2"]
    T, d, f, E, k = 16384, 1024, 4096, 64, 2
    n_kept, tok_any, s = 31499, 16000, 2
    st = bench.stage_work(w, 512, s, n_kept, tok_any)
    assert st["dispatch"][0] == (tok_any + n_kept) * d * s + 9 * T * k
    assert st["combine"][0] == (n_kept + T) * d * s + 9 * T * k
    assert st["expert_ffn"][1] == 4.0 * n_kept * d * f
    g = w.scaled(expert="geglu")
    sg = bench.stage_work(g, 512, s, n_kept, tok_any)
    # GEGLU: W1 holds 2f rows (gate and linear), so three d x f matrices per expert
    # and 6 d f flops per kept row
    assert sg["expert_ffn"] == (3 * E * d * f * s + 2 * n_kept * d * s, 6.0 * n_kept * d * f)


def test_stage_roofline_picks_the_slower_roof():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops_sustained": 1.0}
    # 1 GB at 1 TB/s = 1 ms; 0.5 TFLOP at 1 TFLOP/s = 0.5 s -> tensor-bound, 0.5 s roof
    r = bench.stage_roofline({"a": (1e9, 0.5e12), "b": (2e9, 0.0)}, {"a": 1000.0, "b": 4.0}, peaks)
    assert r["a"]["bound"] == "tensor" and r["a"]["frac"] == 0.5
    assert r["b"]["bound"] == "hbm" and r["b"]["frac"] == 0.5 and r["b"]["gbs"] == 500.0


def test_clock_summary_lines():
    """nvidia-smi lines in ClockSampler.QUERY order: medians of SM clock and board
    power, the last max clock and power limit, every throttle reason seen active;
    an unreadable power field is skipped, a short line ignored."""
    lines = [
        "0, 1200, 1965, 998.50, 0x4, Not Active, Not Active, Not Active, Active, 1000.00",
        "0, 1300, 1965, 1001.20, 0x4, Not Active, Not Active, Not Active, Active, 1000.00",
        "0, 1250, 1965, [N/A], 0x0, Not Active, Not Active, Active, Not Active, 1000.00",
        "0, 1250",
    ]
    s = bench.summarize_clock_lines(lines)
    assert s["sm_mhz"] == 1250.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["power_w"] == pytest.approx((998.5 + 1001.2) / 2)
    assert s["power_limit_w"] == 1000.0
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert bench.summarize_clock_lines([])["sm_mhz"] is None


def test_reference_arm_json_line():
    """`bench.py --impl reference` (the CPU oracle, no GPU) prints one JSON line
    with the contract's keys: the oracle's rate as value, cpu_baseline and an
    e2e object with no host-device bytes."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "switch_base", "--steps", "1", "--warmup", "1",
                          "--cpu-seconds", "1"],
                         capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 1
    assert d["config"]["workload"] == "switch_base"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
