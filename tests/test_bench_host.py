"""Host-side pieces of bench.py that need no GPU: the clock-record summary
and the CPU-baseline record (the oracle timed on a small sample)."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from io_aware_attention_02_b200 import inputs  # noqa: E402


def test_clock_summary_median_max_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1600, 1965, 900.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1620, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 980.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1620.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_flags_throttling_reasons():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1200, 1965, 1000, 0x48, Active, Not Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    c.lines = []
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_cpu_baseline_record_has_the_required_keys():
    q, k, v = inputs.qkv(1, 2, 256, 64, seed=0)
    out = bench.oracle_sample(q, k, v, False, budget_s=0.5)
    for key in ("value", "unit", "cores", "kind", "sample"):
        assert key in out, key
    assert out["kind"] == "oracle" and out["unit"] == "TFLOP/s"
    assert out["value"] > 0 and out["cores"] >= 1
    assert out["single_thread"]["value"] > 0
    # the projection to the whole workload scales the measured rows up
    assert out["extrapolated_full_workload_s"] >= out["seconds"] * 0.999


def test_cpu_baseline_parity_sample_against_given_outputs():
    """With the oracle's own outputs passed in as the 'GPU' result, the
    parity sample is exactly zero."""
    from oracle import attention as A
    q, k, v = inputs.qkv(1, 2, 128, 32, seed=1)
    o, l = A.attention(q, k, v, 1 / 32 ** 0.5, False)
    import torch
    out = bench.oracle_sample(q, k, v, False, budget_s=0.2, gpu_out=(torch.from_numpy(o), torch.from_numpy(l)),
                              single_thread=False)
    assert out["parity_sample"] == {"max_abs_dO": 0.0, "rmse_dO": 0.0, "max_abs_dLSE": 0.0}
    assert "single_thread" not in out


def test_quant_roofline_counts_bytes_per_element_and_block():
    r = bench.quant_roofline(4, 16, 8192, 128, 3, 0.226, 6535.7)
    elems = 4 * 16 * 8192 * 128
    assert r["quant_bytes"] == 3 * (3 * elems + 4 * 4 * 16 * 64)
    assert abs(r["quant_GBs"] - r["quant_bytes"] / 0.226e-3 / 1e9) < 1e-6
    assert 0.40 < r["quant_frac_of_measured_hbm"] < 0.42
    # a ragged last block still has its scale
    assert bench.quant_roofline(1, 1, 129, 64, 1, 1.0, 1.0)["quant_bytes"] == 3 * 129 * 64 + 8


def _run_main(argv, env, capsys, monkeypatch):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
    bench.main()
    return capsys.readouterr().out


def test_reference_arm_other_ranks_exit_without_work(capsys, monkeypatch):
    out = _run_main(["--impl", "reference", "--steps", "1", "--warmup", "3"], {"RANK": "1"}, capsys, monkeypatch)
    assert out == ""


def test_reference_arm_line_has_the_contract_keys(capsys, monkeypatch):
    import json
    out = _run_main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-budget", "0.2",
                     "--ref-total", "1"], {"RANK": "0"}, capsys, monkeypatch)
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["config"]["workload"].startswith("B=4,H=16,N=8192,d=128")
