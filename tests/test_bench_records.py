"""Host-side records of bench.py on CPU: the clock summary over the timed
region, and the oracle's CPU baseline for forward and forward+backward steps."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import Workload, make_inputs  # noqa: E402

BITS = bench.ClockSampler.REASON_BITS


def test_clock_summary_keeps_only_samples_inside_the_timed_region():
    # (time, sm MHz, max MHz, power W, reason bits)
    rows = [(0.0, 1200.0, 1965.0, 300.0, 0), (1.0, 1965.0, 1965.0, 900.0, BITS["sw_power_cap"]),
            (1.01, 1900.0, 1965.0, 950.0, 0), (1.02, 1950.0, 1965.0, 940.0, 0),
            (3.0, 600.0, 1965.0, 100.0, BITS["hw_slowdown"])]
    c = bench.summarise_clocks(rows, 0.5, 2.0, "nvml", BITS)
    assert c["samples_in_timed_region"] == 3 and c["samples"] == 3
    assert c["sm_mhz"] == 1950.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample lies outside


def test_clock_summary_falls_back_to_all_samples_and_reports_none():
    rows = [(0.0, 1800.0, 1965.0, 500.0, BITS["hw_thermal_slowdown"])]
    c = bench.summarise_clocks(rows, 5.0, 6.0, "nvml", BITS)
    assert c["samples_in_timed_region"] == 0 and c["samples"] == 1
    assert c["reasons"] == ["hw_thermal_slowdown"]
    c = bench.summarise_clocks([], 0.0, 1.0, None, BITS)
    assert c["sm_mhz"] is None and c["samples"] == 0


def test_oracle_sample_extrapolates_every_part_of_a_fwd_bwd_step():
    wl = Workload("tiny_fb", "swiglu", "bf16", 64, 32, 4 * 32, 4, seed=3, w_std=0.05,
                  backward=True)
    inp = make_inputs(wl)
    parts = bench.oracle_sample(wl, inp, 16, 32)
    assert {"fwd_rows_s", "dx_rows_s", "dw_cols_s"} <= set(parts)
    want = (parts["fwd_rows_s"] * 64 / 16 + parts["dx_rows_s"] * 64 / 16
            + parts["dw_cols_s"] * 128 / 32)
    assert abs(parts["extrapolated_full_step_s"] - want) <= 1e-12 * max(want, 1.0)
    wf = Workload("tiny_f", "gelu", "bf16", 64, 32, 64, 2, seed=3, w_std=0.05)
    fwd = bench.oracle_sample(wf, make_inputs(wf), 16, 32)
    assert set(fwd) == {"fwd_rows_s", "extrapolated_full_step_s"}


def test_cpu_baseline_reports_the_whole_step():
    wl = Workload("tiny_fb2", "swiglu", "bf16", 96, 32, 2 * 64, 2, seed=4, w_std=0.05,
                  backward=True)
    cb = bench.cpu_baseline(wl, target_s=0.05)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert cb["extrapolated_full_step_s"] > 0
    assert "input gradient" in cb["sample"] and "weight gradients" in cb["sample"]


def test_attention_cpu_baseline_extrapolates_from_two_row_counts():
    from workloads import AttnWorkload, make_attn_inputs
    wl = AttnWorkload("tiny_attn", 64, 256, 2, 2, True, seed=3, w_std=0.05)
    parts = bench.attn_oracle_sample(wl, make_attn_inputs(wl), 8)
    assert parts["extrapolated_full_step_s"] >= parts["fixed_s"] >= 0
    assert abs(parts["extrapolated_full_step_s"]
               - (parts["fixed_s"] + parts["per_row_s"] * 64)) < 1e-12
    cb = bench.attn_cpu_baseline(wl, rows=8)
    assert cb["kind"] == "oracle" and cb["value"] > 0
