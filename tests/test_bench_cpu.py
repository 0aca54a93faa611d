"""Host logic of bench.py that needs no GPU: the clock-sample window and the
rate arithmetic the JSON line reports."""
from __future__ import annotations

import bench


def _sampler_with(lines, t0, t1):
    s = bench.ClockSampler(0)
    s.lines = lines
    s.t0, s.t1 = t0, t1
    return s


def _row(mhz, power_cap=False, thermal=False):
    act = "Active"
    return (f"{mhz}, 1965, 0x0, Not Active, Not Active, {act if thermal else 'Not Active'}, "
            f"{act if power_cap else 'Not Active'}")


def test_clock_summary_keeps_only_samples_inside_the_timed_region():
    lines = [(0.0, _row(1200)), (1.0, _row(1965)), (1.5, _row(1950, power_cap=True)), (3.0, _row(1100))]
    s = _sampler_with(lines, 0.9, 2.0).summary()
    assert s["samples"] == 2 and s["window"] == "timed region"
    assert s["sm_mhz"] == (1965 + 1950) / 2 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_neighbouring_samples_for_a_short_region():
    lines = [(0.95, _row(1965, thermal=True)), (2.5, _row(1000))]
    s = _sampler_with(lines, 1.0, 1.004).summary()
    assert s["samples"] == 1 and s["window"] == "within 100 ms of the timed region"
    assert s["reasons"] == ["sw_thermal_slowdown"]


def test_clock_summary_with_no_samples():
    s = _sampler_with([], 1.0, 2.0).summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None


def test_whole_job_rate_counts_every_rank():
    # T units per rank per step, world ranks, ms per step (max over ranks)
    assert bench.whole_job_rate(8192, 1, 10.0) == 8192 / 0.010
    assert bench.whole_job_rate(8192, 4, 10.0) == 4 * 8192 / 0.010


def test_oracle_timing_runs_rows_until_its_budget():
    from sparse_attention_weight_b200.configs import WORKLOADS
    wl = WORKLOADS["tiny_prefill"]
    sample = bench._oracle_sample(wl, rows_max=4)
    assert len(sample["rows"]) == 4
    rows, secs = bench._time_oracle(wl, sample, 0.2)
    assert rows >= 1 and secs >= 0.2
