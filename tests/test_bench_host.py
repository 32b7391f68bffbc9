"""Host-side pieces of bench.py that need no GPU: the clock summary and the
bounded oracle sample behind cpu_baseline."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_clock_summary_reasons_and_median():
    s = [(1965, 1965, 0), (1800, 1965, 0x4), (1900, 1965, 0x4 | 0x1)]
    out = bench.summarize_clocks(s)
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]          # idle bit 0x1 is not reported
    out = bench.summarize_clocks([(1200, 1965, 0x8 | 0x40 | 0x20)])
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clocks([])["reasons"] == ["unavailable"]


def test_bounded_oracle_sample_stops_at_the_batch():
    from static_token_routed_b200 import workloads as wl
    w = wl.WORKLOADS["tiny_fp32"]
    t, b = wl.make_tables(w), wl.make_batch(w)
    n, dt, cores = bench.time_oracle_bounded(w, t, b, min_seconds=1e9, chunk=256)
    assert n == w.n_tokens and dt > 0 and cores >= 1
