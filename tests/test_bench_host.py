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


def test_tensor_peak_regime():
    """A short region at full clock is held to the burst peak; only a
    seconds-long region whose clock fell well below maximum takes the
    sustained one."""
    peaks = {"bf16_tflops": 1624.7, "bf16_tflops_sustained": 1376.7}
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965}
    slow = {"sm_mhz": 1312, "sm_max_mhz": 1965}
    assert bench.tensor_peak(peaks, 0.034, full) == (1624.7, "burst")
    assert bench.tensor_peak(peaks, 0.034, slow) == (1624.7, "burst")
    assert bench.tensor_peak(peaks, 5.0, full) == (1624.7, "burst")
    assert bench.tensor_peak(peaks, 5.0, slow) == (1376.7, "sustained")
    assert bench.tensor_peak(peaks, 5.0, {"sm_mhz": None, "sm_max_mhz": None})[1] == "burst"


def test_traffic_only_for_unchanged_sources():
    """A stored ncu traffic figure is reported only while its kernel's source
    digest matches the one recorded with the capture."""
    from static_token_routed_b200 import workloads as wl
    w = wl.WORKLOADS["paper_shaped"]
    key = ("mix_gemm_tc", "paper_shaped", w.n_tokens)
    saved = bench.TRAFFIC.get(key)
    try:
        bench.TRAFFIC[key] = {"bytes": 123, "sources": ("gemm_tc.cu",), "digest": "0" * 16,
                              "captured": "x"}
        assert bench.traffic_for("mix_gemm_tc", w)["traffic"] is None
        bench.TRAFFIC[key]["digest"] = bench.source_digest("gemm_tc.cu")
        assert bench.traffic_for("mix_gemm_tc", w)["traffic"] == 123
        assert bench.traffic_for("attn_tail_t1_big", w)["traffic"] is None
    finally:
        if saved is None:
            bench.TRAFFIC.pop(key, None)
        else:
            bench.TRAFFIC[key] = saved
