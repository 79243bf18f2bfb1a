"""CPU checks of bench.py's host logic: the clock-sample summary, the guard
that drops the stored DRAM traffic once the GEMM sources change, the peak
denominators, and the reference arm's non-zero ranks exiting without work."""
import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_clock_summary_reports_median_and_active_reasons():
    lines = [
        "0, 1965, 1965, 600.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 1001.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    c = bench.parse_clocks(lines)
    assert c["sm_mhz"] == 1800.0 and c["sm_max_mhz"] == 1965.0 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]
    c = bench.parse_clocks(["0, 1500, 1965, 700, 0x8, Active, Not Active, Active, Not Active"])
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clocks([])["sm_mhz"] is None


def test_traffic_dropped_when_gemm_sources_differ(monkeypatch):
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "sources_sha256", "0" * 64)
    assert bench.gemm_traffic_per_launch() is None


def test_peaks_are_positive():
    pk, kind = bench.peaks()
    assert kind in ("measured", "fallback")
    assert pk["hbm_gbs"] > 0 and pk["bf16_tflops"] > 0 and pk["bf16_tflops_sustained"] > 0


def test_reference_arm_other_ranks_do_no_work():
    args = argparse.Namespace(gpus=2, steps=1, warmup=3, impl="reference")
    assert bench.run_reference(args, 1, 2) == 0


def test_in_process_clock_summary():
    s = bench.summarize_samples([(1965, 1965, 0), (1900, 1965, 0x4), (1800, 1965, 0x4 | 0x8)])
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.summarize_samples([])["sm_mhz"] is None


def test_stream_plan_matches_the_oracle_bookkeeping():
    """The host-side size plan used for the streaming roofline must follow
    the oracle's FIFO/cache rules (data-independent sizes)."""
    import numpy as np
    import oracle as O
    from synth import make_weights, TINY, synth_clip
    pre = O.PRESETS["low"]
    w = make_weights(TINY, seed=0)
    a, _ = synth_clip(7, 12.0, 2)
    f, L = O.mel_features(a[None], np.array([len(a)]))
    L = int(L[0])
    total = 1 + (L - 1) // 8
    plan = bench.stream_plan((pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period, pre.spkcache_len),
                             total)
    st, taps = O.StreamState(), []
    while st.c0 < total:
        O.stream_step(st, f[0], L, w, pre, taps=taps)
    assert len(plan) == len(taps)
    for (S, new), t in zip(plan, taps):
        assert S == len(t["P"]) and new == len(t["new"])


def test_stream_plan_low_preset_sizes():
    plan = bench.stream_plan((6, 7, 188, 144, 188), 750)
    assert len(plan) == 125
    assert plan[31] == (199, 13) and plan[56] == (249, 13) and plan[-1] == (362, 6)
    assert bench.stream_plan((340, 40, 40, 300, 188), 7500)[1] == (608, 380)
    # one full-size offline clip: 1125 encoder frames, ~351 GFLOP
    assert abs(bench.model_flops(1125, 1125) / 1e9 - 350.7) < 0.1


def test_nemotron_flops_count():
    # 90 s clip: 1125 encoder frames; per frame 2 x 1024 x 512 + 31 x (8 x 512^2
    # + 4 x 512 x 2048 + 2048 x 1125) + 2 x 512 x 64 flops
    per = 2 * 1024 * 512 + 31 * (8 * 512 ** 2 + 4 * 512 * 2048 + 2048 * 1125) + 2 * 512 * 64
    assert abs(bench.nem_model_flops(1125) - 1125 * per) < 1.0
    assert 300e9 < bench.nem_model_flops(1125) < 302e9
