"""Host logic of the benchmark's roofline bookkeeping (no GPU): algorithmic
work per kernel, trellis edges, the source-hash guard on recorded DRAM traffic,
and the bench metric names."""
import dataclasses

import pytest

import tcq_workloads as W
from trellis_coded_weight_bitshift_b200 import roofline as R


def test_kernel_work_counts():
    n, T = 10, 256
    # decode: 64 B of stream + 512 B of fp16 per 256-weight sequence
    assert R.kernel_work("decode_tile16", 16, n, T) == ("hbm", n * (64 + 512), "bytes")
    # the GEMV counts only the 2-bit stream
    assert R.kernel_work("decode_gemv", 16, n, T) == ("hbm", n * 64, "bytes")
    # Viterbi: 4.5 lane-ops per state-step; the tail-biting search runs twice
    assert R.kernel_work("viterbi", 12, n, T) == ("alu", n * T * 4096 * 4.5, "lane-ops")
    assert R.kernel_work("viterbi_tb", 12, n, T)[1] == 2 * n * T * 4096 * 4.5
    # BCJR: 9/4 MUFU ops per state-step, 11/4 with the gradient
    assert R.kernel_work("bcjr_soft_t0.1", 16, n, T) == ("alu", n * T * 65536 * 9 / 4, "mufu-ops")
    assert R.kernel_work("bcjr_soft_vjp_t0.05", 12, n, T)[1] == n * T * 4096 * 11 / 4
    # rotation: one fp32 read and one write per weight
    assert R.kernel_work("rht", 16, n, T) == ("hbm", n * T * 8.0, "bytes")
    with pytest.raises(KeyError):
        R.kernel_work("unknown_kernel", 12, n, T)


def test_trellis_edges():
    w = W.WORKLOADS["l12_gauss1024"]
    assert R.trellis_edges("viterbi", w) == 2 ** 14 * 255 * 1024
    assert R.trellis_edges("viterbi_tb", w) == 2 * 2 ** 14 * 255 * 1024
    assert R.trellis_edges("decode_tile16", w) == 0.0


def test_measured_traffic_scales_and_guards_sources(monkeypatch):
    w = W.WORKLOADS["l16_studentt_2048x8192"]
    t = R.measured_traffic("bcjr_soft_t1", w)
    assert t is not None and t > 1e12                     # 64-sequence capture scaled to 65,536
    half = dataclasses.replace(w, n_seq=w.n_seq // 2)
    assert R.measured_traffic("bcjr_soft_t1", half) == pytest.approx(t / 2)
    # a kernel whose sources changed since the capture reports no traffic
    monkeypatch.setattr(R, "_sha1", lambda name: "0" * 40)
    assert R.measured_traffic("bcjr_soft_t1", w) is None
    # nothing recorded for this pair
    monkeypatch.undo()
    assert R.measured_traffic("viterbi", W.WORKLOADS["l8_gauss64"]) is None


def test_roofline_entry_fraction():
    peaks = {"hbm_gbs": 6500.0, "sm_max_mhz": 2000.0, "source": "measured"}
    w = W.WORKLOADS["l16_decode_8192sq"]
    e = R.roofline_entry("decode_tile16", w, 0.030, peaks)
    bytes_ = w.n_seq * (64 + 512)
    assert e["bound"] == "hbm" and e["unit"] == "GB/s"
    assert e["achieved"] == pytest.approx(bytes_ / 0.030e-3 / 1e9)
    assert e["frac"] == pytest.approx(e["achieved"] / 6500.0)
    w12 = W.WORKLOADS["l12_gauss1024"]
    e = R.roofline_entry("bcjr_soft_vjp_t0.05", w12, 1.25, peaks)
    assert e["peak"] == pytest.approx(16 * 148 * 2000e6 / 1e9)     # MUFU results/s in G
    assert e["frac"] == pytest.approx(1024 * 256 * 4096 * 11 / 4 / 1.25e-3 / 1e9 / e["peak"])


def test_metric_names_cover_the_step():
    import bench
    assert bench._metric_for(W.WORKLOADS["l12_gauss1024"]) == (
        "weights quantized/sec (Viterbi + pack + decode + BCJR soft + BCJR gradient)")
    assert "x3 temps" in bench._metric_for(W.WORKLOADS["l16_studentt_2048x8192"])
    assert bench._metric_for(W.WORKLOADS["l16_decode_8192sq"]).startswith("decoded weights/sec")
