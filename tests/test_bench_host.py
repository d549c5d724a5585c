"""Host-side logic of bench.py: FLOP and byte accounting, the traffic record's
source-hash gate, the clock summary and its rejection rule.  No GPU."""
import pytest

import bench
from exact_attention_154_b200 import synth


def test_workload_flops_and_row_flops_agree():
    w = synth.seqlen_sweep(1024, False)
    assert w.flops == 4.0 * w.B * w.H * w.N ** 2 * w.d
    assert bench.row_flops(w, range(w.N)) * w.B * w.H == pytest.approx(w.flops)
    wc = synth.seqlen_sweep(1024, True)
    # causal: row i sees i + 1 keys; the sum over rows is N (N + 1) / 2
    full = bench.row_flops(wc, range(wc.N)) * wc.B * wc.H
    assert full == pytest.approx(4.0 * wc.B * wc.H * wc.d * wc.N * (wc.N + 1) / 2)
    assert bench.row_flops(wc, [0, 9]) == 4.0 * wc.d * (1 + 10)


def test_algorithmic_bytes_of_the_bench_workload():
    w = synth.seqlen_sweep(4096, False)
    # q, k, v read and o written once in 16 bits, plus the fp32 LSE
    assert bench.algorithmic_bytes(w) == 4 * 64 * 2 ** 20 + 4 * w.B * w.H * w.N


def test_traffic_record_is_gated_by_the_source_hash(tmp_path, monkeypatch):
    rec = tmp_path / "traffic.md"
    rec.write_text(f"source_sha256_fwd: {bench.kernel_source_hash('fwd')}\n"
                   f"source_sha256_bwd: {bench.kernel_source_hash('bwd')}\n"
                   "traffic_bytes_per_launch[sweep-n4096]: 123\n"
                   "traffic_bytes_per_launch[bwd:sweep-n4096]: 456\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(rec))
    assert bench.profiled_traffic("sweep-n4096") == 123.0
    assert bench.profiled_traffic("bwd:sweep-n4096") == 456.0
    assert bench.profiled_traffic("sweep-n8192") is None
    # the backward hash covers the backward header too, the forward one does not
    assert bench.kernel_source_hash("fwd") != bench.kernel_source_hash("bwd")
    rec.write_text(f"source_sha256_fwd: {bench.kernel_source_hash('fwd')}\n"
                   "source_sha256_bwd: 0000000000000000\n"
                   "traffic_bytes_per_launch[sweep-n4096]: 123\n"
                   "traffic_bytes_per_launch[bwd:sweep-n4096]: 456\n")
    assert bench.profiled_traffic("sweep-n4096") == 123.0
    assert bench.profiled_traffic("bwd:sweep-n4096") is None
    rec.write_text("source_sha256_fwd: 0000000000000000\ntraffic_bytes_per_launch[sweep-n4096]: 123\n")
    assert bench.profiled_traffic("sweep-n4096") is None
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.md"))
    assert bench.profiled_traffic("sweep-n4096") is None


def test_clock_summary_and_rejection_rule():
    s = bench.ClockSampler(0)
    s.lines = [
        "0, 1600, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1650, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    c = s.summary()
    assert c == {"sm_mhz": 1650.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert bench.clocks_ok(c)  # the power cap is kept and noted
    s.lines.append("0, 1200, 1965, 700.0, 0x8, Not Active, Active, Not Active, Not Active")
    assert not bench.clocks_ok(s.summary())  # a thermal slowdown rejects the run


def test_peaks_fall_back_when_the_measured_file_is_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_peak_follows_the_length_of_the_timed_region():
    peaks = {"bf16_tflops": 1662.1, "bf16_tflops_sustained": 1414.8, "hbm_gbs": 6453.1}
    p, note = bench.pick_peak(peaks, "measured", 0.1)
    assert p == 1662.1 and "burst" in note
    p, note = bench.pick_peak(peaks, "measured", 1.08)
    assert p == 1414.8 and "sustained" in note
    # e4m3: the bf16 figure times the nominal fp8 / bf16 ratio
    p, note = bench.pick_peak(peaks, "measured", 0.1, 2.0)
    assert p == 2 * 1662.1 and "x 2" in note
    p, _ = bench.pick_peak(dict(bench.FALLBACK_PEAKS), "fallback", 2.0)
    assert p == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_committed_traffic_record_matches_the_current_sources():
    """The committed ncu traffic record was taken on the sources in the tree:
    bench.py reports it for the profiled workloads (after a kernel change the
    record must be re-taken, or this fails)."""
    for key in ("sweep-n4096", "causal-h128-n2048", "hd256-causal-n8192", "bwd:sweep-n4096"):
        assert bench.profiled_traffic(key) is not None, key
