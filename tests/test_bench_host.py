"""Host-side pieces of bench.py (no GPU): the algorithmic units behind the
roofline fractions, checked by brute force against the oracle's band mask, and
the DRAM-traffic record lookup keyed by the kernel sources' hash."""

import pytest

import bench
from block_sparse_local_nb_b200.inputs import AttnWorkload
from oracle.attention import block_band_mask


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,R,lengths,heads,d,dtype", [
    (256, 1, [256], 1, 64, "f32"),
    (512, 2, [512, 333, 1, 0], 3, 64, "bf16"),
    (320, 0, [300, 32], 2, 128, "bf16"),
    (256, 9, [256, 200], 1, 64, "bf16"),  # band wider than the sequence
])
def test_algorithmic_units_match_brute_force(n, R, lengths, heads, d, dtype, causal):
    w = AttnWorkload("t", dtype, len(lengths), heads, n, d, R, 0, causal=causal)
    alg = bench.algorithmic(w, lengths)
    pairs = 0
    for L in lengths:
        m = block_band_mask(n, R, L, causal=causal)[:L]  # valid query rows, visible keys
        pairs += int(m.sum())
    e = 4 if dtype == "f32" else 2
    th = sum(lengths) * heads
    assert alg["tokens"] == sum(lengths)
    assert alg["pairs"] == pairs * heads
    assert alg["fwd_flops"] == 4 * d * pairs * heads
    assert alg["bwd_flops"] == 10 * d * pairs * heads
    assert alg["fwd_bytes"] == th * (4 * d * e + 4)
    assert alg["bwd_bytes"] == th * (8 * d * e + 8)


def test_recorded_traffic_is_keyed_by_source_hash(monkeypatch):
    got = bench.recorded_traffic("nb_attn_bwd", "bf16_varlen")
    assert got is None or got > 0  # present exactly when the sources still match the record
    assert bench.recorded_traffic("no_such_kernel", "bf16_varlen") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("nb_attn_bwd", "bf16_varlen") is None


def test_peaks_are_read_or_fall_back():
    peaks, kind = bench.load_peaks()
    assert kind in ("measured", "fallback")
    assert float(peaks["hbm_gbs"]) > 0


def test_oracle_windows_cover_valid_rows_only():
    from block_sparse_local_nb_b200.inputs import WORKLOADS

    w = WORKLOADS["bf16_n1m"]
    nb = w.n // 32
    for step in range(50):
        b, h, lo, hi = bench.oracle_window(w, [w.n], step)
        assert 0 <= lo < hi <= nb and hi - lo == 256 and 0 <= h < w.heads and b == 0
    w = WORKLOADS["bf16_varlen"]
    lengths = [1030, 4096, 2000, 1]
    for step in range(20):
        b, h, lo, hi = bench.oracle_window(w, lengths, step)
        assert (lo, hi) == (0, (lengths[b] + 31) // 32)


def test_roofline_picks_the_slower_bound():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 50.0}
    r = bench.roofline(2e9, 1e12, 4.0, peaks, 0.1, "bf16")  # 2 ms of HBM vs 10 ms of tensor
    assert r["bound"] == "tensor" and r["peak"] == 100.0 and r["peak_kind"] == "burst"
    assert r["frac"] == pytest.approx(10.0 / 4.0) and r["roofline_ms"] == pytest.approx(10.0)
    r = bench.roofline(2e9, 1e12, 40.0, peaks, 5.0, "bf16")  # a long timed region: sustained peak
    assert r["peak"] == 50.0 and r["peak_kind"] == "sustained"
    r = bench.roofline(8e9, 1e9, 16.0, peaks, 0.1, "bf16")  # 8 ms of HBM vs 0.01 ms of tensor
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(0.5)
    assert bench.tokenizer_bytes(10) == 10 + 2 * 5 + 3
