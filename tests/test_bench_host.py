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
