"""Pins for the causal band of the attention oracle (query q in block i sees
key k in block j iff i - R <= j <= i and k <= q, k < L): textbook causal
softmax attention, keys enumerated by hand, closed forms, invariants and
finite differences."""

import math

import numpy as np
import pytest
from scipy.special import softmax

from oracle import attn_bwd_banded, attn_bwd_dense, attn_fwd_banded, attn_fwd_dense
from oracle.attention import block_band_mask


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_wide_band_is_textbook_causal_attention():
    n, d = 96, 8
    q, k, v = (_rand((1, 1, n, d), s) for s in (1, 2, 3))
    o, lse = attn_fwd_dense(q, k, v, R=5, causal=True)  # R >= nb - 1: only causality remains
    o_b, lse_b = attn_fwd_banded(q, k, v, R=5, causal=True)
    for i in range(n):
        s = np.array([q[0, 0, i] @ k[0, 0, j] for j in range(i + 1)]) / math.sqrt(d)
        assert np.allclose(o[0, 0, i], softmax(s) @ v[0, 0, :i + 1], atol=1e-12)
        assert np.allclose(o_b[0, 0, i], o[0, 0, i], atol=1e-12)
        assert math.isclose(lse[0, 0, i], np.log(np.exp(s).sum()), abs_tol=1e-12)


@pytest.mark.parametrize("n,R,L", [(128, 1, 128), (160, 2, 121), (96, 0, 70)])
def test_keys_enumerated_by_hand(n, R, L):
    d = 4
    q, k, v = (_rand((1, 1, n, d), s) for s in (4, 5, 6))
    o, _ = attn_fwd_dense(q, k, v, R, lengths=[L], causal=True)
    o_b, _ = attn_fwd_banded(q, k, v, R, lengths=[L], causal=True)
    for i in range(L):
        keys = [j for j in range(L) if 0 <= i // 32 - j // 32 <= R and j <= i]
        s = np.array([q[0, 0, i] @ k[0, 0, j] for j in keys]) / math.sqrt(d)
        want = softmax(s) @ v[0, 0, keys]
        assert np.allclose(o[0, 0, i], want, atol=1e-12)
        assert np.allclose(o_b[0, 0, i], want, atol=1e-12)
    assert (o[0, 0, L:] == 0).all()


def test_zero_queries_closed_form():
    """Q = 0: uniform weights over the visible keys, lse = ln(number visible)."""
    n, d, R, L = 160, 4, 1, 150
    q = np.zeros((1, 1, n, d))
    k, v = _rand((1, 1, n, d), 7), _rand((1, 1, n, d), 8)
    o, lse = attn_fwd_banded(q, k, v, R, lengths=[L], causal=True)
    for i in range(L):
        lo = max(0, (i // 32 - R) * 32)
        nvis = i - lo + 1
        assert math.isclose(lse[0, 0, i], math.log(nvis), abs_tol=1e-12)
        assert np.allclose(o[0, 0, i], v[0, 0, lo:i + 1].mean(axis=0), atol=1e-12)


def test_first_token_sees_itself_only():
    q, k, v = (_rand((2, 3, 64, 8), s) for s in (9, 10, 11))
    o, _ = attn_fwd_dense(q, k, v, R=1, causal=True)
    assert np.allclose(o[:, :, 0], v[:, :, 0], atol=1e-14)


def test_future_keys_do_not_matter():
    n, d, R = 128, 4, 2
    q, k, v = (_rand((1, 1, n, d), s) for s in (12, 13, 14))
    o, _ = attn_fwd_banded(q, k, v, R, causal=True)
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, 70:] += 5.0
    v2[0, 0, 70:] -= 3.0
    o2, _ = attn_fwd_banded(q, k2, v2, R, causal=True)
    assert np.allclose(o[0, 0, :70], o2[0, 0, :70], atol=1e-12)


def test_mask_is_band_lower_half_with_causal_triangle():
    m = block_band_mask(128, 1, 100, causal=True)
    for i in range(128):
        for j in range(128):
            assert m[i, j] == (0 <= i // 32 - j // 32 <= 1 and j <= i and j < 100)


@pytest.mark.parametrize("R,lengths", [(1, [128, 77]), (0, [90, 128]), (3, [128, 1])])
def test_dense_equals_banded(R, lengths):
    shape = (2, 2, 128, 8)
    q, k, v, do = (_rand(shape, s) for s in (15, 16, 17, 18))
    od, ld = attn_fwd_dense(q, k, v, R, lengths, causal=True)
    ob, lb = attn_fwd_banded(q, k, v, R, lengths, causal=True)
    assert np.allclose(od, ob, atol=1e-12)
    assert np.allclose(np.nan_to_num(ld, neginf=0), np.nan_to_num(lb, neginf=0), atol=1e-12)
    for a, b in zip(attn_bwd_dense(q, k, v, do, R, lengths, causal=True),
                    attn_bwd_banded(q, k, v, do, R, lengths, causal=True)):
        assert np.allclose(a, b, atol=1e-11)


@pytest.mark.parametrize("banded", [False, True])
def test_finite_differences(banded):
    n, d, R, L = 64, 4, 1, 55
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (19, 20, 21, 22))
    bwd = attn_bwd_banded if banded else attn_bwd_dense
    grads = bwd(q, k, v, do, R, [L], causal=True)
    h = 1e-6

    def loss(qq, kk, vv):
        o, _ = attn_fwd_dense(qq, kk, vv, R, [L], causal=True)
        return float((o * do).sum())

    for which, g in enumerate(grads):
        for i in range(n):
            for t in range(d):
                p = [q.copy(), k.copy(), v.copy()]
                m = [q.copy(), k.copy(), v.copy()]
                p[which][0, 0, i, t] += h
                m[which][0, 0, i, t] -= h
                fd = (loss(*p) - loss(*m)) / (2 * h)
                assert abs(fd - g[0, 0, i, t]) < 1e-6 * (1 + abs(fd)), (which, i, t)


def test_gradient_invariants():
    n, d, R, L = 128, 8, 2, 101
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (23, 24, 25, 26))
    dq, dk, dv = attn_bwd_banded(q, k, v, do, R, [L], causal=True)
    assert np.allclose(dv.sum(axis=2), do[:, :, :L].sum(axis=2), atol=1e-10)
    assert np.allclose(dk.sum(axis=2), 0.0, atol=1e-10)
