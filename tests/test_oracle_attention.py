"""Pins for the attention oracle against things other than itself: textbook
attention by brute force, the page's band figure, SciPy's softmax and
logsumexp, closed forms, invariants, the page's online recurrence written
independently, and central finite differences."""

import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import (
    BLOCK,
    attn_bwd_banded,
    attn_bwd_dense,
    attn_fwd_banded,
    attn_fwd_dense,
    block_band_mask,
)
from tests.conftest import read_golden


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


def _qkv(batch, heads, n, d, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((batch, heads, n, d)) for _ in range(4))


# ---------------------------------------------------------------- band figure

def test_band_mask_matches_page_figure():
    """The page's block figure (8 block rows) is the band |i-j| <= 2 drawn
    block by block; its label says R = 1, which would draw 2 blocks in row 0.
    The predicate on the page is the authority; the figure pins the band shape."""
    rows = [p[0] for p in read_golden("band_figure_8blocks.txt")]
    fig = np.array([[c == "B" for c in r] for r in rows])
    assert fig.shape == (8, 8)
    m = block_band_mask(8 * BLOCK, R=2)
    blk = m[::BLOCK, ::BLOCK]
    # every token pair inside a block pair has the same visibility
    assert (np.kron(blk, np.ones((BLOCK, BLOCK), bool)) == m).all()
    assert (blk == fig).all()
    assert not (block_band_mask(8 * BLOCK, R=1)[::BLOCK, ::BLOCK] == fig).all()


def test_band_mask_length():
    m = block_band_mask(96, R=0, length=40)
    assert m[0, :32].all() and not m[0, 32:].any()
    assert m[33, 32:40].all() and not m[33, 40:].any()
    assert not m[70].any()  # query block 2 sees only key block 2, all past length


# ----------------------------------------------------- brute-force attention

def _bruteforce_full_attention(q, k, v):
    """Textbook softmax attention with explicit loops (no band, no mask)."""
    n, d = q.shape
    o = np.zeros((n, d))
    lse = np.zeros(n)
    for i in range(n):
        s = [sum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d) for j in range(n)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        lse[i] = mx + math.log(z)
        for j in range(n):
            o[i] += (e[j] / z) * v[j]
    return o, lse


@pytest.mark.parametrize("n,R", [(64, 1), (96, 2), (96, 7)])
def test_full_band_equals_textbook_attention(n, R):
    """R >= nblocks - 1 makes every block visible: plain full attention."""
    q, k, v, _ = _qkv(1, 1, n, 8, seed=n + R)
    o, lse = attn_fwd_dense(q, k, v, R)
    o_ref, lse_ref = _bruteforce_full_attention(q[0, 0], k[0, 0], v[0, 0])
    np.testing.assert_allclose(o[0, 0], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lse_ref, rtol=0, atol=1e-12)
    o_b, lse_b = attn_fwd_banded(q, k, v, R)
    np.testing.assert_allclose(o_b[0, 0], o_ref, rtol=0, atol=1e-12)


def test_fwd_matches_scipy_softmax_per_row():
    """Each valid row equals scipy's softmax over exactly the visible keys,
    with the visible set enumerated from block indices (band and length)."""
    n, d, R, L = 160, 16, 1, 131
    q, k, v, _ = _qkv(1, 1, n, d, seed=3)
    o, lse = attn_fwd_dense(q, k, v, R, lengths=[L])
    for i in range(n):
        if i >= L:
            assert (o[0, 0, i] == 0).all() and lse[0, 0, i] == -np.inf
            continue
        ib = i // 32
        keys = [j for j in range(L) if ib - R <= j // 32 <= ib + R]
        s = np.array([q[0, 0, i] @ k[0, 0, j] for j in keys]) / math.sqrt(d)
        np.testing.assert_allclose(o[0, 0, i], softmax(s) @ v[0, 0, keys], atol=1e-12)
        assert abs(lse[0, 0, i] - logsumexp(s)) < 1e-12


def _online_recurrence(q, k, v, R, L):
    """The page's running (m, d, O) updates over active key blocks, followed by
    the final division O / d.  Written block by block with explicit loops."""
    n, dim = q.shape
    nb = n // 32
    out = np.zeros((n, dim))
    for i in range(n):
        if i >= L:
            continue
        ib = i // 32
        m, dsum, acc = -np.inf, 0.0, np.zeros(dim)
        for jb in range(max(0, ib - R), min(nb - 1, ib + R) + 1):
            ks = [j for j in range(jb * 32, jb * 32 + 32) if j < L]
            if not ks:
                continue
            s = np.array([q[i] @ k[j] for j in ks]) / math.sqrt(dim)
            m_new = max(m, s.max())
            corr = math.exp(m - m_new) if m > -np.inf else 0.0
            e = np.exp(s - m_new)
            dsum = dsum * corr + e.sum()
            acc = acc * corr + e @ v[ks]
            m = m_new
        out[i] = acc / dsum
    return out


def test_fwd_equals_page_online_recurrence():
    n, d, R, L = 192, 8, 2, 170
    q, k, v, _ = _qkv(1, 1, n, d, seed=11)
    o, _ = attn_fwd_dense(q, k, v, R, lengths=[L])
    np.testing.assert_allclose(o[0, 0], _online_recurrence(q[0, 0], k[0, 0], v[0, 0], R, L), atol=1e-12)


# ------------------------------------------------------------- closed forms

def test_constant_v_gives_constant_output():
    n, d = 128, 16
    q, k, _, _ = _qkv(2, 2, n, d, seed=5)
    c = np.random.default_rng(1).standard_normal(d)
    v = np.broadcast_to(c, (2, 2, n, d)).copy()
    lens = [128, 77]
    o, _ = attn_fwd_dense(q, k, v, 1, lengths=lens)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(o[b, :, :L], np.broadcast_to(c, o[b, :, :L].shape), atol=1e-12)
        assert (o[b, :, L:] == 0).all()


@pytest.mark.parametrize("R,L", [(0, 256), (1, 256), (2, 200), (3, 33), (1, 1)])
def test_zero_query_closed_form(R, L):
    """Q = 0 makes every visible score 0: P is uniform over the n_vis visible
    keys, LSE = ln(n_vis) and O is the mean of the visible V rows."""
    n, d = 256, 8
    _, k, v, _ = _qkv(1, 1, n, d, seed=R + L)
    q = np.zeros_like(k)
    o, lse = attn_fwd_dense(q, k, v, R, lengths=[L])
    o_b, lse_b = attn_fwd_banded(q, k, v, R, lengths=[L])
    nb = n // 32
    for i in range(L):
        ib = i // 32
        lo = max(0, ib - R) * 32
        hi = min(min(nb - 1, ib + R) * 32 + 32, L)
        n_vis = hi - lo
        assert abs(lse[0, 0, i] - math.log(n_vis)) < 1e-12
        assert abs(lse_b[0, 0, i] - math.log(n_vis)) < 1e-12
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, lo:hi].mean(axis=0), atol=1e-12)


def test_locality_outside_band_is_ignored():
    n, d, R = 320, 8, 1
    q, k, v, _ = _qkv(1, 1, n, d, seed=9)
    o, _ = attn_fwd_dense(q, k, v, R)
    k2, v2 = k.copy(), v.copy()
    k2[..., 5 * 32:, :] += 100.0  # blocks 5..9 are outside the band of blocks 0..3
    v2[..., 5 * 32:, :] -= 100.0
    o2, _ = attn_fwd_dense(q, k2, v2, R)
    np.testing.assert_array_equal(o[..., :4 * 32, :], o2[..., :4 * 32, :])
    assert np.abs(o[..., 4 * 32:5 * 32, :] - o2[..., 4 * 32:5 * 32, :]).max() > 1.0


def test_padding_contents_are_ignored():
    """Keys and values past the true length (large garbage) change nothing."""
    n, d, R, L = 192, 8, 2, 100
    q, k, v, do = _qkv(1, 2, n, d, seed=21)
    o, lse = attn_fwd_dense(q, k, v, R, lengths=[L])
    grads = attn_bwd_dense(q, k, v, do, R, lengths=[L])
    q2, k2, v2, do2 = q.copy(), k.copy(), v.copy(), do.copy()
    for t in (q2, k2, v2, do2):
        t[..., L:, :] = 1e4
    o2, lse2 = attn_fwd_dense(q2, k2, v2, R, lengths=[L])
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    for g, g2 in zip(grads, attn_bwd_dense(q2, k2, v2, do2, R, lengths=[L])):
        np.testing.assert_array_equal(g, g2)
        assert (g[..., L:, :] == 0).all()


def test_extending_n_with_garbage_keeps_valid_rows():
    n, d, R, L = 128, 8, 1, 128
    q, k, v, _ = _qkv(1, 1, n, d, seed=4)
    o, lse = attn_fwd_dense(q, k, v, R, lengths=[L])
    ext = [np.concatenate([t, 1e3 * np.ones((1, 1, 64, d))], axis=2) for t in (q, k, v)]
    o2, lse2 = attn_fwd_dense(*ext, R, lengths=[L])
    np.testing.assert_allclose(o2[..., :n, :], o, atol=1e-13)
    np.testing.assert_allclose(lse2[..., :n], lse, atol=1e-13)


def test_empty_sequence():
    q, k, v, do = _qkv(2, 1, 64, 8, seed=2)
    o, lse = attn_fwd_dense(q, k, v, 1, lengths=[0, 64])
    assert (o[0] == 0).all() and (lse[0] == -np.inf).all()
    for g in attn_bwd_banded(q, k, v, do, 1, lengths=[0, 64]):
        assert (g[0] == 0).all()


# ---------------------------------------------------------- dense == banded

@pytest.mark.parametrize("n,R,lens", [(96, 0, [96, 50]), (128, 1, [128, 1]), (288, 2, [200, 288]), (160, 9, [31, 160])])
def test_dense_equals_banded(n, R, lens):
    q, k, v, do = _qkv(2, 2, n, 16, seed=n * 10 + R)
    o, lse = attn_fwd_dense(q, k, v, R, lens)
    o_b, lse_b = attn_fwd_banded(q, k, v, R, lens)
    np.testing.assert_allclose(o_b, o, atol=1e-12)
    np.testing.assert_allclose(lse_b, lse, atol=1e-12)
    for g, g_b in zip(attn_bwd_dense(q, k, v, do, R, lens), attn_bwd_banded(q, k, v, do, R, lens)):
        np.testing.assert_allclose(g_b, g, atol=1e-12)


# ----------------------------------------------------------------- gradients

def test_finite_difference_gradients():
    """Central differences (h = 1e-6, fp64) of the scalar sum(O * dO) with
    respect to every element of Q, K and V (n=96, d=8, R=1, L=80)."""
    n, d, R, L = 96, 8, 1, 80
    q, k, v, do = _qkv(1, 1, n, d, seed=31)
    dq, dk, dv = attn_bwd_dense(q, k, v, do, R, lengths=[L])
    h = 1e-6

    def loss(qq, kk, vv):
        o, _ = attn_fwd_dense(qq, kk, vv, R, lengths=[L])
        return float((o * do).sum())

    for name, grad, which in (("dq", dq, 0), ("dk", dk, 1), ("dv", dv, 2)):
        fd = np.zeros((n, d))
        for i in range(n):
            for t in range(d):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][0, 0, i, t] += h
                args_m[which][0, 0, i, t] -= h
                fd[i, t] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(fd - grad[0, 0]) / np.linalg.norm(grad[0, 0])
        assert err < 1e-6, (name, err)


def test_gradient_invariants():
    """Rows of P sum to one, so sum_k dV_k = sum of dO over valid rows; the
    softmax gradient has zero row sums, so sum_k dK_k = 0."""
    q, k, v, do = _qkv(2, 3, 256, 16, seed=17)
    lens = [256, 143]
    dq, dk, dv = attn_bwd_banded(q, k, v, do, 2, lens)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(dv[b].sum(axis=1), do[b, :, :L].sum(axis=1), atol=1e-10)
        np.testing.assert_allclose(dk[b].sum(axis=1), 0.0, atol=1e-10)


def test_gradient_locality():
    """dQ of a query block depends only on keys in its band; a gradient from a
    single output row reaches only keys within R blocks of it."""
    n, d, R = 256, 8, 1
    q, k, v, _ = _qkv(1, 1, n, d, seed=8)
    do = np.zeros((1, 1, n, d))
    do[0, 0, 100] = 1.0  # row 100 is in block 3
    dq, dk, dv = attn_bwd_dense(q, k, v, do, R)
    nz = np.nonzero(np.abs(dk[0, 0]).sum(axis=1) + np.abs(dv[0, 0]).sum(axis=1))[0]
    assert nz.min() >= 2 * 32 and nz.max() < 5 * 32
    assert np.nonzero(np.abs(dq[0, 0]).sum(axis=1))[0].tolist() == [100]
