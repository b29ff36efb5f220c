"""fp64 oracle for banded block-sparse local attention (forward and backward).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed, following the NucleoByte page, section 3 "Mathematical
Foundations":

* "Localized Block-Sparse Attention Matrix": tokens are grouped in blocks of
  B = 32; query block i may attend key block j only when |i - j| <= R.
* "Softmax Normalization & Online Numerical Stability": scores are
  S = Q K^T / sqrt(d_k).  The page accumulates a running max m_i, running sum
  d_i and running output O_i over the active key blocks; that recurrence
  reaches exactly (up to rounding order) the plain softmax of S over the
  visible keys, which is what the oracle writes out: a two-pass softmax
  (pass 1: row max, pass 2: exponentials and their sum), then O = P V.
  The page never writes the final division O_i / d_i; it is the only reading
  under which the recurrence is a softmax, so the oracle normalises.
* Sections 1-2 ("Padding Waste", "Dynamic Ceiling Hardware Alignment"):
  sequences are padded up to a multiple of 32 and keys at positions >= the
  sequence's true length L are masked.  Query rows >= L are padding: their
  outputs are defined as 0 and their log-sum-exp as -inf; their upstream
  gradient is ignored.
* "Custom Backpropagation": the backward uses the row term
  D_i = sum_k dO_ik O_ik and the softmax gradient dS_ij = P_ij (dO_i V_j^T - D_i);
  the remaining gradients are the chain rule through S = scale Q K^T and O = P V:
  dV = P^T dO, dQ = scale dS K, dK = scale dS^T Q.

Layout: every tensor is [batch, heads, n, d] (d innermost); log-sum-exp is
[batch, heads, n].  ``lengths`` is an int array [batch] with 0 <= L <= n
(None means every sequence is full length).

Causal band (a variant the page does not print; the plainest causal reading
of its band): query q in block i sees key k in block j only when
i - R <= j <= i and k <= q, i.e. the band's lower half plus the token-level
causal triangle of the diagonal block.  Every function takes ``causal``.

Two restatements of the same definition are given:
* ``*_dense``: the full n x n score matrix with the band mask applied
  (small n only);
* ``*_banded``: the same definition evaluated only on each query block's band
  of key blocks [max(0, i-R), min(nb-1, i+R)].  Masked entries have exactly zero
  probability, so both reach the same numbers; a CPU test checks that.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 32  # the page's block size B


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _lengths(lengths, batch: int, n: int) -> np.ndarray:
    if lengths is None:
        return np.full(batch, n, dtype=np.int64)
    lens = np.asarray(lengths, dtype=np.int64).reshape(batch)
    if (lens < 0).any() or (lens > n).any():
        raise ValueError("lengths must lie in [0, n]")
    return lens


def block_band_mask(n: int, R: int, length: int | None = None, block: int = BLOCK,
                    causal: bool = False) -> np.ndarray:
    """Boolean visibility matrix M[q, k] for one sequence.

    M[q, k] is True iff the key block of k lies within R blocks of the query
    block of q (|q // B - k // B| <= R) and k < length; with ``causal`` also
    k <= q.  Query-row padding is not part of the mask (rows q >= length are
    handled by the callers).
    """
    blk = np.arange(n) // block
    m = np.abs(blk[:, None] - blk[None, :]) <= R
    if causal:
        m &= np.arange(n)[None, :] <= np.arange(n)[:, None]
    if length is not None:
        m &= (np.arange(n) < length)[None, :]
    return m


def _softmax_rows(S: np.ndarray):
    """Two-pass softmax of each row of S (entries may be -inf).

    Returns (P, m, l) with m the row max and l = sum exp(S - m).  Rows whose
    entries are all -inf get P = 0, m = -inf, l = 0.
    """
    m = S.max(axis=1)
    finite = np.isfinite(m)
    shifted = np.where(finite[:, None], S - np.where(finite, m, 0.0)[:, None], -np.inf)
    E = np.exp(shifted)
    l = E.sum(axis=1)
    P = np.where(l[:, None] > 0, E / np.where(l > 0, l, 1.0)[:, None], 0.0)
    return P, m, l


def attn_fwd_dense(q, k, v, R: int, lengths=None, causal: bool = False):
    """Forward pass from the dense definition.

    Returns (o, lse): o [batch, heads, n, d] fp64 and lse [batch, heads, n]
    fp64, where lse = m + ln(l) is the natural-log log-sum-exp of the row's
    scaled scores.  Rows q >= L: o = 0, lse = -inf.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    batch, heads, n, d = q.shape
    lens = _lengths(lengths, batch, n)
    scale = 1.0 / math.sqrt(d)
    o = np.zeros_like(q)
    lse = np.full((batch, heads, n), -np.inf)
    for b in range(batch):
        L = int(lens[b])
        mask = block_band_mask(n, R, L, causal=causal)
        for h in range(heads):
            S = scale * (q[b, h] @ k[b, h].T)
            S = np.where(mask, S, -np.inf)
            P, m, l = _softmax_rows(S[:L])
            o[b, h, :L] = P @ v[b, h]
            lse[b, h, :L] = m + np.log(l)
    return o, lse


def attn_bwd_dense(q, k, v, do, R: int, lengths=None, causal: bool = False):
    """Analytic gradients from the dense definition.

    Returns (dq, dk, dv), each [batch, heads, n, d] fp64.  P and O are
    recomputed from the definition; D_i = sum_k dO_ik O_ik and
    dS = P * (dO V^T - D) as on the page; upstream gradient rows q >= L are
    ignored and gradient rows >= L come out as exactly zero.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    batch, heads, n, d = q.shape
    lens = _lengths(lengths, batch, n)
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(batch):
        L = int(lens[b])
        mask = block_band_mask(n, R, L, causal=causal)
        for h in range(heads):
            S = np.where(mask, scale * (q[b, h] @ k[b, h].T), -np.inf)
            P = np.zeros((n, n))
            P[:L], _, _ = _softmax_rows(S[:L])
            dO = np.zeros((n, d))
            dO[:L] = do[b, h, :L]
            O = P @ v[b, h]
            D = (dO * O).sum(axis=1)  # row correction term D_i
            dv[b, h] = P.T @ dO
            dP = dO @ v[b, h].T
            dS = P * (dP - D[:, None])  # softmax gradient
            dq[b, h] = scale * (dS @ k[b, h])
            dk[b, h] = scale * (dS.T @ q[b, h])
    return dq, dk, dv


def _band(i: int, R: int, nb: int, causal: bool = False):
    return max(0, i - R), (i if causal else min(nb - 1, i + R))


def _causal_cut(S: np.ndarray, r0: int, k0: int) -> np.ndarray:
    """S with entries of keys after their query (k > q) set to -inf."""
    qi = r0 + np.arange(S.shape[0])[:, None]
    ki = k0 + np.arange(S.shape[1])[None, :]
    return np.where(ki <= qi, S, -np.inf)


def attn_fwd_banded(q, k, v, R: int, lengths=None, causal: bool = False):
    """Forward pass evaluated only on each query block's band of key blocks.

    Same definition and outputs as :func:`attn_fwd_dense`; memory is linear in
    n, so it serves long sequences.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    batch, heads, n, d = q.shape
    if n % BLOCK:
        raise ValueError("n must be a multiple of the block size")
    nb = n // BLOCK
    lens = _lengths(lengths, batch, n)
    scale = 1.0 / math.sqrt(d)
    o = np.zeros_like(q)
    lse = np.full((batch, heads, n), -np.inf)
    for b in range(batch):
        L = int(lens[b])
        for i in range(nb):
            r0 = i * BLOCK
            rows = min(BLOCK, L - r0)
            if rows <= 0:
                break
            j0, j1 = _band(i, R, nb, causal)
            k0, k1 = j0 * BLOCK, min((j1 + 1) * BLOCK, L)  # keys past L are masked
            for h in range(heads):
                S = scale * (q[b, h, r0:r0 + rows] @ k[b, h, k0:k1].T)
                if causal:
                    S = _causal_cut(S, r0, k0)
                P, m, l = _softmax_rows(S)
                o[b, h, r0:r0 + rows] = P @ v[b, h, k0:k1]
                lse[b, h, r0:r0 + rows] = m + np.log(l)
    return o, lse


def attn_bwd_banded(q, k, v, do, R: int, lengths=None, causal: bool = False):
    """Analytic gradients evaluated only on each query block's band.

    Same definition and outputs as :func:`attn_bwd_dense`: for every query
    block i, P_i over its visible keys, O_i = P_i V, D_i = rowsum(dO_i O_i),
    dS_i = P_i (dO_i V^T - D_i); then dV += P_i^T dO_i, dQ_i = scale dS_i K,
    dK += scale dS_i^T Q_i over the band's keys.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    batch, heads, n, d = q.shape
    if n % BLOCK:
        raise ValueError("n must be a multiple of the block size")
    nb = n // BLOCK
    lens = _lengths(lengths, batch, n)
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(batch):
        L = int(lens[b])
        for i in range(nb):
            r0 = i * BLOCK
            rows = min(BLOCK, L - r0)
            if rows <= 0:
                break
            j0, j1 = _band(i, R, nb, causal)
            k0, k1 = j0 * BLOCK, min((j1 + 1) * BLOCK, L)
            for h in range(heads):
                Qi = q[b, h, r0:r0 + rows]
                dOi = do[b, h, r0:r0 + rows]
                Kb, Vb = k[b, h, k0:k1], v[b, h, k0:k1]
                S = scale * (Qi @ Kb.T)
                if causal:
                    S = _causal_cut(S, r0, k0)
                P, _, _ = _softmax_rows(S)
                Oi = P @ Vb
                D = (dOi * Oi).sum(axis=1)
                dP = dOi @ Vb.T
                dS = P * (dP - D[:, None])
                dv[b, h, k0:k1] += P.T @ dOi
                dq[b, h, r0:r0 + rows] = scale * (dS @ Kb)
                dk[b, h, k0:k1] += scale * (dS.T @ Qi)
    return dq, dk, dv


def attn_bwd_from_saved(q, k, v, o, do, lse, R: int, lengths=None, causal: bool = False):
    """Analytic gradients from the forward's saved outputs, as the page's
    backward uses them (NucleoByte page, section 3 "Custom Backpropagation"):
    the probabilities are rebuilt from the stored log-sum-exp,
    P_ij = exp(scale Q_i K_j^T - lse_i) over the band's visible keys, and the
    row term is D_i = sum_k dO_ik O_ik with the given O.  With O and lse from
    :func:`attn_fwd_banded` of the same inputs this is :func:`attn_bwd_banded`;
    the difference is that a row's P and D come from the given lse and O, not
    from the keys this call sees (a shard of a longer sequence sees only part
    of a halo row's keys, while the row's lse and O are the whole sequence's).
    Rows >= L_b and rows whose lse is -inf contribute nothing.
    """
    q, k, v, o, do = _f64(q), _f64(k), _f64(v), _f64(o), _f64(do)
    lse = _f64(lse)
    batch, heads, n, d = q.shape
    if n % BLOCK:
        raise ValueError("n must be a multiple of the block size")
    nb = n // BLOCK
    lens = _lengths(lengths, batch, n)
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(batch):
        L = int(lens[b])
        for i in range(nb):
            r0 = i * BLOCK
            rows = min(BLOCK, L - r0)
            if rows <= 0:
                break
            j0, j1 = _band(i, R, nb, causal)
            k0, k1 = j0 * BLOCK, min((j1 + 1) * BLOCK, L)
            for h in range(heads):
                Qi = q[b, h, r0:r0 + rows]
                dOi = do[b, h, r0:r0 + rows]
                Kb, Vb = k[b, h, k0:k1], v[b, h, k0:k1]
                S = scale * (Qi @ Kb.T)
                if causal:
                    S = _causal_cut(S, r0, k0)
                li = lse[b, h, r0:r0 + rows][:, None]
                with np.errstate(invalid="ignore"):
                    P = np.where(np.isfinite(li), np.exp(S - li), 0.0)
                D = (dOi * o[b, h, r0:r0 + rows]).sum(axis=1)
                dP = dOi @ Vb.T
                dS = P * (dP - D[:, None])
                dv[b, h, k0:k1] += P.T @ dOi
                dq[b, h, r0:r0 + rows] = scale * (dS @ Kb)
                dk[b, h, k0:k1] += scale * (dS.T @ Qi)
    return dq, dk, dv
