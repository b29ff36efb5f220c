"""GPU parity of nb_attn_fwd / nb_attn_bwd against the fp64 oracle.

Small cases compare every element; the full-size workloads compare sampled
windows of blocks (the oracle evaluated on a sub-sequence with two band radii
of context on each side, where its outputs are exact).  Tolerances:
fp32 max-abs 1e-4 (O, lse); bf16 max-abs 1.5e-2 on O, 1e-3 on lse,
relative Frobenius 1e-2 on dQ, dK, dV.
"""

import numpy as np
import pytest
import torch

from block_sparse_local_nb_b200.inputs import (WORKLOADS, AttnWorkload, make_attn_inputs,
                                               random_attn_inputs)
from oracle import attn_bwd_banded, attn_fwd_banded, attn_fwd_dense
from tests.gpu_util import (ATOL_F32, GRAD_RFRO_BF16, LSE_ATOL_BF16, O_ATOL_BF16, f64, max_abs,
                            rel_fro, run_bwd, run_fwd, window)

pytestmark = pytest.mark.gpu
BLOCK = 32


def _lengths(vals):
    return torch.tensor(vals, dtype=torch.int32)


def _cuda(*ts):
    return [t.cuda() for t in ts]


# ------------------------------------------------------------------ fp32

def test_fp32_n256_workload():
    """fp32, 1 x 1 x 256 x 64, R = 1, full length, seed 0: every element."""
    w = WORKLOADS["fp32_n256"]
    q, k, v, _, lengths = make_attn_inputs(w)
    o, lse = run_fwd(*_cuda(q, k, v), lengths, w.R)
    o_ref, lse_ref = attn_fwd_dense(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    w.R, lengths.numpy())
    assert max_abs(f64(o), o_ref) <= ATOL_F32
    assert max_abs(f64(lse), lse_ref) <= ATOL_F32


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,R,lens", [
    (32, 0, [32, 1]), (64, 1, [64, 33]), (96, 2, [0, 95]), (288, 2, [288, 200]),
    (288, 9, [17, 288]), (160, 0, [160, 31]),
])
def test_fp32_small(n, R, lens, d):
    q, k, v, _ = random_attn_inputs(2, 3, n, d, "f32", seed=n + R + d)
    L = _lengths(lens)
    o, lse = run_fwd(*_cuda(q, k, v), L, R)
    o_ref, lse_ref = attn_fwd_dense(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    R, L.numpy())
    assert max_abs(f64(o), o_ref) <= ATOL_F32
    assert max_abs(f64(lse), lse_ref) <= ATOL_F32


# ----------------------------------------------------------------- bf16 small

SMALL = [
    (32, 0, [32]), (64, 1, [64, 1]), (96, 2, [96, 50]), (128, 1, [100, 128]),
    (160, 1, [160, 0]), (288, 2, [288, 257]), (288, 9, [200, 288]), (416, 3, [33, 416]),
    (512, 4, [512, 480]), (544, 8, [544, 321]),
]


def _bf16_case(n, R, lens, d, seed, heads=3):
    q, k, v, do = random_attn_inputs(len(lens), heads, n, d, "bf16", seed=seed)
    L = _lengths(lens)
    qd, kd, vd, dod = _cuda(q, k, v, do)
    o, lse = run_fwd(qd, kd, vd, L, R)
    dq, dk, dv = run_bwd(qd, kd, vd, o, dod, lse, L, R)
    args = [t.double().numpy() for t in (q, k, v)]
    o_ref, lse_ref = attn_fwd_banded(*args, R, L.numpy())
    grads_ref = attn_bwd_banded(*args, do.double().numpy(), R, L.numpy())
    return (o, lse, dq, dk, dv), (o_ref, lse_ref, *grads_ref), L


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,R,lens", SMALL)
def test_bf16_fwd_bwd_small(n, R, lens, d):
    got, ref, L = _bf16_case(n, R, lens, d, seed=7 * n + R + d)
    o, lse, dq, dk, dv = got
    o_ref, lse_ref, dq_ref, dk_ref, dv_ref = ref
    assert max_abs(f64(o), o_ref) <= O_ATOL_BF16
    assert max_abs(f64(lse), lse_ref) <= LSE_ATOL_BF16
    for name, g, r in (("dq", dq, dq_ref), ("dk", dk, dk_ref), ("dv", dv, dv_ref)):
        assert rel_fro(f64(g), r) <= GRAD_RFRO_BF16, name
    # padding rows are exactly zero, log-sum-exp -inf
    for b, Lb in enumerate(L.tolist()):
        for t in (o, dq, dk, dv):
            assert (t[b, :, Lb:] == 0).all()
        assert torch.isneginf(lse[b, :, Lb:]).all()


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_dk_dv_deterministic(d):
    """dK and dV accumulate in tensor memory in a fixed order: bit-identical on a
    second call (both backward kernels); dQ differs only by the order of its fp32
    atomic additions; the forward is deterministic."""
    q, k, v, do = _cuda(*random_attn_inputs(2, 4, 1024, d, "bf16", seed=5))
    L = _lengths([1024, 700])
    o, lse = run_fwd(q, k, v, L, 2)
    a = run_bwd(q, k, v, o, do, lse, L, 2)
    b = run_bwd(q, k, v, o, do, lse, L, 2)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert rel_fro(f64(a[0]), f64(b[0])) < 1e-3
    o2, lse2 = run_fwd(q, k, v, L, 2)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_bf16_chained_calls_without_sync_match_synchronized():
    """Kernels start early (programmatic dependent launch) but wait for the
    previous kernel before touching memory: a chain in which each call
    consumes the previous call's outputs gives the same bits with or without
    a device synchronisation between the calls."""
    q, k, v, do = _cuda(*random_attn_inputs(2, 4, 1024, 64, "bf16", seed=21))
    L = _lengths([1024, 613])

    def chain(sync):
        o, lse = run_fwd(q, k, v, L, 2)
        sync()
        _, dk, dv = run_bwd(q, k, v, o, do, lse, L, 2)
        sync()
        o2, lse2 = run_fwd(dk, dv, k, L, 2)  # reads what the last kernel just wrote
        sync()
        return o, lse, dk, dv, o2, lse2

    a = chain(lambda: None)
    b = chain(torch.cuda.synchronize)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bf16_padding_contents_are_ignored():
    """Garbage (1e4) in Q, K, V and dO past each length changes nothing."""
    n, R, d = 640, 2, 64
    q, k, v, do = _cuda(*random_attn_inputs(2, 2, n, d, "bf16", seed=9))
    L = _lengths([500, 333])
    o, lse = run_fwd(q, k, v, L, R)
    grads = run_bwd(q, k, v, o, do, lse, L, R)
    q2, k2, v2, do2 = (t.clone() for t in (q, k, v, do))
    for b, Lb in enumerate(L.tolist()):
        for t in (q2, k2, v2, do2):
            t[b, :, Lb:] = 1e4
    o2, lse2 = run_fwd(q2, k2, v2, L, R)
    grads2 = run_bwd(q2, k2, v2, o2, do2, lse2, L, R)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(grads[1], grads2[1]) and torch.equal(grads[2], grads2[2])
    assert rel_fro(f64(grads2[0]), f64(grads[0])) < 1e-3


def test_bf16_lse_optional_and_lengths_null():
    n, R, d = 256, 1, 64
    q, k, v, _ = _cuda(*random_attn_inputs(1, 2, n, d, "bf16", seed=4))
    o_full, _ = run_fwd(q, k, v, None, R)
    o_none, _ = run_fwd(q, k, v, _lengths([n]), R, with_lse=False)
    assert torch.equal(o_full, o_none)


def test_bf16_out_of_range_lengths_are_clamped():
    n, R, d = 128, 1, 64
    q, k, v, do = _cuda(*random_attn_inputs(2, 1, n, d, "bf16", seed=6))
    o_a, lse_a = run_fwd(q, k, v, _lengths([n + 1000, -5]), R)
    o_b, lse_b = run_fwd(q, k, v, _lengths([n, 0]), R)
    assert torch.equal(o_a, o_b) and torch.equal(lse_a, lse_b)


# ------------------------------------------------------- full-size workloads

def _check_window(w, tensors, outs, bh, blk_lo, blk_hi, lengths, check_bwd=True):
    """Compare the GPU outputs of one (batch, head) on blocks [blk_lo, blk_hi)."""
    q, k, v, do = tensors
    o, lse, dq, dk, dv = outs
    b, h = bh
    nb = w.n // BLOCK
    s, e = window(nb, blk_lo, blk_hi, w.R)
    Lb = int(lengths[b])
    Lsub = min(max(Lb - s * BLOCK, 0), (e - s) * BLOCK)
    sl = slice(s * BLOCK, e * BLOCK)
    sub = [t[b, h, sl].double().cpu().numpy()[None, None] for t in (q, k, v, do)]
    o_ref, lse_ref = attn_fwd_banded(*sub[:3], w.R, [Lsub], causal=w.causal)
    r0, r1 = (blk_lo - s) * BLOCK, (blk_hi - s) * BLOCK
    g0, g1 = blk_lo * BLOCK, blk_hi * BLOCK
    assert max_abs(f64(o[b, h, g0:g1]), o_ref[0, 0, r0:r1]) <= O_ATOL_BF16
    assert max_abs(f64(lse[b, h, g0:g1]), lse_ref[0, 0, r0:r1]) <= LSE_ATOL_BF16
    if check_bwd:
        grads_ref = attn_bwd_banded(*sub, w.R, [Lsub], causal=w.causal)
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), grads_ref):
            err = rel_fro(f64(g[b, h, g0:g1]), r[0, 0, r0:r1])
            assert err <= GRAD_RFRO_BF16, (name, err)


def _run_workload(w):
    q, k, v, do, lengths = make_attn_inputs(w, device="cuda")
    o, lse = run_fwd(q, k, v, lengths, w.R, causal=w.causal)
    grads = run_bwd(q, k, v, o, do, lse, lengths, w.R, causal=w.causal) if w.backward else (None,) * 3
    torch.cuda.synchronize()
    return (q, k, v, do), (o, lse, *grads), lengths


@pytest.mark.parametrize("name", ["bf16_varlen", "bf16_varlen_causal"])
def test_bf16_varlen_workload(name):
    """bf16, 4 x 12 x 4096 x 64, R = 2, lengths ~ U[1024, 4096] (symmetric and
    causal band): three whole heads and sampled windows of the rest, including
    each sequence's length boundary.  The windows carry 2R blocks of context on
    each side, which covers every dependency of the checked blocks in both bands."""
    w = WORKLOADS[name]
    tensors, outs, lengths = _run_workload(w)
    nb = w.n // BLOCK
    for bh in [(0, 0), (1, 5), (3, 11)]:
        _check_window(w, tensors, outs, bh, 0, nb, lengths)
    rng = np.random.default_rng(0)
    for b in range(w.batch):
        Lb = int(lengths[b])
        edge = (Lb - 1) // BLOCK
        h = int(rng.integers(w.heads))
        _check_window(w, tensors, outs, (b, h), max(0, edge - 3), min(nb, edge + 4), lengths)
    for t in outs:
        for b in range(w.batch):
            Lb = int(lengths[b])
            assert (t[b, :, Lb:] == 0).all() or torch.isneginf(t[b, :, Lb:]).all()


def test_bf16_d128_ragged_many_items():
    """bf16, 6 x 8 x 8192 x 128, R = 3, lengths ~ U[1500, 8192]: about 21 work
    items per CTA with empty tiles, so every role of both d = 128 kernels wraps
    its buffer and barrier parities many times over ragged items.  Two whole
    heads, each sequence's length boundary and the last wave of items."""
    w = AttnWorkload("bf16_d128_ragged", "bf16", 6, 8, 8192, 128, 3, 5, varlen=(1500, 8192),
                     desc="fwd+bwd bf16 6x8x8192x128 R=3 L~U[1500,8192]")
    tensors, outs, lengths = _run_workload(w)
    nb = w.n // BLOCK
    for bh in [(0, 3), (5, 7)]:
        _check_window(w, tensors, outs, bh, 0, nb, lengths)
    rng = np.random.default_rng(3)
    for b in range(w.batch):
        edge = (int(lengths[b]) - 1) // BLOCK
        _check_window(w, tensors, outs, (b, int(rng.integers(w.heads))), max(0, edge - 3),
                      min(nb, edge + 4), lengths)
    # the last non-empty tile of the last sequence, every head
    edge = (int(lengths[-1]) - 1) // BLOCK
    for h in range(w.heads):
        _check_window(w, tensors, outs, (w.batch - 1, h), max(0, edge - 7), edge + 1, lengths)
    for t in outs:
        for b in range(w.batch):
            Lb = int(lengths[b])
            assert (t[b, :, Lb:] == 0).all() or torch.isneginf(t[b, :, Lb:]).all()


def _full_size_windows(w, width, seed):
    """(head, first block) of the windows checked on a full-length, batch-1
    workload: the first and last window and one random window of every head,
    plus windows on the persistent kernels' last wave of work items (one
    128-row tile per item, items handed round-robin to one CTA per SM): the
    wave's first tile, its middle and the sequence's last tile, where each
    CTA runs its final item and the epilogue of that item (the forward's
    epilogue warpgroup, the backward's deferred dK/dV epilogue)."""
    nb = w.n // BLOCK
    rng = np.random.default_rng(seed)
    out = []
    for h in range(w.heads):
        out += [(h, 0), (h, nb - width), (h, int(rng.integers(0, nb - width)))]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = w.n // 128
    items = w.heads * tiles
    first_last = (items - 1) // sms * sms  # first item of the last wave
    for it in (first_last, (first_last + items) // 2, items - 1):
        h, tile = divmod(it, tiles)
        lo = min(max(0, 4 * tile - width // 2), nb - width)
        out.append((h, lo))
    return out


def test_bf16_n131k_workload():
    """bf16, 1 x 16 x 131072 x 128, R = 4: first, last and a random window of
    every head, and the persistent kernels' last wave."""
    w = WORKLOADS["bf16_n131k"]
    tensors, outs, lengths = _run_workload(w)
    for h, lo in _full_size_windows(w, 12, seed=1):
        _check_window(w, tensors, outs, (0, h), lo, lo + 12, lengths)


def test_bf16_n1m_workload():
    """bf16, 1 x 8 x 1048576 x 64, R = 8: first, last and a random window of
    every head, and the persistent kernels' last wave; peak memory linear in n."""
    w = WORKLOADS["bf16_n1m"]
    torch.cuda.reset_peak_memory_stats()
    tensors, outs, lengths = _run_workload(w)
    peak = torch.cuda.max_memory_allocated()
    elems = w.batch * w.heads * w.n * w.d
    # 9 bf16 tensors (q k v do o dq dk dv + slack), lse, D and the fp32 dQ accumulator
    assert peak <= elems * 2 * 9 + elems * 4 + w.batch * w.heads * w.n * 8 + (64 << 20)
    for h, lo in _full_size_windows(w, 20, seed=2):
        _check_window(w, tensors, outs, (0, h), lo, lo + 20, lengths)
