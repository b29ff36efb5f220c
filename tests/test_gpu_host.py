"""GPU parity of nb_attn_fwd_bwd_host (forward + backward of host tensors, cut
into chunks whose copies overlap the compute) against the fp64 oracle and
against the device entry points on the same tensors."""

import pytest
import torch

import block_sparse_local_nb_b200 as nb
from block_sparse_local_nb_b200.inputs import random_attn_inputs
from oracle import attn_bwd_banded, attn_fwd_banded
from tests.gpu_util import (GRAD_RFRO_BF16, LSE_ATOL_BF16, O_ATOL_BF16, f64, max_abs, rel_fro,
                            run_bwd, run_fwd)

pytestmark = pytest.mark.gpu


def _host_step(q, k, v, do, lengths, R, causal=False, pinned=True):
    """Run the host entry point on CPU copies of the inputs; returns CPU outputs."""
    batch, heads, n, d = q.shape
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    hq, hk, hv, hdo = (pin(t.cpu().contiguous()) for t in (q, k, v, do))
    hl = None if lengths is None else pin(lengths.to(torch.int32).cpu())
    outs = [pin(torch.empty_like(hq)) for _ in range(4)]  # o dq dk dv
    lse = pin(torch.empty((batch, heads, n), dtype=torch.float32))
    ws_bytes = nb.attn_fwd_bwd_host_workspace_size(batch, heads, n, d, R, nb.NB_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    nb.nb_attn_fwd_bwd_host(hq, hk, hv, hdo, hl, outs[0], lse, outs[1], outs[2], outs[3], ws,
                            ws_bytes, batch, heads, n, d, R, nb.NB_BF16, causal, stream)
    stream.synchronize()
    return outs[0], lse, outs[1], outs[2], outs[3]


def _device_step(q, k, v, do, lengths, R, causal=False):
    o, lse = run_fwd(q, k, v, lengths, R, causal=causal)
    dq, dk, dv = run_bwd(q, k, v, o, do, lse, lengths, R, causal=causal)
    return o, lse, dq, dk, dv


# (batch, heads, n, R, lengths, windowed): one chunk; chunks of whole batch rows;
# chunks of a few heads of one row (a short last chunk); more chunks than
# workspace slots; too few slices, so each is cut into windows with 2R blocks
# of context (8 windows of 8 blocks at R = 2; 3 windows of 43 blocks at R = 9,
# lengths ending inside a window's context and inside an owned range; 32
# windows of a 65536-token sequence)
CASES = [
    (1, 1, 288, 2, [200], False),
    (16, 2, 96, 1, [96, 1, 33, 64] * 4, False),
    (2, 12, 160, 2, [160, 97], False),
    (3, 5, 288, 9, [288, 0, 131], False),
    (1, 2, 2048, 2, [1900], True),
    (2, 1, 4096, 9, [4096, 2790], True),
    # 32 windows of 64 blocks, the last ones all padding
    (1, 1, 65536, 1, [60000], True),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("batch,heads,n,R,lens,windowed", CASES)
def test_host_step_matches_oracle_and_device_path(batch, heads, n, R, lens, windowed, d, causal):
    q, k, v, do = random_attn_inputs(batch, heads, n, d, "bf16", seed=batch * heads + n + d + R)
    L = torch.tensor(lens, dtype=torch.int32)
    ho, hlse, hdq, hdk, hdv = _host_step(q, k, v, do, L, R, causal)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    do_, dlse, ddq, ddk, ddv = _device_step(qd, kd, vd, dod, L.cuda(), R, causal)
    if not windowed:
        # the same kernels on the same slices: forward, dK and dV identical; dQ
        # up to the order of its fp32 atomic additions
        assert torch.equal(ho, do_.cpu())
        assert torch.equal(hlse, dlse.cpu())
        assert torch.equal(hdk, ddk.cpu()) and torch.equal(hdv, ddv.cpu())
        assert rel_fro(f64(hdq), f64(ddq)) <= 1e-3
    else:
        # windows group the same keys into other chunks: fp32 rounding only
        assert max_abs(f64(ho), f64(do_)) <= 1e-2
        assert max_abs(f64(hlse), f64(dlse)) <= 1e-4
        for got, want in ((hdq, ddq), (hdk, ddk), (hdv, ddv)):
            assert rel_fro(f64(got), f64(want)) <= 2e-3
    args = [t.double().numpy() for t in (q, k, v)]
    o_ref, lse_ref = attn_fwd_banded(*args, R, L.numpy(), causal=causal)
    dq_ref, dk_ref, dv_ref = attn_bwd_banded(*args, do.double().numpy(), R, L.numpy(),
                                             causal=causal)
    assert max_abs(f64(ho), o_ref) <= O_ATOL_BF16
    assert max_abs(f64(hlse), lse_ref) <= LSE_ATOL_BF16
    for got, want in ((hdq, dq_ref), (hdk, dk_ref), (hdv, dv_ref)):
        assert rel_fro(f64(got), want) <= GRAD_RFRO_BF16


def test_host_step_pageable_memory_and_no_lengths():
    """Pageable host buffers (copies serialised) and lengths = NULL give the same results."""
    q, k, v, do = random_attn_inputs(2, 3, 128, 64, "bf16", seed=7)
    a = _host_step(q, k, v, do, None, 2, pinned=False)
    b = _host_step(q, k, v, do, None, 2, pinned=True)
    for x, y in zip(a[:2] + a[3:], b[:2] + b[3:]):
        assert torch.equal(x, y)
    assert rel_fro(f64(a[2]), f64(b[2])) <= 1e-3


def test_host_step_lse_optional():
    q, k, v, do = random_attn_inputs(1, 2, 64, 64, "bf16", seed=3)
    hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
    outs = [torch.empty_like(hq).pin_memory() for _ in range(4)]
    ws_bytes = nb.attn_fwd_bwd_host_workspace_size(1, 2, 64, 64, 1, nb.NB_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    nb.nb_attn_fwd_bwd_host(hq, hk, hv, hdo, None, outs[0], None, outs[1], outs[2], outs[3], ws,
                            ws_bytes, 1, 2, 64, 64, 1, nb.NB_BF16)
    torch.cuda.synchronize()
    ref = _host_step(q, k, v, do, None, 1)
    assert torch.equal(outs[0], ref[0]) and torch.equal(outs[2], ref[3])
