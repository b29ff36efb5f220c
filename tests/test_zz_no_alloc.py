"""nb_attn_bwd_noalloc, the backward entry point for callers that cannot
allocate device memory (for instance a host program whose GPU memory is all
owned by another allocator, or a foreign-function caller with no allocator):
it must give the same gradients as nb_attn_bwd with a caller workspace, on
consecutive calls that reuse its built-in scratch array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test."""

import ctypes

import pytest
import torch

import block_sparse_local_nb_b200 as nb
from block_sparse_local_nb_b200.inputs import random_attn_inputs
from tests.gpu_util import GRAD_RFRO_BF16, f64, rel_fro, run_bwd, run_fwd

pytestmark = pytest.mark.gpu

NB_ERR_WORKSPACE = -5
SCRATCH_BYTES = 64 << 20  # NB_NOALLOC_SCRATCH_BYTES in include/nb.h


def _noalloc():
    fn = nb.lib().nb_attn_bwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    return fn


def _call(fn, q, k, v, o, do, lse, lengths, R):
    batch, heads, n, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
            lengths.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), batch, heads, n, d, R,
            nb.NB_BF16, torch.cuda.current_stream().cuda_stream)
    assert st == 0, nb.nb_status_string(st)
    return dq, dk, dv


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(d):
    fn = _noalloc()
    # two different problems in a row: the second reuses the scratch the first wrote
    cases = [((2, 3, 512, d), [512, 301], 2, 21), ((3, 2, 800, d), [800, 45, 613], 1, 22)]
    for shape, lens, R, seed in cases:
        q, k, v, do = (t.cuda() for t in random_attn_inputs(*shape, "bf16", seed=seed))
        lengths = torch.tensor(lens, dtype=torch.int32, device="cuda")
        o, lse = run_fwd(q, k, v, lengths, R)
        want = run_bwd(q, k, v, o, do, lse, lengths, R)
        got = _call(fn, q, k, v, o, do, lse, lengths, R)
        torch.cuda.synchronize()
        # dK and dV are deterministic: bit-identical to the workspace path
        assert torch.equal(got[1], want[1]) and torch.equal(got[2], want[2])
        # dQ is accumulated with fp32 atomics (order may differ): within the bf16 bar
        assert rel_fro(f64(got[0]), f64(want[0])) <= GRAD_RFRO_BF16


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fn = _noalloc()
    batch, heads, n, d = 1, 8, 65536, 64  # needs about 130 MiB of scratch
    assert nb.attn_bwd_workspace_size(batch, heads, n, d, nb.NB_BF16) > SCRATCH_BYTES
    # every pointer null: whatever the order of the checks, the call fails on the host
    st = fn(None, None, None, None, None, None, None, None, None, None, batch, heads, n, d, 1,
            nb.NB_BF16, None)
    assert st == NB_ERR_WORKSPACE
