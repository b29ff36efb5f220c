"""GPU parity of the causal band (nb_attn_fwd_causal / nb_attn_bwd_causal)
against the fp64 oracle: query q in block i sees key k in block j iff
i - R <= j <= i and k <= q (and k < L).  Same tolerances as the symmetric band."""

import pytest
import torch

from oracle import attn_bwd_banded, attn_fwd_banded, attn_fwd_dense
from block_sparse_local_nb_b200.inputs import random_attn_inputs
from tests.gpu_util import (ATOL_F32, GRAD_RFRO_BF16, LSE_ATOL_BF16, O_ATOL_BF16, f64, max_abs,
                            rel_fro, run_bwd, run_fwd)

pytestmark = pytest.mark.gpu

CASES = [(32, 0, [32]), (64, 1, [64, 1]), (96, 2, [96, 50]), (160, 1, [160, 0]),
         (288, 2, [288, 257]), (288, 9, [200, 288]), (544, 8, [544, 321]), (512, 4, [512, 480])]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,R,lens", CASES)
def test_causal_bf16_fwd_bwd(n, R, lens, d):
    q, k, v, do = random_attn_inputs(len(lens), 3, n, d, "bf16", seed=11 * n + R + d)
    L = torch.tensor(lens, dtype=torch.int32)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = run_fwd(qd, kd, vd, L, R, causal=True)
    dq, dk, dv = run_bwd(qd, kd, vd, o, dod, lse, L, R, causal=True)
    args = [t.double().numpy() for t in (q, k, v)]
    o_ref, lse_ref = attn_fwd_banded(*args, R, L.numpy(), causal=True)
    grads_ref = attn_bwd_banded(*args, do.double().numpy(), R, L.numpy(), causal=True)
    assert max_abs(f64(o), o_ref) <= O_ATOL_BF16
    assert max_abs(f64(lse), lse_ref) <= LSE_ATOL_BF16
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), grads_ref):
        assert rel_fro(f64(g), r) <= GRAD_RFRO_BF16, name
    for b, Lb in enumerate(lens):
        for t in (o, dq, dk, dv):
            assert (t[b, :, Lb:] == 0).all()
        assert torch.isneginf(lse[b, :, Lb:]).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,R,lens", [(64, 1, [64, 33]), (288, 2, [288, 200]), (160, 0, [160, 31])])
def test_causal_fp32_fwd(n, R, lens, d):
    q, k, v, _ = random_attn_inputs(2, 2, n, d, "f32", seed=n + R + d + 1)
    L = torch.tensor(lens, dtype=torch.int32)
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), L, R, causal=True)
    o_ref, lse_ref = attn_fwd_dense(q.double().numpy(), k.double().numpy(), v.double().numpy(), R,
                                    L.numpy(), causal=True)
    assert max_abs(f64(o), o_ref) <= ATOL_F32
    assert max_abs(f64(lse), lse_ref) <= ATOL_F32


def test_causal_first_token_and_symmetric_band_differ():
    q, k, v, _ = random_attn_inputs(1, 2, 256, 64, "bf16", seed=3)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    oc, _ = run_fwd(qd, kd, vd, None, 2, causal=True)
    os_, _ = run_fwd(qd, kd, vd, None, 2)
    torch.cuda.synchronize()
    assert torch.allclose(oc[:, :, 0].float(), vd[:, :, 0].float(), atol=1e-2)  # sees only itself
    assert not torch.equal(oc, os_)
