"""Sequence parallelism on one GPU: every shard of a sequence is computed
through the C ABI on [left halo | shard | right halo] (the halos cut from the
whole sequence, as the exchange between ranks delivers them), and the shards'
outputs are compared with the fp64 oracle on the whole sequence.  (The
exchange itself runs on gloo ranks in tests/test_seqpar.py.)"""

import numpy as np
import pytest
import torch

from block_sparse_local_nb_b200 import seqpar
from block_sparse_local_nb_b200.inputs import random_attn_inputs
from oracle import attn_bwd_banded, attn_fwd_banded
from tests.gpu_util import GRAD_RFRO_BF16, LSE_ATOL_BF16, O_ATOL_BF16, f64, max_abs, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,n,R,lens,world,align", [
    (64, 2048, 3, [2048, 1500], 3, 256),
    (64, 1536, 8, [1536, 1100], 4, 256),
    (128, 1024, 2, [1000, 1024], 2, 256),
])
def test_shards_with_halos_match_the_whole_sequence(d, n, R, lens, world, align, causal):
    q, k, v, do = random_attn_inputs(len(lens), 2, n, d, "bf16", seed=n + R + d)
    lengths = torch.tensor(lens, dtype=torch.int32)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    ld = lengths.cuda()
    h = seqpar.halo_rows(R)
    outs = {"o": [], "lse": [], "dq": [], "dk": [], "dv": []}
    shards = [seqpar.shard_bounds(n, world, r, align) for r in range(world)]
    fwd = []
    for a, b in shards:
        sl = (slice(None), slice(None), slice(a, b))
        o, lse = seqpar.fwd_with_halo(qd[sl], kd[sl], vd[sl], seqpar.halo_slices(kd, a, b, h),
                                      seqpar.halo_slices(vd, a, b, h), ld, R, a, causal=causal)
        fwd.append((o, lse))
    o_all = torch.cat([o for o, _ in fwd], dim=2)
    lse_all = torch.cat([lse for _, lse in fwd], dim=2)
    for (a, b), (o, lse) in zip(shards, fwd):
        sl = (slice(None), slice(None), slice(a, b))
        halos = {name: seqpar.halo_slices(t, a, b, h)
                 for name, t in (("q", qd), ("k", kd), ("v", vd), ("o", o_all), ("do", dod))}
        halos["lse"] = seqpar.halo_slices(lse_all.unsqueeze(-1), a, b, h)
        halos["lse"] = tuple(t.squeeze(-1) for t in halos["lse"])
        dq, dk, dv = seqpar.bwd_with_halo(qd[sl], kd[sl], vd[sl], o, dod[sl], lse, halos, ld, R, a,
                                          causal=causal)
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            outs[name].append(t)
    torch.cuda.synchronize()
    args = [t.double().numpy() for t in (q, k, v)]
    o_ref, lse_ref = attn_fwd_banded(*args, R, lens, causal=causal)
    grads_ref = attn_bwd_banded(*args, do.double().numpy(), R, lens, causal=causal)
    assert max_abs(f64(o_all), o_ref) <= O_ATOL_BF16
    assert max_abs(f64(lse_all), lse_ref) <= LSE_ATOL_BF16
    for name, r in zip(("dq", "dk", "dv"), grads_ref):
        got = torch.cat(outs[name], dim=2)
        assert rel_fro(f64(got), r) <= GRAD_RFRO_BF16, name
