"""Sequence parallelism (block_sparse_local_nb_b200/seqpar.py) on CPU: the
shard partition, and the halo exchange on gloo ranks with the fp64 oracle as
the per-shard computation.  Sharded forward + backward must give the
whole-sequence oracle's O, lse, dQ, dK and dV (fp64: to rounding).  The
oracle's backward from saved outputs (what each shard runs, because a halo
row's lse and O belong to the whole sequence) is first pinned to the plain
backward."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_local_nb_b200 import seqpar
from oracle import attn_bwd_banded, attn_bwd_from_saved, attn_fwd_banded


def _inputs(batch, heads, n, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((batch, heads, n, d)) for _ in range(4)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,R,lens", [(256, 2, [256, 150]), (320, 0, [7, 320]), (192, 9, [192, 33])])
def test_backward_from_saved_outputs_is_the_plain_backward(n, R, lens, causal):
    q, k, v, do = _inputs(2, 2, n, 8, seed=n + R)
    o, lse = attn_fwd_banded(q, k, v, R, lens, causal=causal)
    want = attn_bwd_banded(q, k, v, do, R, lens, causal=causal)
    got = attn_bwd_from_saved(q, k, v, o, do, lse, R, lens, causal=causal)
    for g, w in zip(got, want):
        assert np.allclose(g, w, rtol=1e-12, atol=1e-12)


def test_backward_from_saved_uses_the_given_lse_and_o():
    """A row whose lse is raised by ln 2 has half its P, so its dV
    contribution halves; an O shifted by c changes D by c . dO."""
    q, k, v, do = _inputs(1, 1, 64, 8, seed=3)
    o, lse = attn_fwd_banded(q, k, v, 0)
    lse2 = lse.copy()
    lse2[0, 0, :32] += np.log(2.0)
    do_first = do.copy()
    do_first[0, 0, 32:] = 0  # only block 0 contributes
    _, _, dv1 = attn_bwd_from_saved(q, k, v, o, do_first, lse, 0)
    _, _, dv2 = attn_bwd_from_saved(q, k, v, o, do_first, lse2, 0)
    assert np.allclose(dv2, dv1 / 2)


@pytest.mark.parametrize("n,world,align", [(4096, 3, 256), (256, 4, 32), (96, 5, 32), (512, 1, 256)])
def test_shards_partition_the_sequence(n, world, align):
    bounds = [seqpar.shard_bounds(n, world, r, align) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == n
    for (a, b), (c, _) in zip(bounds, bounds[1:]):
        assert b == c and a <= b
    for a, b in bounds:
        assert a % align == 0 and (b % align == 0 or b == n)


def _np_fwd(q, k, v, lengths, R, causal):
    o, lse = attn_fwd_banded(q.numpy(), k.numpy(), v.numpy(), R, lengths.numpy(), causal=causal)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _np_bwd(q, k, v, o, do, lse, lengths, R, causal):
    g = attn_bwd_from_saved(q.numpy(), k.numpy(), v.numpy(), o.numpy(), do.numpy(), lse.numpy(),
                            R, lengths.numpy(), causal=causal)
    return tuple(torch.from_numpy(x) for x in g)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = [  # (n, R, lengths, align, causal)
    (1024, 2, [1024, 700], 256, False),
    (1024, 3, [1000, 1024], 256, True),
    (768, 8, [768, 530], 256, False),   # halo of 256 rows = a whole shard
    (512, 0, [512, 77], 128, False),
]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        errs = []
        for ci, (n, R, lens, align, causal) in enumerate(CASES):
            q, k, v, do = (torch.from_numpy(x) for x in _inputs(2, 2, n, 8, seed=40 + ci))
            lengths = torch.tensor(lens, dtype=torch.int32)
            o_ref, lse_ref = attn_fwd_banded(q.numpy(), k.numpy(), v.numpy(), R, lens, causal=causal)
            g_ref = attn_bwd_banded(q.numpy(), k.numpy(), v.numpy(), do.numpy(), R, lens,
                                    causal=causal)
            a, b = seqpar.shard_bounds(n, world, rank, align)
            sl = (slice(None), slice(None), slice(a, b))
            o, lse = seqpar.seqpar_attn_fwd(q[sl], k[sl], v[sl], lengths, R, a, rank, world,
                                            causal=causal, fwd_fn=_np_fwd)
            grads = seqpar.seqpar_attn_bwd(q[sl], k[sl], v[sl], o, do[sl], lse, lengths, R, a,
                                           rank, world, causal=causal, bwd_fn=_np_bwd)
            e = [np.abs(o.numpy() - o_ref[sl]).max(),
                 np.abs(np.nan_to_num(lse.numpy() - lse_ref[:, :, a:b], nan=0.0)).max()]
            e += [np.abs(g.numpy() - r[sl]).max() for g, r in zip(grads, g_ref)]
            # -inf lse must match exactly where the rows are padding
            e.append(float((np.isneginf(lse.numpy()) != np.isneginf(lse_ref[:, :, a:b])).sum()))
            errs.append(max(e))
        out[rank] = errs
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_attention_equals_whole_sequence(world):
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        assert max(res[rank]) < 1e-10, (rank, res[rank])
