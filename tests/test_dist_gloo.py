"""The multi-rank benchmark logic on two gloo ranks (CPU): distinct per-rank
inputs, job time = max over ranks, whole-job throughput counts every rank."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_local_nb_b200.dist import job_throughput, max_over_ranks, rank_seed
from block_sparse_local_nb_b200.inputs import WORKLOADS, make_attn_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["bf16_varlen"]
        q, _, _, _, lengths = make_attn_inputs(w, batch=2, heads=1, n=64,
                                               seed=rank_seed(w.seed, rank))
        fp = torch.tensor([float(q.float().sum())], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, fp)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        job_ms = max_over_ranks(my_ms)
        out[rank] = (job_ms, [float(g) for g in gathered],
                     job_throughput(1000.0, 4, world, job_ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        job_ms, fps, thr = res[rank]
        assert job_ms == 15.0  # the max over ranks, seen identically by every rank
        assert thr == pytest.approx(1000.0 * 4 * 2 / 0.015)
        assert fps[0] != fps[1]  # each rank drew its own inputs
    assert rank_seed(2, 0) == 2


def test_single_process_identity():
    assert max_over_ranks(3.5) == 3.5
    assert job_throughput(10, 2, 1, 1000.0) == 20.0
