"""Host-side logic of the multi-GPU benchmark: one process per GPU, each rank
processes its own batch (the path shards over independent sequences and heads,
so there is no collective on the data path).  Only the timing is combined:
the job time is the maximum over ranks and the throughput counts the work of
every rank."""

from __future__ import annotations


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's inputs: distinct per rank, rank 0 keeps the workload's seed."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, job_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank_step * steps * world / (job_ms / 1e3)
