"""Host logic of a multi-GPU run (one process per GPU, weak scaling).

Decode steps of different sequences are independent, so a run on N GPUs
gives every rank its own batch of sequences (its own seeded synthetic
inputs) and exchanges no data on the hot path. The only collective is the
timing reduction: the job's time is the slowest rank's, and the job's
throughput counts the units of all ranks.
"""
import torch
import torch.distributed as dist


def rank_recipe(base, rank, world):
    """The workload of `rank`: the base recipe with a rank-specific seed, so
    ranks decode different sequences of the same shape."""
    return base.scaled(seed=base.seed + 1000 * rank) if world > 1 else base


def max_over_ranks(value, device=None):
    """Maximum of a float over the ranks of the default process group (the
    value itself when there is none)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, total_ms_max, steps):
    """Units per second of the whole job: every rank's units over the slowest
    rank's time per step."""
    ms = total_ms_max / steps
    return units_per_rank * world / (ms * 1e-3), ms
