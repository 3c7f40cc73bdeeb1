"""Replicas over the GPUs of one node.

FRM pairs (and exhaustive-set problems) are independent, so N ranks each
match their own pairs: there is no collective on the data path.  The ranks
meet only to time a step: a barrier on both sides of the timed region and the
maximum of the per-rank step times, from which the whole-job rate is taken.

Ranks read RANK / LOCAL_RANK / WORLD_SIZE from the environment (as torchrun
sets them); the process group is NCCL on GPUs and gloo on CPU.
"""
from __future__ import annotations

import os


def env():
    """``(world, rank, local_rank)`` from the environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def pair_ids(rank: int, per_rank: int) -> range:
    """The pairs rank ``rank`` matches when every rank takes ``per_rank``."""
    return range(rank * per_rank, (rank + 1) * per_rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest ``x`` over the ranks (all-reduce MAX); ``x`` itself alone."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def aggregate_rate(units_per_rank: float, world: int, step_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's
    step time."""
    return world * units_per_rank / (step_ms * 1e-3)
