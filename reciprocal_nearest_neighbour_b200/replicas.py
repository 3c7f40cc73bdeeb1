"""Several GPUs of one node.

FRM pairs (and exhaustive-set problems) are independent, so N ranks each
match their own pairs: there is no collective on the data path.  The ranks
meet only to time a step: a barrier on both sides of the timed region and the
maximum of the per-rank step times, from which the whole-job rate is taken.

One exhaustive reciprocal set can also be split over the ranks
(``mnn_sharded``): each rank finds NN2 for a slice of the image-1 pixels and
NN1 for a slice of the image-2 pixels against the whole other map, the
argmax arrays are all-gathered (the one exchange of the method), and every
rank runs the mutual test on the full arrays.

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


def row_slice(n: int, world: int, rank: int) -> range:
    """Rank ``rank``'s contiguous share of ``n`` rows (ceil(n / world) a rank,
    the last shares possibly shorter or empty)."""
    per = -(-n // world)
    return range(min(n, rank * per), min(n, (rank + 1) * per))


def all_gather_rows(part, n: int, world: int):
    """Concatenate every rank's ``row_slice`` part of an ``[n]`` int32 array
    (parts padded to equal length for the collective)."""
    if world == 1:
        return part
    import torch
    import torch.distributed as dist

    per = -(-n // world)
    buf = torch.full((per,), -1, dtype=part.dtype, device=part.device)
    buf[: part.numel()] = part
    out = torch.empty(per * world, dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, buf)
    return out[:n]


def mnn_sharded(D1, D2, world: int, rank: int, *, metric: str = "dot", nn=None, mutual=None):
    """The exhaustive reciprocal set of ``D1 [H1, W1, d]`` and ``D2 [H2, W2, d]``
    split over ``world`` ranks (every rank holds both maps).  Returns
    ``(pairs, count)`` on every rank, as ``mnn_exhaustive``.

    ``nn(Q, X) -> int32 argmax`` and ``mutual(rowarg, colarg) -> (pairs,
    count)`` default to the library's CUDA kernels (``nn_argmax``,
    ``mnn_mutual``)."""
    from . import mnn_mutual, nn_argmax

    if nn is None:
        def nn(Q, X):
            return nn_argmax(Q, X, metric=metric, with_scores=False)[0]
    if mutual is None:
        mutual = mnn_mutual
    d = D1.shape[-1]
    A, B = D1.reshape(-1, d), D2.reshape(-1, d)
    n1, n2 = A.shape[0], B.shape[0]
    r1, r2 = row_slice(n1, world, rank), row_slice(n2, world, rank)
    rowpart = nn(A[r1.start:r1.stop], B)
    colpart = nn(B[r2.start:r2.stop], A)
    rowarg = all_gather_rows(rowpart, n1, world)
    colarg = all_gather_rows(colpart, n2, world)
    return mutual(rowarg, colarg)
