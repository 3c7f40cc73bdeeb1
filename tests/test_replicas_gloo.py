"""The multi-GPU path on CPU: two gloo ranks run the replica logic that
bench.py uses under torchrun (pair sharding, barrier, max over ranks,
whole-job rate).  Matching itself needs no collective, so this is all the
ranks share."""
import os
import socket

import pytest
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank, times, out):
    from datetime import timedelta

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from reciprocal_nearest_neighbour_b200 import replicas

    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        w, r, local = replicas.env()
        ids = list(replicas.pair_ids(r, per_rank))
        gathered = [None] * w
        dist.all_gather_object(gathered, ids)
        replicas.barrier(w)
        slowest = replicas.max_over_ranks(times[r], w)
        rate = replicas.aggregate_rate(per_rank, w, slowest)
        out.put((r, w, local, gathered, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_pairs_and_take_the_slowest_step():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [2.5, 4.0]                     # ms per step on each rank
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, 8, times, q))
             for r in range(WORLD)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, world, local, gathered, slowest, rate) in enumerate(res):
        assert (rank, world, local) == (r, WORLD, r)
        flat = [i for ids in gathered for i in ids]
        assert sorted(flat) == list(range(WORLD * 8))          # disjoint, complete
        assert slowest == 4.0                                   # the max over ranks
        assert rate == pytest.approx(WORLD * 8 / 4.0e-3)        # whole-job pairs/s


def test_single_rank_needs_no_process_group():
    from reciprocal_nearest_neighbour_b200 import replicas

    assert replicas.max_over_ranks(3.0, 1) == 3.0
    assert list(replicas.pair_ids(0, 4)) == [0, 1, 2, 3]
    assert replicas.aggregate_rate(8, 1, 2.0) == pytest.approx(4000.0)
    replicas.barrier(1)
