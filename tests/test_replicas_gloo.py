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


# ------------------------------------------- one reciprocal set over the ranks

def _cpu_nn(Q, X):
    import numpy as np
    import torch

    import oracle

    if Q.shape[0] == 0:
        return torch.empty(0, dtype=torch.int32)
    return torch.from_numpy(oracle.nn(Q, X).arg.astype(np.int32))


def _cpu_mutual(rowarg, colarg):
    import torch

    i = torch.arange(rowarg.numel(), dtype=torch.int32)
    ok = colarg[rowarg.long()] == i
    pairs = torch.stack([i[ok], rowarg[ok]], dim=1)
    return pairs, torch.tensor([pairs.shape[0]], dtype=torch.int32)


def _mnn_rank(rank, world, port, seed, out):
    from datetime import timedelta

    import numpy as np
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from reciprocal_nearest_neighbour_b200 import replicas, synth

    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        rng = np.random.default_rng(seed)
        D1 = synth.to_storage(synth.quantised_map(rng, 13, 11, 16), "f16").float()
        D2 = synth.to_storage(synth.quantised_map(rng, 9, 14, 16), "f16").float()
        pairs, count = replicas.mnn_sharded(D1, D2, world, rank, nn=_cpu_nn, mutual=_cpu_mutual)
        out.put((rank, pairs[: int(count[0])].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_one_reciprocal_set():
    import numpy as np

    import oracle
    from reciprocal_nearest_neighbour_b200 import synth

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_mnn_rank, args=(r, WORLD, port, 17, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rng = np.random.default_rng(17)
    D1 = synth.to_storage(synth.quantised_map(rng, 13, 11, 16), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, 9, 14, 16), "f16")
    ref = oracle.mnn(D1, D2).pairs.tolist()
    assert res[0] == ref and res[1] == ref      # every rank holds the whole set


def test_row_slices_cover_and_gather_alone():
    from reciprocal_nearest_neighbour_b200 import replicas

    for n in (1, 7, 143, 1000):
        for world in (1, 2, 3, 8):
            parts = [replicas.row_slice(n, world, r) for r in range(world)]
            assert [i for p in parts for i in p] == list(range(n))
