"""The multi-GPU logic of bench.py on CPU: two gloo ranks (world size 2).

Each GPU runs its own batch with no collective on the data path (the channels of
different batches are independent); the only cross-rank step is taking the maximum of
the ranks' timings, and the whole-job rate counts every rank's elements over the slowest
rank's time. Both are checked here with gloo, and so is the sharding itself: each rank
draws its own batch from the rank-seeded generator and runs the operator (here the fp64
oracle) on it; rank r's result equals a single-process run with seed r, and the two
ranks' batches differ.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank 0 is slower on the first timing, rank 1 on the second
        got = bench.max_over_ranks([10.0 - rank, 3.0 + rank], dist)
        rate = bench.aggregate_rate(world, 8 * 4096 * 4096, 100, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in results:
        assert got == [10.0, 4.0]
        # both ranks' elements over the slowest rank's 10 ms
        assert rate == pytest.approx(2 * 8 * 4096 * 4096 * 100 / 10e-3 / 1e9)


def _shard_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = bench.rank_batch(rank, 2, 48, 16)
        y = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r)
        # every rank's checksum of its own batch, gathered (test-only collective)
        mine = torch.tensor([float(x.k.sum()), float(y.sum())], dtype=torch.float64)
        allv = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(allv, mine)
        q.put((rank, y, [t.tolist() for t in allv]))
    finally:
        dist.destroy_process_group()


def test_rank_batches_are_independent_shards():
    import numpy as np
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((q.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, y, sums in results:
        x = bench.rank_batch(rank, 2, 48, 16)
        y1 = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r)
        assert np.array_equal(y, y1), f"rank {rank} differs from a single run with seed {rank}"
        assert sums == results[0][2]          # both ranks saw the same gathered checksums
    (s0k, s0y), (s1k, s1y) = results[0][2]
    assert s0k != s1k and s0y != s1y         # the two shards are different batches
    assert not np.array_equal(results[0][1], results[1][1])


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.aggregate_rate(1, 1000, 10, 1.0) == pytest.approx(1e-2)
