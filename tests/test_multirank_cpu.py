"""The multi-rank path of bench.py on CPU: two gloo ranks.

Each rank runs an independent replica (its own seeded layers, no data-path
exchange); the job's time is the slowest rank's and its throughput counts
the units of every rank.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        secs = 0.5 + rank                       # rank 1 is the slow one
        mx = bench.max_over_ranks(secs, world, device="cpu")
        thr = bench.job_throughput(1000, secs, world, device="cpu")
        seed = bench.replica_seed_base(rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        bench.barrier(world)
        out[rank] = (mx, thr, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_throughput():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        mx, thr, seeds = res[r]
        assert mx == pytest.approx(1.5)                  # max over ranks
        assert thr == pytest.approx(1000 * world / 1.5)  # all ranks' units over the slowest time
        assert len(set(seeds)) == world                  # independent replicas


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, 1) == 0.25
    assert bench.job_throughput(10, 0.5, 1) == pytest.approx(20.0)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 12])
def test_build_head_shards_cover_the_heads_in_whole_groups(world):
    """The build leg's head shards: disjoint, in order, whole KV groups (the
    G = 4 query heads of a KV head together), as even as the groups allow;
    with more ranks than KV heads some ranks get none."""
    sys.path.insert(0, ROOT)
    import bench
    Hq, Hkv = 32, 8
    shards = [bench.build_head_shard(Hq, Hkv, world, r) for r in range(world)]
    assert shards[0][0] == 0 and shards[-1][1] == Hq
    for (a0, a1), (b0, b1) in zip(shards, shards[1:]):
        assert a1 == b0
    sizes = [h1 - h0 for h0, h1 in shards]
    assert all(s % (Hq // Hkv) == 0 for s in sizes)
    groups = [s // (Hq // Hkv) for s in sizes]
    assert max(groups) - min(groups) <= 1
    assert sum(s == 0 for s in sizes) == max(0, world - Hkv)
