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
        # the line rank 0 prints: whole-job throughput, the slowest rank's time, N ranks
        roof = bench.decode_roofline(16_801_920, 11.0, 6543.4, "measured", None, "k")
        line = bench.decode_line(thr, mx * 1e3 / 10, world, 10, 3, {"workload": "w"}, roof,
                                 {"value": thr}, 10 * 32 * 2, {"sm_mhz": None})
        out[rank] = (mx, thr, seeds, line["n_gpus"], line["value"])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_throughput():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        mx, thr, seeds, n_gpus, value = res[r]
        assert mx == pytest.approx(1.5)                  # max over ranks
        assert thr == pytest.approx(1000 * world / 1.5)  # all ranks' units over the slowest time
        assert len(set(seeds)) == world                  # independent replicas
        assert n_gpus == world and value == pytest.approx(thr)


def test_gpus_flag_is_honoured():
    """`--gpus N` runs N ranks: started directly it re-launches itself under
    torchrun with N processes on 127.0.0.1; under a launcher the launcher's
    world size must be N, else the run is refused rather than measured on
    another number of GPUs."""
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.torchrun_argv(4, ["--gpus", "4", "--steps", "20"], 29123)
    assert "--nproc-per-node=4" in cmd and "torch.distributed.run" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and "29123" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "20"] and cmd[-5].endswith("bench.py")
    assert cmd[:3] == ["timeout", "-k", "60"]
    bench.check_world(2, 2)
    with pytest.raises(SystemExit):
        bench.check_world(2, 1)
    with pytest.raises(SystemExit):
        bench.check_world(1, 8)


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


# ------------------------------------------------ build split over ranks --

@pytest.mark.parametrize("world", [1, 2, 3, 4, 5, 8, 12])
def test_chunk_and_head_shards_cover_the_work_once(world):
    """Every prefix chunk is encoded by exactly one rank, in contiguous runs
    in rank order (so the gathered states arrive in chunk order); every head
    is built by exactly one rank, in whole KV groups."""
    sys.path.insert(0, ROOT)
    from long_prefix_attention_b200 import sharding
    for n_chunks in (1, 3, 4, 7, 16):
        runs = [sharding.chunk_shard(n_chunks, world, r) for r in range(world)]
        covered = [c for c0, c1 in runs for c in range(c0, c1)]
        assert covered == list(range(n_chunks))
        assert all(c0 <= c1 for c0, c1 in runs)
    heads = [h for r in range(world) for h in range(*sharding.head_shard(32, 8, world, r))]
    assert heads == list(range(32))


def _split_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import numpy as np
        from long_prefix_attention_b200 import inputs, sharding
        from oracle import asm_oracle as O
        cfg = dict(inputs.CONFIGS[0])
        bi = inputs.build_inputs(cfg, N=96, L=200, K=4)
        Hq, N, d = bi["q"].shape
        bounds = [0, 37, 80, 81, 150, 200]  # five uneven chunks, one of a single key
        kc = [bi["k"][:, b0:b1] for b0, b1 in zip(bounds, bounds[1:])]
        vc = [bi["v"][:, b0:b1] for b0, b1 in zip(bounds, bounds[1:])]

        def encode(q, k, v, s, a, z, acc):  # the oracle's states as the payload
            oa, oz = O.build_states(q, k, v, s, A=a.numpy() if acc else None,
                                    logZ=z.numpy() if acc else None, accumulate=acc)
            a.copy_(torch.from_numpy(oa))
            z.copy_(torch.from_numpy(oz))

        seen = []

        def merge(a, z, a_in, z_in):  # the oracle's merge, row by row, recording the order
            seen.append(float(z_in.sum()))
            A, Z, Ai, Zi = a.numpy().reshape(-1, d), z.numpy().reshape(-1), a_in.numpy().reshape(-1, d), \
                z_in.numpy().reshape(-1)
            for i in range(Z.size):
                m, zz = O.merge(A[i], Z[i], Ai[i], Zi[i])
                A[i], Z[i] = m, zz

        a = torch.zeros(Hq, N, d, dtype=torch.float64)
        z = torch.zeros(Hq, N, dtype=torch.float64)
        sharding.build_states_split(bi["q"], kc, vc, bi["scale"], a, z, encode=encode, merge=merge)
        # what each rank gathered: its own states, in rank order
        own = [None] * world
        c0, c1 = sharding.chunk_shard(len(kc), world, rank)
        dist.all_gather_object(own, (c0, c1))
        ref_a, ref_z = O.build_states(bi["q"], bi["k"], bi["v"], bi["scale"])
        out[rank] = (float(np.abs(a.numpy() - ref_a).max()), float(np.abs(z.numpy() - ref_z).max()), own, seen)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_prefix_chunks_split_over_gloo_ranks_fold_to_the_single_pass(world):
    """Each rank encodes its run of the five prefix chunks, the ranks
    all-gather their states and fold them in chunk order: the result equals
    the single-pass oracle state over the whole prefix on every rank."""
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_split_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        ea, ez, runs, seen = res[r]
        assert ea < 1e-12 and ez < 1e-12
        assert [c for c0, c1 in runs for c in range(c0, c1)] == list(range(5))  # chunk order = rank order
        assert len(seen) == world - 1                                           # one merge per other rank
