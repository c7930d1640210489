"""Benchmark of the ASM hot path on B200.

Headline: the decode step of Attention State Memory at the LLaMA-3.1-8B
single-layer shape (32 query heads, 8 KV heads, head dim 128, K=1024
centroids per head, local KV cache of 2048 tokens, batch 1, bf16).  One
benchmark step decodes one token through 32 such layers, each with its own
memory and KV cache (537 MB in all, more than the 126 MB L2, so every step
streams its bytes from HBM); the 32 layer steps (two kernels each) are
replayed from a CUDA graph.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl asm|reference]
    python bench.py --only states|assign|seed|seed_batched|lloyd|aggregate [--steps K] [--warmup W]
    python bench.py --sweep [--steps K] [--warmup W]
    python bench.py --index [--steps K] [--warmup W]
    python bench.py --whiten [--steps K] [--warmup W]

Prints ONE JSON line (rank 0).  `value` is decode query-heads/s over all
ranks (each rank runs its own independent replica: weak scaling), timed with
CUDA events between barriers; `roofline` is the decode step's algorithmic
HBM bytes per layer over its average time per layer against the measured
HBM copy peak; `e2e` repeats the measurement through the public API with the
per-step queries copied from pinned host memory and the outputs copied back;
`cpu_baseline` times the fp64 oracle on the host cores (a bounded sample);
`build` times the offline memory build at its full shape (32/8 heads,
N=65536, L=16384 in 4 chunks, K=8192, 10 Lloyd rounds).
``--impl reference`` times the fp64 CPU oracle on the same workload.
``--only`` times one build stage alone at the build shape (for profiling a
single kernel) and prints its own JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_prefix_attention_b200 import inputs  # noqa: E402

METRIC = "decode attention query-heads/sec and HBM GB/s vs 8 TB/s; build queries/sec"
NOMINAL_HBM_GBS = 8000.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", 0)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def decode_bytes(B, Hq, Hkv, K, T, d, eb=2):
    """Algorithmic HBM bytes of one decode step of one layer."""
    centroids = Hq * K * d * eb
    local_kv = B * Hkv * T * 2 * d * eb
    gathered = B * Hq * (d * eb + 4)
    q_out = 2 * B * Hq * d * eb
    return centroids + local_kv + gathered + q_out


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"asm_bench_clocks_{os.getpid()}.csv")
        self.gpu = gpu_index

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- distributed --

def torchrun_argv(n_gpus, argv, port):
    """The command that runs this script as `n_gpus` ranks on this node (one
    per GPU), bounded by `timeout` well above the process group's own."""
    return ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n_gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__)] + list(argv)


def launcher_world():
    """WORLD_SIZE set by a launcher (torchrun), or 0 when started directly."""
    return int(os.environ.get("WORLD_SIZE", "0"))


def check_world(n_gpus, world):
    """--gpus N must be the launcher's world size: a mismatch is refused, not
    silently measured on another number of GPUs."""
    if world != n_gpus:
        raise SystemExit(f"bench.py: --gpus {n_gpus} but the launcher started {world} rank(s)")


def dist_setup(n_gpus):
    world = launcher_world() or 1
    check_world(n_gpus, world)
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cuda"):
    """Largest value of `x` over the ranks (every rank gets it)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed_base(rank):
    """Input seed of rank `rank`'s replica: each rank decodes its own layers."""
    return inputs.BASE_SEED + 1000 + 100 * rank


def job_throughput(units_per_rank, secs_per_rank, world, device="cuda"):
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (ranks run the same workload; weak scaling)."""
    return units_per_rank * world / max_over_ranks(secs_per_rank, world, device)


# -------------------------------------------------------------- workloads --

class DecodeStack:
    """`layers` independent C1-shaped layers resident in HBM, one graph per step."""

    def __init__(self, cfg, layers, seed_base, flags=0):
        from long_prefix_attention_b200 import ops
        self.ops = ops
        self.flags = flags
        self.cfg = cfg
        self.layers = []
        for l in range(layers):
            ins = inputs.decode_inputs(cfg, seed=seed_base + l)
            dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in ins.items()}
            B, Hq, d = dev["q"].shape
            _, Hkv, T, _ = dev["k_cache"].shape
            K = dev["centroids"].shape[1]
            dev["ws"] = ops.alloc_workspace(
                ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, d, dev["q"].dtype), "cuda")
            self.layers.append(dev)
        # every layer's queries and outputs are views of one tensor each, so a
        # step's inputs arrive and its results leave in one copy each
        self.q_all = torch.stack([L["q"] for L in self.layers]).contiguous()
        self.out_all = torch.empty_like(self.q_all)
        for i, L in enumerate(self.layers):
            L["q"] = self.q_all[i]
            L["out"] = self.out_all[i]
        self.B, self.Hq, self.d = self.layers[0]["q"].shape
        self.Hkv, self.T = self.layers[0]["k_cache"].shape[1:3]
        self.K = self.layers[0]["centroids"].shape[1]
        self.graph = None

    def launch_all(self):
        for L in self.layers:
            self.ops.asm_decode_step(L["q"], L["centroids"], L["a_bar"], L["logz_bar"], L["k_cache"],
                                     L["v_cache"], L["local_len"], L["scale"], L["out"], L["ws"],
                                     flags=self.flags)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.launch_all()  # warm the per-kernel attributes outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.launch_all()
        torch.cuda.synchronize()

    def step(self):
        self.graph.replay()

    def bytes_per_launch(self):
        return decode_bytes(self.B, self.Hq, self.Hkv, self.K, self.T, self.d)


def time_steps(fn, steps, warmup, world):
    """Seconds for exactly `steps` calls of fn after `warmup` untimed ones,
    CUDA events on the current stream, a barrier and a synchronize on both
    sides (this rank's time; the job's is the max over ranks)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def cpu_decode_baseline(cfg, budget_s=12.0):
    """fp64 oracle decode of C1-shaped layers on the host cores (bounded sample)."""
    from oracle import asm_oracle as O
    ins = inputs.decode_inputs(cfg, seed=inputs.BASE_SEED + 1)
    args = (ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"], ins["k_cache"], ins["v_cache"],
            ins["local_len"], ins["scale"])
    # marshal once (the oracle's own fp64 copies), then time whole-layer calls
    f = [O._f64(a) if torch.is_tensor(a) else a for a in args]
    f[6] = O._i32(ins["local_len"])
    O.decode(*f)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        O.decode(*f)
        n += 1
    dt = time.perf_counter() - t0
    B, Hq = ins["q"].shape[:2]
    return {"value": n * B * Hq / dt, "unit": "query-heads/s", "cores": O.max_threads(), "kind": "oracle",
            "sample": f"{n} single-layer decode steps of the K=1024/T=2048/B=1 layer shape "
                      f"({dt:.1f} s of fp64 CPU work)"}


def cpu_build_baseline(cfg, bi):
    """fp64 oracle of each build stage on the host cores, on bounded samples
    of head 0 at the build shape, extrapolated to the whole build (all heads,
    queries, rounds and Lloyd iterations): states over the full 16384-key
    prefix for 192 queries, one assignment pass of 4096 points against the
    8192 centres, 128 k-means++ rounds, and one head's aggregation."""
    from oracle import asm_oracle as O
    H, N, d = bi["q"].shape
    K, iters = cfg["K"], cfg["iters"]
    Hkv = bi["k"].shape[0]
    q0 = O._f64(bi["q"][0:1])
    k0, v0 = O._f64(bi["k"][0:1]), O._f64(bi["v"][0:1])
    out = {}
    t = time.perf_counter()
    O.build_states(q0[:, :192], k0, v0, bi["scale"])
    ts = time.perf_counter() - t
    out["states_s"] = ts / 192 * N * H
    x0 = q0[0]
    t = time.perf_counter()
    O.assign(x0[:4096], x0[:K])
    ta = time.perf_counter() - t
    out["lloyd_s"] = ta / 4096 * N * H * iters
    u = O._f64(bi["u"][0:1, :128])
    t = time.perf_counter()
    O.kmeanspp_seed(q0, u)
    tk = time.perf_counter() - t
    out["kmeanspp_s"] = tk / 128 * K * H
    lz = np.zeros(N)
    asg = np.arange(N, dtype=np.int32) % K
    t = time.perf_counter()
    O.aggregate(x0, lz, asg, K)
    tg = time.perf_counter() - t
    out["aggregate_s"] = tg * H
    total = sum(out.values())
    return {"value": H * N / total, "unit": "queries/s", "cores": O.max_threads(), "kind": "oracle",
            "extrapolated": True, "stage_s": out,
            "sample": f"head 0 of the build shape: states of 192 queries over all 16384 keys ({ts:.1f} s), one "
                      f"assignment pass of 4096 points against {K} centres ({ta:.1f} s), 128 k-means++ rounds "
                      f"({tk:.1f} s), one head's aggregation ({tg:.1f} s); scaled to {H} heads, {N} queries, "
                      f"{K} rounds and {iters} Lloyd iterations"}


def build_head_shard(Hq, Hkv, world, rank):
    """Query heads [h0, h1) that rank `rank` of `world` builds (whole KV groups)."""
    from long_prefix_attention_b200 import sharding
    return sharding.head_shard(Hq, Hkv, world, rank)


SEED_BATCH = 128  # draws per round of the opt-in batched seeding


def batched_seed_draws(H, K):
    """Draws of the batched seeding: twice K per head, so that rounds that
    drop repeated draws still use fresh ones."""
    return inputs.kmeanspp_uniforms(inputs.BASE_SEED + 4, H, 2 * K)


def run_build(cfg, with_cpu=True, world=1, rank=0):
    """Full offline build at the 32/8-head, N=65536, L=16384, K=8192 shape.
    With several ranks each builds its shard of the heads (heads are
    independent: no data-path exchange); the job's time is the slowest
    rank's, stage by stage."""
    from long_prefix_attention_b200 import ops
    bi = inputs.build_inputs(cfg)
    Htot = bi["q"].shape[0]
    h0, h1 = build_head_shard(Htot, bi["k"].shape[0], world, rank)
    G = Htot // bi["k"].shape[0]
    if h1 == h0:  # nothing to build on this rank: it joins the same collectives
        for _ in range(2):
            barrier(world)  # the two stage_times() calls
        for _ in range(5):
            max_over_ranks(0.0, world)  # the five stage maxima
        return None
    x, u = bi["q"][h0:h1].cuda(), bi["u"][h0:h1].cuda()
    k, v = bi["k"][h0 // G:h1 // G].cuda(), bi["v"][h0 // G:h1 // G].cuda()
    H, N, d = x.shape
    K, iters, L = cfg["K"], cfg["iters"], cfg["L"]
    chunks = cfg["chunks"]
    a = torch.empty_like(x)
    logz = torch.empty(H, N, dtype=torch.float32, device="cuda")
    init = torch.empty(H, K, dtype=torch.int32, device="cuda")
    ws_s = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(H, N, d, K), "cuda", zero=False)
    cen = torch.empty(H, K, d, dtype=torch.float32, device="cuda")
    cdt = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
    assign = torch.empty(H, N, dtype=torch.int32, device="cuda")
    counts = torch.empty(H, K, dtype=torch.int32, device="cuda")
    perm = torch.empty(H, N, dtype=torch.int32, device="cuda")
    seg = torch.empty(H, K + 1, dtype=torch.int32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda", zero=False)
    # the opt-in batched seeding (BATCH draws per round), timed beside the exact one
    ub = batched_seed_draws(Htot, K)[h0:h1].cuda()
    init_b = torch.empty(H, K, dtype=torch.int32, device="cuda")
    ws_b = ops.alloc_workspace(ops.asm_kmeanspp_batched_workspace_size(H, N, d, K, SEED_BATCH), "cuda",
                               zero=False)
    a_bar = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
    lz_bar = torch.empty(H, K, dtype=torch.float32, device="cuda")
    cl = L // chunks
    kc = [k[:, i * cl:(i + 1) * cl].contiguous() for i in range(chunks)]
    vc = [v[:, i * cl:(i + 1) * cl].contiguous() for i in range(chunks)]

    def stage_times():
        barrier(world)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        ev[0].record()
        for i in range(chunks):
            ops.asm_build_states(x, kc[i], vc[i], bi["scale"], a, logz, accumulate=i > 0)
        ev[1].record()
        ops.asm_kmeanspp_seed(x, u, init, ws_s)
        ev[2].record()
        ops.asm_kmeans(x, init, iters, cen, cdt, assign, counts, perm, seg, ws)
        ev[3].record()
        ops.asm_aggregate(a, logz, perm, seg, a_bar, lz_bar)
        ev[4].record()
        ops.asm_kmeanspp_seed_batched(x, ub, init_b, SEED_BATCH, ws_b)
        ev[5].record()
        torch.cuda.synchronize()
        return [ev[i].elapsed_time(ev[i + 1]) for i in range(5)]

    stage_times()  # warm-up
    t = stage_times()
    t = [max_over_ranks(x, world) for x in t]  # the slowest rank, stage by stage
    total = sum(t[:4])
    total_b = total - t[1] + t[4]
    hbm, tf, tfs, src = peaks()
    states_flops = 4.0 * N * L * d * Htot
    assign_flops = 2.0 * N * K * d * Htot * iters
    cpu = cpu_build_baseline(cfg, bi) if with_cpu else None
    return {
        "workload": cfg["name"], "queries": Htot * N, "cpu_baseline": cpu,
        "ranks": world, "heads_per_rank": H,
        "value": Htot * N / (total / 1e3), "unit": "queries/s",
        "ms": {"states_4chunks": t[0], "kmeanspp_seed": t[1], "lloyd_10": t[2], "aggregate": t[3],
               "total": total, f"kmeanspp_seed_batched{SEED_BATCH}": t[4]},
        f"value_with_batched{SEED_BATCH}_seeding": Htot * N / (total_b / 1e3),
        "seeding": f"exact sequential k-means++ (value); batched, {SEED_BATCH} draws per round from one "
                   f"D2 distribution (value_with_batched{SEED_BATCH}_seeding, opt-in)",
        "states_tflops": states_flops / (t[0] / 1e3) / 1e12,
        "states_frac_of_bf16_peak": states_flops / (t[0] / 1e3) / 1e12 / tf,
        "lloyd_assign_tflops_incl_update": assign_flops / (t[2] / 1e3) / 1e12,
        "peak_source": src,
    }


def run_stage(name, steps, warmup):
    """One build stage at the full build shape, `steps` timed launches (for
    profiling single kernels): states = one 4096-key block of the prefix
    (fresh states, no merge); assign = one Lloyd assignment against K
    calibration points; lloyd = the 10 Lloyd rounds (assign + update);
    aggregate = the Z-weighted aggregation; seed = the whole k-means++
    seeding."""
    from long_prefix_attention_b200 import ops
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg)
    x = bi["q"].cuda()
    H, N, d = x.shape
    K, L = cfg["K"], cfg["L"] // cfg["chunks"]
    hbm, tf, tfs, src = peaks()
    if name == "states":
        k, v = bi["k"][:, :L].contiguous().cuda(), bi["v"][:, :L].contiguous().cuda()
        a = torch.empty_like(x)
        logz = torch.empty(H, N, dtype=torch.float32, device="cuda")
        fn = lambda: ops.asm_build_states(x, k, v, bi["scale"], a, logz, accumulate=False)
        flops = 4.0 * N * L * d * H
    elif name == "assign":
        g = torch.Generator().manual_seed(5)
        pick = torch.stack([torch.randperm(N, generator=g)[:K] for _ in range(H)])
        cdt = x[torch.arange(H, device="cuda")[:, None], pick.cuda()].contiguous()
        assign = torch.empty(H, N, dtype=torch.int32, device="cuda")
        ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda")
        fn = lambda: ops.asm_kmeans_assign(x, cdt, assign, ws)
        flops = 2.0 * N * K * d * H
    elif name in ("lloyd", "aggregate"):
        g = torch.Generator().manual_seed(5)
        init = torch.stack([torch.randperm(N, generator=g)[:K] for _ in range(H)]).to(torch.int32).cuda()
        cen = torch.empty(H, K, d, dtype=torch.float32, device="cuda")
        cdt = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
        assign = torch.empty(H, N, dtype=torch.int32, device="cuda")
        counts = torch.empty(H, K, dtype=torch.int32, device="cuda")
        perm = torch.empty(H, N, dtype=torch.int32, device="cuda")
        seg = torch.empty(H, K + 1, dtype=torch.int32, device="cuda")
        ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda")
        iters = cfg["iters"]
        if name == "lloyd":
            fn = lambda: ops.asm_kmeans(x, init, iters, cen, cdt, assign, counts, perm, seg, ws)
            flops = 2.0 * N * K * d * H * iters
        else:
            ops.asm_kmeans(x, init, 1, cen, cdt, assign, counts, perm, seg, ws)
            a = torch.randn(H, N, d, device="cuda").to(x.dtype)
            logz = torch.rand(H, N, device="cuda") * 5 + 5
            a_bar = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
            lz_bar = torch.empty(H, K, dtype=torch.float32, device="cuda")
            fn = lambda: ops.asm_aggregate(a, logz, perm, seg, a_bar, lz_bar)
            flops = None
    elif name == "seed_batched":
        u = batched_seed_draws(H, K).cuda()
        init = torch.empty(H, K, dtype=torch.int32, device="cuda")
        ws = ops.alloc_workspace(ops.asm_kmeanspp_batched_workspace_size(H, N, d, K, SEED_BATCH), "cuda",
                                 zero=False)
        fn = lambda: ops.asm_kmeanspp_seed_batched(x, u, init, SEED_BATCH, ws)
        flops = None
    else:
        u = bi["u"].cuda()
        init = torch.empty(H, K, dtype=torch.int32, device="cuda")
        ws = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(H, N, d, K), "cuda", zero=False)
        fn = lambda: ops.asm_kmeanspp_seed(x, u, init, ws)
        flops = None
    for _ in range(max(1, warmup)):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    out = {"stage": name, "workload": cfg["name"], "ms_per_launch": ms, "steps": steps}
    if flops is not None:
        out.update({"tflops": flops / (ms / 1e3) / 1e12, "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / tf,
                    "peak_tflops": tf, "peak_source": src})
    print(json.dumps(out))


def run_sweep(steps, warmup):
    """ASM decode over the 36-point grid of the 32-layer sweep (B x K x T at the
    LLaMA layer shape), each point against full attention over an explicit
    32K prefix plus the same local tokens (timed once per (B, T)).  Each point cycles enough distinct layer
    buffers (at least two, at least 3x L2 in all, at most the layer count and
    60% of free HBM) that every step streams from HBM; inputs are generated on
    the device.  Times are CUDA events around `steps` graph replays of all
    layers, after `warmup` replays."""
    from long_prefix_attention_b200 import ops
    cfg = inputs.CONFIGS[4]
    layers, Hq, Hkv, d, Lp = cfg["layers"], cfg["Hq"], cfg["Hkv"], cfg["d"], cfg["Lp"]
    hbm, tf, tfs, src = peaks()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size

    def time_graph(run_layer, nbuf):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(nbuf):
                run_layer(i)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for l in range(layers):
                run_layer(l % nbuf)
        secs = time_steps(g.replay, steps, max(3, warmup), 1)
        del g
        return secs / (steps * layers)

    def nbuf_for(bytes_per_layer, mem_per_layer):
        free, _ = torch.cuda.mem_get_info()
        n = max(2, math.ceil(3 * l2 / bytes_per_layer))
        return max(1, min(layers, n, int(0.6 * free // mem_per_layer)))

    points = []
    full = {}
    for B in cfg["B"]:
        for K in cfg["K"]:
            for T in cfg["T"]:
                byt = decode_bytes(B, Hq, Hkv, K, T, d)
                mem = 2 * Hq * K * d * 2 + Hq * K * 4 + 2 * B * Hkv * T * d * 2
                nbuf = nbuf_for(byt, mem)
                bufs = []
                for i in range(nbuf):
                    L = inputs.decode_layer_device(cfg, inputs.BASE_SEED + 5000 + i, B, K, T)
                    L["out"] = torch.empty_like(L["q"])
                    L["ws"] = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, d, L["q"].dtype),
                                                  "cuda")
                    bufs.append(L)

                def asm_layer(i, bufs=bufs):
                    L = bufs[i]
                    ops.asm_decode_step(L["q"], L["centroids"], L["a_bar"], L["logz_bar"], L["k_cache"],
                                        L["v_cache"], L["local_len"], L["scale"], L["out"], L["ws"], flags=1)

                per = time_graph(asm_layer, nbuf)
                pt = {"B": B, "K": K, "T": T, "asm_us_per_layer": per * 1e6, "asm_bytes_per_layer": byt,
                      "asm_gbs": byt / per / 1e9, "asm_frac_of_hbm": byt / per / 1e9 / hbm, "buffers": nbuf}
                del bufs
                torch.cuda.empty_cache()
                key = (B, T)
                if key not in full:
                    # full attention: the explicit prefix plus the same local tokens
                    fbyt = Hkv * Lp * 2 * d * 2 + B * Hkv * T * 2 * d * 2 + 2 * B * Hq * d * 2
                    fmem = 2 * Hkv * Lp * d * 2 + 2 * B * Hkv * T * d * 2
                    fnb = nbuf_for(fbyt, fmem)
                    fb = []
                    for i in range(fnb):
                        L = inputs.decode_layer_device(cfg, inputs.BASE_SEED + 6000 + i, B, 1, T, Lp=Lp)
                        L["out"] = torch.empty_like(L["q"])
                        L["ws"] = ops.alloc_workspace(
                            ops.asm_flash_decode_workspace_size(B, Hq, Hkv, Lp, T, d, L["q"].dtype), "cuda")
                        fb.append(L)

                    def fa_layer(i, fb=fb):
                        L = fb[i]
                        ops.asm_flash_decode(L["q"], L["k_prefix"], L["v_prefix"], L["k_cache"], L["v_cache"],
                                             L["local_len"], L["scale"], L["out"], L["ws"])

                    fper = time_graph(fa_layer, fnb)
                    full[key] = (fper, fbyt)
                    del fb
                    torch.cuda.empty_cache()
                fper, fbyt = full[key]
                pt.update({"full_us_per_layer": fper * 1e6, "full_bytes_per_layer": fbyt,
                           "full_gbs": fbyt / fper / 1e9, "speedup_vs_full": fper / per})
                points.append(pt)
                print(json.dumps(pt), file=sys.stderr, flush=True)
    line = {"sweep": cfg["name"], "layers": layers, "prefix_len_full_attention": Lp, "steps": steps,
            "warmup": max(3, warmup), "hbm_peak_gbs": hbm, "peak_source": src,
            "note": "full attention: the batch rows that read one prefix tile run together, so the "
                    "tile streams from HBM once and from L2 for the other rows",
            "points": points}
    print(json.dumps(line))


def run_index(steps, warmup, Ps=(4, 8, 16)):
    """Two-level (hierarchical) search against the flat search at the LLaMA
    layer shape (B = 1, T = 2048) for K in {1024, 4096, 8192, 16384}: centres
    drawn from a Gaussian mixture (clustered like k-means centres of real
    queries), index built by the library's k-means on the centres with
    K1 = round(sqrt(K)) clusters, memory ordered by cluster.  Times are per
    layer step over 32 layers in one graph (distinct buffers cycled, each step
    from HBM); recall@1 is the fraction of 64 x 32 queries from the same
    mixture whose indexed retrieval equals the flat one."""
    from long_prefix_attention_b200 import ops
    cfg = dict(inputs.CONFIGS[1])
    Hq, Hkv, d, T, layers = cfg["Hq"], cfg["Hkv"], cfg["d"], cfg["T"], 32
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    hbm, tf, tfs, src = peaks()

    def mix(g, n, means):
        comp = torch.randint(0, means.shape[1], (Hq, n), generator=g, device="cuda")
        x = means[torch.arange(Hq, device="cuda")[:, None], comp]
        return (x + 0.3 * torch.randn(Hq, n, d, generator=g, device="cuda")).to(torch.bfloat16)

    def graph_time(run, nbuf):
        run_all = lambda: [run(i % nbuf) for i in range(layers)]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run_all()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            run_all()
        secs = time_steps(gr.replay, steps, max(3, warmup), 1)
        del gr
        return secs / (steps * layers)

    rows = []
    for K in (1024, 4096, 8192, 16384):
        K1 = int(round(math.sqrt(K)))
        per_layer = 2 * Hq * K * d * 2 + Hkv * T * 2 * d * 2
        nbuf = min(layers, max(2, math.ceil(3 * l2 / per_layer)))
        bufs = []
        for i in range(nbuf):
            g = torch.Generator(device="cuda")
            g.manual_seed(inputs.BASE_SEED + 7000 + i)
            means = torch.randn(Hq, 1024, d, generator=g, device="cuda")
            L = inputs.decode_layer_device(cfg, inputs.BASE_SEED + 7100 + i, 1, K, T)
            x = mix(g, K, means)
            u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 7200 + i, Hq, K1).cuda()
            init = torch.empty(Hq, K1, dtype=torch.int32, device="cuda")
            wss = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(Hq, K, d, K1), "cuda", zero=False)
            ops.asm_kmeanspp_seed(x, u, init, wss)
            c = torch.empty(Hq, K1, d, dtype=torch.float32, device="cuda")
            sdt = torch.empty(Hq, K1, d, dtype=torch.bfloat16, device="cuda")
            asg = torch.empty(Hq, K, dtype=torch.int32, device="cuda")
            cnt = torch.empty(Hq, K1, dtype=torch.int32, device="cuda")
            perm = torch.empty(Hq, K, dtype=torch.int32, device="cuda")
            seg = torch.empty(Hq, K1 + 1, dtype=torch.int32, device="cuda")
            wsk = ops.alloc_workspace(ops.asm_kmeans_workspace_size(Hq, K, d, K1), "cuda")
            ops.asm_kmeans(x, init, 4, c, sdt, asg, cnt, perm, seg, wsk)
            co, ao, lo = torch.empty_like(x), torch.empty_like(L["a_bar"]), torch.empty_like(L["logz_bar"])
            ops.asm_index_reorder(perm, x, L["a_bar"], L["logz_bar"], co, ao, lo)
            L.update(centroids=co, a_bar=ao, logz_bar=lo, supers=sdt, seg=seg, max_seg=int(cnt.max().item()),
                     q=mix(g, 1, means).transpose(0, 1).contiguous(), out=torch.empty(1, Hq, d, dtype=torch.bfloat16,
                                                                                      device="cuda"))
            L["ws"] = ops.alloc_workspace(ops.asm_decode_workspace_size(1, Hq, Hkv, K, T, d, torch.bfloat16), "cuda")
            bufs.append(L)
            if i == 0:
                qr = mix(g, 64, means).transpose(0, 1).contiguous()
        torch.cuda.synchronize()

        def flat(i):
            L = bufs[i]
            ops.asm_decode_step(L["q"], L["centroids"], L["a_bar"], L["logz_bar"], L["k_cache"], L["v_cache"],
                                L["local_len"], L["scale"], L["out"], L["ws"], flags=1)

        t_flat = graph_time(flat, nbuf)
        row = {"K": K, "K1": K1, "flat_us_per_layer": t_flat * 1e6, "buffers": nbuf, "indexed": []}
        L0 = bufs[0]
        kc64 = torch.zeros(64, Hkv, T, d, dtype=torch.bfloat16, device="cuda")
        ll64 = torch.full((64,), 1, dtype=torch.int32, device="cuda")
        ws64 = ops.alloc_workspace(ops.asm_decode_workspace_size(64, Hq, Hkv, K, T, d, torch.bfloat16), "cuda")
        i_flat = torch.empty(64, Hq, dtype=torch.int32, device="cuda")
        o64 = torch.empty_like(qr)
        ops.asm_decode_step(qr, L0["centroids"], L0["a_bar"], L0["logz_bar"], kc64, kc64, ll64, L0["scale"], o64,
                            ws64, idx_out=i_flat)
        for P in Ps:
            for L in bufs:
                L["wsi"] = ops.alloc_workspace(ops.asm_decode_indexed_workspace_size(
                    1, Hq, Hkv, K1, P, L["max_seg"], T, d, torch.bfloat16), "cuda")

            def indexed(i, P=P):
                L = bufs[i]
                ops.asm_decode_step_indexed(L["q"], L["supers"], L["seg"], P, L["max_seg"], L["centroids"],
                                            L["a_bar"], L["logz_bar"], L["k_cache"], L["v_cache"], L["local_len"],
                                            L["scale"], L["out"], L["wsi"])

            t_idx = graph_time(indexed, nbuf)
            wsr = ops.alloc_workspace(ops.asm_decode_indexed_workspace_size(
                64, Hq, Hkv, K1, P, L0["max_seg"], T, d, torch.bfloat16), "cuda")
            i_idx = torch.empty_like(i_flat)
            ops.asm_decode_step_indexed(qr, L0["supers"], L0["seg"], P, L0["max_seg"], L0["centroids"], L0["a_bar"],
                                        L0["logz_bar"], kc64, kc64, ll64, L0["scale"], o64, wsr, idx_out=i_idx)
            torch.cuda.synchronize()
            recall = (i_idx == i_flat).float().mean().item()
            row["indexed"].append({"P": P, "us_per_layer": t_idx * 1e6, "speedup": t_flat / t_idx,
                                   "recall_at_1": recall})
        rows.append(row)
        print(json.dumps(row), file=sys.stderr, flush=True)
        del bufs
        torch.cuda.empty_cache()
    print(json.dumps({"index": "two-level search vs flat, LLaMA layer shape, B=1, T=2048, 32 layers",
                      "steps": steps, "warmup": max(3, warmup), "rows": rows}))


# -------------------------------------------------------------------- main --

def run_whiten(steps, warmup, layers=16):
    """Whitened retrieval.  Build shape: the whitening of the 32 x 65536
    calibration queries (fp64 moments and inverse square root) and their
    transform.  LLaMA layer shape (K = 1024, T = 2048, B = 1): the decode step
    with the whitened search (the query's transform, then the step searching
    with it against whitened centres) against the plain step, `layers`
    distinct layers per graph so every step streams from HBM."""
    from long_prefix_attention_b200 import ops
    bi = inputs.build_inputs(inputs.CONFIGS[3])
    x = bi["q"].cuda()
    H, N, d = x.shape
    mu = torch.empty(H, d, dtype=torch.float32, device="cuda")
    W = torch.empty(H, d, d, dtype=torch.float32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_whitening_workspace_size(H, d), "cuda")
    y = torch.empty_like(x)

    def ev_time(fn, n):
        for _ in range(max(1, warmup // 4)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    t_wh = ev_time(lambda: ops.asm_whitening(x, mu, W, ws), 3)
    err = ops.asm_workspace_error(ws)
    t_ap = ev_time(lambda: ops.asm_whiten(x, mu, W, y), 3)
    del y, x
    cfg = inputs.CONFIGS[1]
    stack = DecodeStack(cfg, layers, inputs.BASE_SEED + 500)
    for L in stack.layers:  # the memory's centres, whitened once with the heads' W
        L["cw"] = torch.empty_like(L["centroids"])
        ops.asm_whiten(L["centroids"], mu, W, L["cw"], layout="heads")
        L["qs"] = torch.empty_like(L["q"])

    def whitened_all():
        for L in stack.layers:
            ops.asm_whiten(L["q"], mu, W, L["qs"], layout="batch")
            ops.asm_decode_step_search(L["q"], L["qs"], L["cw"], L["a_bar"], L["logz_bar"], L["k_cache"],
                                       L["v_cache"], L["local_len"], L["scale"], L["out"], L["ws"])

    def graph_of(fn):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g

    g_plain = graph_of(stack.launch_all)
    g_wh = graph_of(whitened_all)
    t_plain = time_steps(g_plain.replay, steps, warmup, 1) / steps / layers * 1e6
    t_white = time_steps(g_wh.replay, steps, warmup, 1) / steps / layers * 1e6
    print(json.dumps({
        "whiten": "ZCA whitening of the calibration queries and the decode step with the whitened search",
        "build": {"workload": inputs.CONFIGS[3]["name"], "whitening_ms": t_wh, "whitening_error": err,
                  "moments_read_gbs": x_bytes(H, N, d) / (t_wh / 1e3) / 1e9, "transform_ms": t_ap,
                  "transform_gbs": 2 * x_bytes(H, N, d) / (t_ap / 1e3) / 1e9},
        "decode": {"workload": cfg["name"] + f" x {layers} layers", "plain_us_per_layer": t_plain,
                   "whitened_search_us_per_layer": t_white, "steps": steps, "warmup": warmup}}))


def x_bytes(H, N, d):
    return H * N * d * 2


# ----------------------------------------------------------------- traffic --

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per layer step,
# summed over the step's two kernels (mean of 8 layer steps of one ncu
# capture of this benchmark), with the digest of the kernel source they were
# taken on: a changed kernel reports null until it is measured again.
TRAFFIC = {
    "llama31-8b-layer-decode-K1024-T2048-B1": {  # units 16 943 872 + merge 577 504
        "bytes": 17521376, "source": "34fb8ab3bad75454"},
    "llama31-8b-layer-decode-K8192-T4096-B16": {  # units 356 988 672 + merge 17 535 872
        "bytes": 374524544, "source": "34fb8ab3bad75454"},
}
TRAFFIC_SOURCE = os.path.join(ROOT, "long_prefix_attention_b200", "csrc", "decode_tc.cu")


def source_digest(path):
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(key):
    rec = TRAFFIC.get(key)
    if rec is None or rec["source"] != source_digest(TRAFFIC_SOURCE):
        return None
    return rec["bytes"]


# ------------------------------------------------------------- JSON line --

def decode_line(value, ms_per_step, world, steps, warmup, config, roofline, e2e, launches, clocks,
                cpu=None, build=None, extra=None):
    """The benchmark's JSON line (rank 0 prints it)."""
    line = {
        "metric": METRIC, "value": value, "unit": "query-heads/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config,
        "hbm_gbs": roofline["achieved"], "hbm_frac_of_8tbs": roofline["achieved"] / NOMINAL_HBM_GBS,
        "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        "cpu_baseline": cpu, "build": build,
    }
    if extra:
        line.update(extra)
    return line


def decode_roofline(bytes_per_launch, us_per_launch, peak, peak_src, traffic, kernel):
    achieved = bytes_per_launch / (us_per_launch * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel, "bytes_per_launch": bytes_per_launch,
            "us_per_launch": us_per_launch, "peak_source": f"{peak_src} HBM copy"}


def run_decode_large(cfg, layers, steps, warmup, world, rank, hbm, src):
    """The largest single-GPU decode configuration (K = 8192, T = 4096, B = 16,
    where the search is a [16 x 128] x [128 x 8192] product per head): the
    same 32-layer graph as the headline, inputs generated on the device."""
    from long_prefix_attention_b200 import ops
    B, K, T = cfg["B"], cfg["K"], cfg["T"]
    Hq, Hkv, d = cfg["Hq"], cfg["Hkv"], cfg["d"]
    bufs = []
    for l in range(layers):
        L = inputs.decode_layer_device(cfg, replica_seed_base(rank) + 500 + l, B, K, T)
        L["out"] = torch.empty_like(L["q"])
        L["ws"] = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, d, L["q"].dtype), "cuda")
        bufs.append(L)

    def run_all():
        for L in bufs:
            ops.asm_decode_step(L["q"], L["centroids"], L["a_bar"], L["logz_bar"], L["k_cache"], L["v_cache"],
                                L["local_len"], L["scale"], L["out"], L["ws"], flags=1)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_all()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_all()
    secs = max_over_ranks(time_steps(g.replay, steps, max(3, warmup), world), world)
    del g
    per = secs / (steps * layers)
    byt = decode_bytes(B, Hq, Hkv, K, T, d)
    err = max(ops.asm_workspace_error(L["ws"]) for L in bufs)
    launches = ops.asm_decode_step_launches(B, Hq, Hkv, K, T, d, torch.bfloat16)
    out = {"workload": cfg["name"] + f" x {layers} layers", "K": K, "local_len": T, "batch": B,
           "value": B * Hq * layers * steps * world / secs, "unit": "query-heads/s",
           "ms_per_step": secs * 1e3 / steps, "gpu_launches": steps * layers * launches,
           "device_error_word": err,
           "roofline": decode_roofline(byt, per * 1e6, hbm, src, recorded_traffic(cfg["name"]),
                                       "asm_decode_step = asm_decode_units<128,4> + asm_decode_merge<128,32>")}
    del bufs
    torch.cuda.empty_cache()
    return out


# ncu's sm__pipe_tensor_cycles_active (percent of active cycles) of the build
# stages' tensor-core kernels, from one `--set full` capture each (the
# profiles named), with the digest of the kernel's source text they were taken
# on: a changed kernel reports null until it is captured again.
NCU_TENSOR = {
    "states": {"pct": 52.2, "profile": "profiles/states_tc_build_n65536_l4096.md",
               "file": "build_states_tc.cu", "begin": "states_tc_kernel(const __grid_constant__",
               "end": "}  // namespace stc", "source": "36063807717c30d6"},
    "lloyd": {"pct": 59.7, "profile": "profiles/assign_tc_build_n65536_k8192.md",
              "file": "assign_tc.cu", "begin": "assign_tc_kernel(const __grid_constant__",
              "end": "}  // namespace atc", "source": "d76c541cd98fb6cd"},
}


def kernel_digest(name, begin, end):
    import hashlib
    with open(os.path.join(ROOT, "long_prefix_attention_b200", "csrc", name)) as f:
        text = f.read()
    i = text.find(begin)
    j = text.find(end, i) if i >= 0 else -1
    if i < 0 or j < 0:
        return None
    return hashlib.sha256(text[i:j].encode()).hexdigest()[:16]


def recorded_tensor_pipe(stage):
    rec = NCU_TENSOR[stage]
    if rec["pct"] is None or kernel_digest(rec["file"], rec["begin"], rec["end"]) != rec["source"]:
        return None
    return {"sm__pipe_tensor_cycles_active_pct": rec["pct"], "profile": rec["profile"]}


def build_rooflines(build, tf, hbm, src):
    """Each build stage against the roofline that bounds it: the states and
    the assignment on the bf16 tensor peak (flops of the definition), the
    aggregation on the HBM copy rate (one read of the member states, logZ and
    the member lists, one write of the cluster states); the seeding is K
    dependent rounds and is reported as time per round."""
    cfg = inputs.CONFIGS[3]
    H, N, d, K, L, iters = cfg["Hq"], cfg["N"], cfg["d"], cfg["K"], cfg["L"], cfg["iters"]
    ms = build["ms"]
    states = 4.0 * N * L * d * H / (ms["states_4chunks"] / 1e3) / 1e12
    lloyd = 2.0 * N * K * d * H * iters / (ms["lloyd_10"] / 1e3) / 1e12
    agg_bytes = H * N * (d * 2 + 4 + 4) + H * K * (d * 2 + 4)
    agg = agg_bytes / (ms["aggregate"] / 1e3) / 1e9
    return {
        "states": {"bound": "tensor", "achieved": states, "peak": tf, "unit": "TFLOP/s", "frac": states / tf,
                   "peak_source": f"{src} bf16", "flops": 4.0 * N * L * d * H,
                   "ncu": recorded_tensor_pipe("states")},
        "lloyd": {"bound": "tensor", "achieved": lloyd, "peak": tf, "unit": "TFLOP/s", "frac": lloyd / tf,
                  "peak_source": f"{src} bf16", "flops": 2.0 * N * K * d * H * iters,
                  "note": "assignment flops over the 10 rounds, update included in the time",
                  "ncu": recorded_tensor_pipe("lloyd")},
        "aggregate": {"bound": "hbm", "achieved": agg, "peak": hbm, "unit": "GB/s", "frac": agg / hbm,
                      "peak_source": f"{src} HBM copy", "bytes": agg_bytes},
        "kmeanspp_seed": {"bound": "sequential rounds", "rounds": K,
                          "us_per_round": ms["kmeanspp_seed"] * 1e3 / K},
        f"kmeanspp_seed_batched{SEED_BATCH}": batched_seed_roofline(
            ms[f"kmeanspp_seed_batched{SEED_BATCH}"], H, N, d, K, hbm, src),
    }


def batched_seed_roofline(ms, H, N, d, K, hbm, src):
    """Per round of the batched seeding (bf16, d = 128: one fused kernel): the
    points are read once, D2 and |x|^2 are read and D2 is written back:
    H * N * (2 d + 20) bytes (the round's centres, draws and range sums are
    negligible; D2 is written only where it changed, so this is an upper
    bound on the writes).  The time per round includes the pick kernel."""
    rounds = (K - 1 + SEED_BATCH - 1) // SEED_BATCH
    per_round = H * N * (2 * d + 20)
    us = ms * 1e3 / rounds
    achieved = per_round / (us * 1e-6) / 1e9
    return {"bound": "hbm", "rounds": rounds, "us_per_round": us, "bytes_per_round": per_round,
            "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "peak_source": f"{src} HBM copy", "note": "round time includes the pick kernel"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="asm", choices=["asm", "reference"])
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--no-build", action="store_true", help="skip the offline-build measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--no-large", action="store_true", help="skip the K=8192/T=4096/B=16 decode entry")
    ap.add_argument("--no-prefetch", action="store_true",
                    help="do not let a layer's kernel stream its (static) centroids before the "
                         "preceding kernel finishes")
    ap.add_argument("--only", choices=["states", "assign", "seed", "seed_batched", "lloyd", "aggregate"],
                    help="time one build stage alone (single-kernel profiling) and exit")
    ap.add_argument("--index", action="store_true",
                    help="two-level (hierarchical) search against the flat search (time and recall) and exit")
    ap.add_argument("--whiten", action="store_true",
                    help="whitening at the build shape and the decode step with the whitened search, and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="decode over the 36-point B x K x T grid (and full attention at B=1) and exit")
    ap.add_argument("--decode-large", action="store_true",
                    help="only the K=8192/T=4096/B=16 decode entry (one GPU), printed as its own line")
    args = ap.parse_args()
    if args.only:
        run_stage(args.only, args.steps, args.warmup)
        return
    if args.sweep:
        run_sweep(args.steps, args.warmup)
        return
    if args.index:
        run_index(args.steps, args.warmup)
        return
    if args.whiten:
        run_whiten(args.steps, args.warmup)
        return
    if args.decode_large:
        torch.cuda.set_device(0)
        hbm, _, _, src = peaks()
        print(json.dumps(run_decode_large(inputs.CONFIGS[2], args.layers, args.steps, max(3, args.warmup), 1, 0,
                                          hbm, src)))
        return
    if args.gpus > 1 and launcher_world() == 0:
        # started directly: run as N ranks, one per GPU, and hand back their status
        with __import__("socket").socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        sys.exit(subprocess.call(torchrun_argv(args.gpus, sys.argv[1:], port)))
    cfg = inputs.CONFIGS[1]
    if args.impl == "reference":
        # the fp64 oracle on the host cores: rank 0 alone (the others exit without work)
        world = launcher_world() or 1
        check_world(args.gpus, world)
        if int(os.environ.get("RANK", "0")) != 0:
            return
        config = {"workload": cfg["name"] + f" x {args.layers} layers", "layers": args.layers,
                  "Hq": cfg["Hq"], "Hkv": cfg["Hkv"], "d": cfg["d"], "K": cfg["K"], "local_len": cfg["T"],
                  "batch": cfg["B"], "parallelism": f"replicas x{world}"}
        cb = cpu_decode_baseline(cfg, budget_s=max(3.0, min(20.0, 0.05 * args.steps)))
        line = {"metric": METRIC, "value": cb["value"], "unit": "query-heads/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "impl": "reference",
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "query-heads/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    world, rank, local = dist_setup(args.gpus)
    hbm, tf, tfs, peak_src = peaks()
    config = {"workload": cfg["name"] + f" x {args.layers} layers", "layers": args.layers,
              "Hq": cfg["Hq"], "Hkv": cfg["Hkv"], "d": cfg["d"], "K": cfg["K"], "local_len": cfg["T"],
              "batch": cfg["B"], "l2": f"inputs larger than L2: {args.layers} distinct layer buffers",
              "parallelism": f"replicas x{world}"}
    flags = 0 if args.no_prefetch else 1  # ASM_DECODE_PREFETCH_CENTROIDS
    config["prefetch_centroids"] = bool(flags)
    stack = DecodeStack(cfg, args.layers, seed_base=replica_seed_base(rank), flags=flags)
    stack.capture()
    warmup = max(3, args.warmup)
    with ClockSampler(local) as clk:
        secs_rank = time_steps(stack.step, args.steps, warmup, world)
    value = job_throughput(stack.B * stack.Hq * args.layers * args.steps, secs_rank, world)
    secs = max_over_ranks(secs_rank, world)
    per_step_launches = stack.ops.asm_decode_step_launches(stack.B, stack.Hq, stack.Hkv, stack.K, stack.T,
                                                           stack.d, torch.bfloat16)
    launches = args.steps * args.layers * per_step_launches
    ms_per_step = secs * 1e3 / args.steps
    per_launch_s = secs / (args.steps * args.layers)  # one decode step (both kernels) of one layer
    roofline = decode_roofline(stack.bytes_per_launch(), per_launch_s * 1e6, hbm, peak_src,
                               recorded_traffic(cfg["name"]),
                               "asm_decode_step = asm_decode_units<128,4> + asm_decode_merge<128,16>")

    # end to end through the public API: every step copies that step's queries
    # from pinned host memory and reads its outputs back.  "graph": the layer
    # steps replayed from the captured CUDA graph; "eager": asm_decode_step
    # called layer by layer (host-side validation and launch every call).
    qh_host = stack.q_all.cpu().pin_memory()
    out_host = torch.empty_like(qh_host).pin_memory()

    def e2e_graph():
        stack.q_all.copy_(qh_host, non_blocking=True)
        stack.graph.replay()
        out_host.copy_(stack.out_all, non_blocking=True)

    def e2e_eager():
        stack.q_all.copy_(qh_host, non_blocking=True)
        stack.launch_all()
        out_host.copy_(stack.out_all, non_blocking=True)

    e2e_steps = max(10, args.steps // 4)
    e2e_secs = max_over_ranks(time_steps(e2e_graph, e2e_steps, 3, world), world)
    eager_secs = max_over_ranks(time_steps(e2e_eager, e2e_steps, 3, world), world)
    h2d = qh_host[0].numel() * qh_host.element_size() * args.layers
    d2h = h2d
    units = stack.B * stack.Hq * args.layers * e2e_steps * world
    e2e = {"value": units / e2e_secs, "unit": "query-heads/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "path": "CUDA graph of the layer steps between the two copies",
           "eager_value": units / eager_secs,
           "eager_path": "asm_decode_step called per layer (validation and launches every call)"}

    large = None
    if not args.no_large:
        try:
            large = run_decode_large(inputs.CONFIGS[2], args.layers, max(5, args.steps // 10), warmup, world,
                                     rank, hbm, peak_src)
        except Exception as e:  # report, do not hide
            large = {"error": repr(e)}

    build = None
    if not args.no_build:
        # every rank builds its shard of the heads (the same collectives on
        # every rank: barriers and the per-stage max over ranks)
        try:
            build = run_build(inputs.CONFIGS[3], with_cpu=not args.no_cpu and world == 1, world=world,
                              rank=rank)
            if build is not None:
                build["roofline"] = build_rooflines(build, tf, hbm, peak_src)
        except Exception as e:  # report, do not hide
            build = {"error": repr(e)}
    cpu = None
    if not args.no_cpu and rank == 0 and world == 1:
        cpu = cpu_decode_baseline(cfg)

    if rank == 0:
        line = decode_line(value, ms_per_step, world, args.steps, warmup, config, roofline, e2e, launches,
                           clk.summary(), cpu=cpu, build=build, extra={"decode_large": large})
        print(json.dumps(line))
    if world > 1:
        stack.graph = None
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
