"""Parity of the memory-build calls (CUDA, through the C ABI) with the fp64
oracle: prefix states with the chunk merge ("Recoleccion", "Eficiencia"),
k-means++ seeding and Lloyd iterations ("Agrupamiento"), centroid means and
Z-weighted state aggregation ("Agregacion") of "Context Memorization for
Efficient Long Context Generation", Metodologia.

k-means is chaotic, so it is checked by teacher forcing: every iteration
the oracle is handed the GPU's own storage-dtype centres and the GPU's
assignment/update are compared with the oracle's on exactly those.
"""
import numpy as np
import pytest
import torch

from long_prefix_attention_b200 import inputs, ops
from oracle import asm_oracle as O

from gpu_common import TOL, check_indices, dev, f64, host, max_abs

pytestmark = pytest.mark.gpu


def gpu_states(q, k, v, scale, chunks=1):
    Hq, N, d = q.shape
    L = k.shape[1]
    a = torch.empty_like(q)
    logz = torch.empty(Hq, N, dtype=torch.float32, device=q.device)
    bounds = np.linspace(0, L, chunks + 1).astype(int)
    for c in range(chunks):
        lo, hi = bounds[c], bounds[c + 1]
        ops.asm_build_states(q, k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(), scale, a, logz,
                             accumulate=c > 0)
    torch.cuda.synchronize()
    return a, logz


@pytest.mark.parametrize("chunks", [1, 4])
def test_states_tiny_fp32_config(chunks):
    cfg = inputs.CONFIGS[0]
    bi = inputs.build_inputs(cfg)
    a, logz = gpu_states(dev(bi["q"]), dev(bi["k"]), dev(bi["v"]), bi["scale"], chunks)
    oa, olz = O.build_states(bi["q"], bi["k"], bi["v"], bi["scale"])
    assert max_abs(f64(a), oa) <= 1e-4
    assert max_abs(f64(logz), olz) <= 1e-4


@pytest.mark.parametrize("dt,d,Hq,Hkv,N,L", [("bf16", 128, 8, 2, 300, 700), ("bf16", 64, 4, 4, 129, 257),
                                            ("f32", 128, 8, 1, 77, 1000), ("bf16", 128, 16, 2, 200, 1)])
def test_states_shapes(dt, d, Hq, Hkv, N, L):
    cfg = dict(inputs.CONFIGS[3], dtype=dt, d=d, Hq=Hq, Hkv=Hkv, n_mix=8)
    bi = inputs.build_inputs(cfg, seed=d + N, N=N, L=L, K=4)
    for chunks in (1, 3) if L >= 3 else (1,):
        a, logz = gpu_states(dev(bi["q"]), dev(bi["k"]), dev(bi["v"]), bi["scale"], chunks)
        oa, olz = O.build_states(bi["q"], bi["k"], bi["v"], bi["scale"])
        tol = TOL[bi["q"].dtype]
        assert max_abs(f64(a), oa) <= tol
        assert max_abs(f64(logz), olz) <= tol


def test_states_running_max_rises():
    """Key norms grow along the prefix, so later key tiles raise the row
    maximum by many units: exercises the rescale of the stored numerator."""
    cfg = dict(inputs.CONFIGS[3], Hq=2, Hkv=1, n_mix=8)
    bi = inputs.build_inputs(cfg, seed=11, N=300, L=1000, K=4)
    ramp = torch.linspace(0.1, 6.0, 1000, dtype=torch.float64)[None, :, None]
    k = (bi["k"].to(torch.float64) * ramp).to(torch.bfloat16)
    for chunks in (1, 2):
        a, logz = gpu_states(dev(bi["q"]), dev(k), dev(bi["v"]), bi["scale"], chunks)
        oa, olz = O.build_states(bi["q"], k, bi["v"], bi["scale"])
        assert max_abs(f64(a), oa) <= 2e-2
        assert max_abs(f64(logz), olz) <= 2e-2


def test_states_llama_build_config_every_head_and_tile():
    """Full build shape (32/8 heads, N=65536, L=16384 as 4 chunks of 4096)
    against the single-pass oracle on one row of every 128-query tile of
    every head: 512 rows per head, 16384 in all, so every KV group, every
    CTA of the tensor-core kernel (two tiles each) and, through the random
    offsets, rows handled by every softmax warp are compared."""
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg)
    q, k, v = dev(bi["q"]), dev(bi["k"]), dev(bi["v"])
    a, logz = gpu_states(q, k, v, bi["scale"], chunks=cfg["chunks"])
    a_h, lz_h = f64(a), f64(logz)
    g = np.random.default_rng(0)
    G = cfg["Hq"] // cfg["Hkv"]
    tiles = cfg["N"] // 128
    worst = 0.0
    for h in range(cfg["Hq"]):
        rows = np.arange(tiles) * 128 + g.integers(0, 128, tiles)
        oa, olz = O.build_states(bi["q"][h:h + 1, rows], bi["k"][h // G:h // G + 1],
                                 bi["v"][h // G:h // G + 1], bi["scale"])
        err = max(max_abs(a_h[h, rows], oa[0]), max_abs(lz_h[h, rows], olz[0]))
        worst = max(worst, err)
        assert err <= 2e-2, f"head {h}: {err}"
    assert worst > 0.0  # the comparison saw bf16 rounding, not identical buffers


# --------------------------------------------------------------- k-means ----

def gpu_seed(x, u):
    H, N, d = x.shape
    K = u.shape[1]
    ws = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(H, N, d, K), x.device, zero=False)
    idx = torch.empty(H, K, dtype=torch.int32, device=x.device)
    ops.asm_kmeanspp_seed(x, u, idx, ws)
    torch.cuda.synchronize()
    return host(idx).numpy()


def test_kmeanspp_tiny_fp32_config_exact():
    bi = inputs.build_inputs(inputs.CONFIGS[0])
    idx = gpu_seed(dev(bi["q"]), dev(bi["u"]))
    np.testing.assert_array_equal(idx, O.kmeanspp_seed(bi["q"], bi["u"]))
    assert all(len(set(r.tolist())) == r.size for r in idx)


def test_kmeanspp_llama_build_config_prefix():
    """K = 8192 rounds on all 32 heads; picks compared with the oracle (a pick
    depends only on earlier rounds): the first 2048 of head 0, which span the
    pruned rounds from the first regrouping (round 1024) through four
    regroupings, and the first 192 of head 31."""
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg)
    idx = gpu_seed(dev(bi["q"]), dev(bi["u"]))
    assert all(len(set(r.tolist())) == r.size for r in idx[[0, 31]])
    for h, n in ((0, 2048), (31, 192)):
        o = O.kmeanspp_seed(bi["q"][h:h + 1], bi["u"][h:h + 1, :n])
        np.testing.assert_array_equal(idx[h, :n], o[0])


@pytest.mark.parametrize("dt,d,N,K", [("bf16", 128, 8192, 1024), ("f32", 64, 5000, 600),
                                       ("bf16", 64, 3001, 520), ("f32", 128, 2500, 300),
                                       ("bf16", 128, 9001, 600)])
def test_kmeanspp_pruned_rounds_match_the_oracle(dt, d, N, K):
    """From round 256 the D2 update skips groups of points that the triangle
    inequality shows cannot move; the picks are those of the full update.
    Clustered data (so that most groups are skipped), ragged N, both storage
    types and head dims, several regroupings.  The bf16 d = 128 cases with
    N >= 8192 and K >= 512 also run the static anchor groups before round
    256 (K = 1024: 512 anchors from round 85; N = 9001, K = 600: 300 anchors,
    ragged, from round 85)."""
    x = inputs.mixture(inputs.BASE_SEED + 40 + d, "seed_q", 2, N, d, 48, 0.3, dt)
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 41 + N, 2, K)
    idx = gpu_seed(dev(x), dev(u))
    np.testing.assert_array_equal(idx, O.kmeanspp_seed(x, u))
    assert all(len(set(r.tolist())) == r.size for r in idx)


def test_kmeanspp_duplicate_points_exhaust_the_distinct_ones():
    """Fewer distinct points than centres: once every distinct point is
    chosen, sum(D2) = 0 and the smallest unchosen index is taken, past the
    regrouping rounds too."""
    base = inputs.mixture(inputs.BASE_SEED + 42, "seed_q", 1, 200, 64, 8, 0.3, "f32")
    x = base.repeat(1, 4, 1).contiguous()  # 800 points, 200 distinct
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 43, 1, 700)
    idx = gpu_seed(dev(x), dev(u))
    np.testing.assert_array_equal(idx, O.kmeanspp_seed(x, u))
    assert len(set(idx[0].tolist())) == 700


def kmeans_buffers(H, N, d, K, dtype):
    c = torch.empty(H, K, d, dtype=torch.float32, device="cuda")
    cdt = torch.empty(H, K, d, dtype=dtype, device="cuda")
    assign = torch.empty(H, N, dtype=torch.int32, device="cuda")
    counts = torch.empty(H, K, dtype=torch.int32, device="cuda")
    perm = torch.empty(H, N, dtype=torch.int32, device="cuda")
    seg = torch.empty(H, K + 1, dtype=torch.int32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda", zero=False)
    return c, cdt, assign, counts, perm, seg, ws


def teacher_forced(bi, iters, metric=ops.ASM_L2, heads=None):
    x = dev(bi["q"])
    H, N, d = x.shape
    K = bi["u"].shape[1]
    init = torch.from_numpy(O.kmeanspp_seed(bi["q"], bi["u"]))
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, K, x.dtype)
    # start from the seeds and walk the rounds one by one
    idx0 = init.long()
    c0 = bi["q"].to(torch.float32)[torch.arange(H)[:, None], idx0]
    c.copy_(c0)
    cdt.copy_(c0.to(x.dtype))
    xs = f64(bi["q"])
    heads = range(H) if heads is None else heads
    tol = TOL[x.dtype]
    inertia = {h: [] for h in heads}
    for t in range(iters):
        ops.asm_kmeans_assign(x, cdt, assign, ws, metric)
        torch.cuda.synchronize()
        g_assign = host(assign).numpy()
        g_cdt = f64(cdt)
        for h in heads:
            o_assign, o_gap = O.assign(xs[h], g_cdt[h], metric)
            check_indices(g_assign[h], o_assign, o_gap)
            inertia[h].append(((xs[h] - g_cdt[h][g_assign[h]]) ** 2).sum())
        c_before = f64(c)
        ops.asm_kmeans_update(x, assign, c, cdt, counts, perm, seg, ws)
        torch.cuda.synchronize()
        g_c, g_counts = f64(c), host(counts).numpy()
        g_perm, g_seg = host(perm).numpy(), host(seg).numpy()
        for h in heads:
            o_c, o_counts = O.update(xs[h], g_assign[h], c_before[h])
            np.testing.assert_array_equal(g_counts[h], o_counts)
            assert max_abs(g_c[h], o_c) <= 1e-4
            # members of each cluster, ascending
            np.testing.assert_array_equal(g_seg[h], np.concatenate([[0], np.cumsum(o_counts)]))
            np.testing.assert_array_equal(g_perm[h], np.argsort(g_assign[h], kind="stable"))
            np.testing.assert_array_equal(f64(cdt)[h], O.round_storage(g_c[h], 1 if x.dtype == torch.bfloat16 else 0))
    if metric == ops.ASM_L2:
        # storage rounding of the centres perturbs the objective by ~|c| 2^-9 (bf16)
        slack = 1e-6 if x.dtype == torch.float32 else 5e-4
        for h in heads:
            v = np.array(inertia[h])
            assert (np.diff(v) <= slack * v[0]).all(), "Lloyd objective went up"
    return x, c, cdt, assign, counts, perm, seg, ws


def test_kmeans_teacher_forced_tiny_fp32_config():
    bi = inputs.build_inputs(inputs.CONFIGS[0])
    teacher_forced(bi, iters=10)


def test_kmeans_teacher_forced_cosine():
    bi = inputs.build_inputs(dict(inputs.CONFIGS[0], dtype="bf16"), N=700, K=40)
    teacher_forced(bi, iters=3, metric=ops.ASM_COSINE)


def test_kmeans_teacher_forced_llama_shape_subset():
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg, N=16384, K=2048, H=4)
    teacher_forced(bi, iters=2, heads=[0, 3])


@pytest.mark.parametrize("metric", [ops.ASM_L2, ops.ASM_COSINE])
@pytest.mark.parametrize("N,K", [(1000, 300), (513, 5), (256, 128), (2304, 1153)])
def test_assign_tensor_core_ragged(metric, N, K):
    """bf16, d = 128 (the tcgen05 path): ragged point tail (N % 256), ragged
    centre tail (K % 128), a single partial centre tile, several tiles; the
    workspace error word stays 0."""
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg, N=N, K=K, H=3, L=64)
    x = dev(bi["q"])
    H, _, d = x.shape
    # centres: K distinct calibration points plus noise, in storage precision
    rng = np.random.default_rng(N * 7 + K)
    pick = np.stack([rng.choice(N, K, replace=False) for _ in range(H)])
    cen = bi["q"].to(torch.float64)[torch.arange(H)[:, None], torch.from_numpy(pick)]
    cen = cen + 0.05 * torch.from_numpy(rng.standard_normal(cen.shape))
    cdt = dev(cen.to(torch.bfloat16))
    assign = torch.full((H, N), -1, dtype=torch.int32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda", zero=True)
    ops.asm_kmeans_assign(x, cdt, assign, ws, metric)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    g = host(assign).numpy()
    xs, cs = f64(bi["q"]), f64(cdt)
    for h in range(H):
        o, gap = O.assign(xs[h], cs[h], metric)
        check_indices(g[h], o, gap)


def test_kmeans_every_point_a_centre_tensor_core():
    bi = inputs.build_inputs(inputs.CONFIGS[3], N=300, K=300, H=2, L=64)
    x = dev(bi["q"])
    H, N, d = x.shape
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, N, x.dtype)
    init = torch.arange(N, dtype=torch.int32).repeat(H, 1).contiguous()
    ops.asm_kmeans(x, dev(init), 2, c, cdt, assign, counts, perm, seg, ws)
    torch.cuda.synchronize()
    assert torch.equal(host(assign), init)
    assert (host(counts) == 1).all()


def test_kmeans_free_running_tiny_fp32_config():
    """Ten free iterations: final inertia within 1e-3 relative of the oracle's
    and the same number of non-empty clusters."""
    bi = inputs.build_inputs(inputs.CONFIGS[0])
    x = dev(bi["q"])
    H, N, d = x.shape
    K = bi["u"].shape[1]
    init = O.kmeanspp_seed(bi["q"], bi["u"])
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, K, x.dtype)
    ops.asm_kmeans(x, dev(torch.from_numpy(init)), 10, c, cdt, assign, counts, perm, seg, ws)
    torch.cuda.synchronize()
    oC, oCq, oa, ocounts, oin = O.kmeans(bi["q"], init, 10, O.L2, O.F32)
    xs = f64(bi["q"])
    ga, gc = host(assign).numpy(), f64(c)
    for h in range(H):
        g_in = ((xs[h] - gc[h][ga[h]]) ** 2).sum()
        o_in = ((xs[h] - oC[h][oa[h]]) ** 2).sum()
        assert abs(g_in - o_in) <= 1e-3 * o_in
        assert (host(counts).numpy()[h] > 0).sum() == (ocounts[h] > 0).sum()


def test_kmeans_every_point_a_centre():
    bi = inputs.build_inputs(dict(inputs.CONFIGS[0], dtype="bf16"), N=96, K=96)
    x = dev(bi["q"])
    H, N, d = x.shape
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, N, x.dtype)
    init = torch.arange(N, dtype=torch.int32).repeat(H, 1).contiguous()
    ops.asm_kmeans(x, dev(init), 2, c, cdt, assign, counts, perm, seg, ws)
    torch.cuda.synchronize()
    assert torch.equal(host(assign), init)
    assert (host(counts) == 1).all()


# ------------------------------------------------------------- aggregate ----

@pytest.mark.parametrize("zmode", [ops.ASM_ZBAR_MEAN, ops.ASM_ZBAR_SUM])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_aggregate_matches_oracle(zmode, dt):
    H, N, K, d = 3, 1000, 37, 128
    a = inputs.normal(1, "a", (H, N, d), dt)
    lz = inputs.uniform(1, "lz", (H, N), 2.0, 12.0)
    assign = torch.from_numpy(np.random.default_rng(1).integers(0, K - 1, (H, N)).astype(np.int32))
    lz[0, 5] = -float("inf")  # an empty member state
    # members sorted by cluster as the k-means update produces them
    perm = torch.from_numpy(np.argsort(assign.numpy(), axis=1, kind="stable").astype(np.int32))
    counts = np.stack([np.bincount(r, minlength=K) for r in assign.numpy()])
    seg = torch.from_numpy(np.concatenate([np.zeros((H, 1)), np.cumsum(counts, 1)], 1).astype(np.int32))
    a_bar = torch.empty(H, K, d, dtype=a.dtype, device="cuda")
    lz_bar = torch.empty(H, K, dtype=torch.float32, device="cuda")
    ops.asm_aggregate(dev(a), dev(lz), dev(perm), dev(seg), a_bar, lz_bar, zmode)
    torch.cuda.synchronize()
    tol = TOL[a.dtype]
    for h in range(H):
        oa, olz = O.aggregate(a[h], lz[h], assign[h], K, zmode)
        assert max_abs(f64(a_bar[h]), oa) <= tol
        assert max_abs(f64(lz_bar[h]), olz) <= tol
    assert f64(lz_bar)[:, K - 1].tolist() == [-np.inf] * H  # empty cluster


def test_aggregate_llama_build_config_two_heads():
    """Aggregation at the build shape (N = 65536 members per head into
    K = 8192 clusters of about 8) on two heads of different KV groups, with
    member states and logZ (about ln 16384 + O(1)) from the GPU's own
    prefix states over the full 16384-key prefix, and clusters from one
    GPU Lloyd round on k-means++-free random centres."""
    cfg = inputs.CONFIGS[3]
    heads = (0, 17)
    bi = inputs.build_inputs(cfg)
    G = cfg["Hq"] // cfg["Hkv"]
    x = dev(bi["q"][list(heads)])
    kv = [h // G for h in heads]
    H, N, d = x.shape
    K = cfg["K"]
    a = torch.empty_like(x)
    logz = torch.empty(H, N, dtype=torch.float32, device="cuda")
    for i, g in enumerate(kv):  # each head over its own KV head, 4 chunks
        ai, li = gpu_states(x[i:i + 1].contiguous(), dev(bi["k"][g:g + 1]), dev(bi["v"][g:g + 1]),
                            bi["scale"], chunks=cfg["chunks"])
        a[i], logz[i] = ai[0], li[0]
    g = np.random.default_rng(3)
    init = torch.from_numpy(np.stack([g.choice(N, K, replace=False) for _ in range(H)]).astype(np.int32))
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, K, x.dtype)
    ops.asm_kmeans(x, dev(init), 1, c, cdt, assign, counts, perm, seg, ws)
    a_bar = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
    lz_bar = torch.empty(H, K, dtype=torch.float32, device="cuda")
    ops.asm_aggregate(a, logz, perm, seg, a_bar, lz_bar)
    torch.cuda.synchronize()
    lz_h = f64(logz)
    assert 8.0 < np.median(lz_h) < 12.0  # logZ of a 16384-key prefix
    for i in range(H):
        oa, olz = O.aggregate(host(a)[i], host(logz)[i], host(assign)[i], K)
        assert max_abs(f64(a_bar[i]), oa) <= 2e-2
        assert max_abs(f64(lz_bar[i]), olz) <= 2e-2
    sizes = f64(counts)
    assert sizes.max() > 1 and (sizes == 0).sum() < K // 4  # real clusters of several members


def test_full_build_pipeline_tiny_fp32_config():
    """States -> k-means++ -> 10 Lloyd rounds -> aggregation, all on the GPU;
    the aggregation is checked against the oracle on the GPU's clusters."""
    cfg = inputs.CONFIGS[0]
    bi = inputs.build_inputs(cfg)
    x, k, v = dev(bi["q"]), dev(bi["k"]), dev(bi["v"])
    H, N, d = x.shape
    K = cfg["K"]
    a, logz = gpu_states(x, k, v, bi["scale"], chunks=2)
    init = torch.empty(H, K, dtype=torch.int32, device="cuda")
    ws_s = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(H, N, d, K), "cuda", zero=False)
    ops.asm_kmeanspp_seed(x, dev(bi["u"]), init, ws_s)
    c, cdt, assign, counts, perm, seg, ws = kmeans_buffers(H, N, d, K, x.dtype)
    ops.asm_kmeans(x, init, cfg["iters"], c, cdt, assign, counts, perm, seg, ws)
    a_bar = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
    lz_bar = torch.empty(H, K, dtype=torch.float32, device="cuda")
    ops.asm_aggregate(a, logz, perm, seg, a_bar, lz_bar)
    torch.cuda.synchronize()
    oa, olz = O.build_states(bi["q"], bi["k"], bi["v"], bi["scale"])
    for h in range(H):
        ab, lzb = O.aggregate(oa[h], olz[h], host(assign)[h], K)
        assert max_abs(f64(a_bar[h]), ab) <= 1e-4
        assert max_abs(f64(lz_bar[h]), lzb) <= 1e-4


# ------------------------------------------------- state merge (chunk split) --

@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_merge_states_matches_the_oracle_merge(dt, d):
    """asm_merge_states row by row against the oracle's merge, with empty
    states on either side and on both."""
    R = 3 * 333
    a1 = inputs.normal(21, "m_a1", (R, d), dt)
    a2 = inputs.normal(21, "m_a2", (R, d), dt)
    z1 = inputs.uniform(21, "m_z1", (R,), -5.0, 15.0)
    z2 = inputs.uniform(21, "m_z2", (R,), -5.0, 15.0)
    z1[::7] = -float("inf")
    z2[::11] = -float("inf")
    a, z = dev(a1).clone(), dev(z1).clone()
    ops.asm_merge_states(a.view(3, 333, d), z.view(3, 333), dev(a2).view(3, 333, d), dev(z2).view(3, 333))
    torch.cuda.synchronize()
    oa = np.zeros((R, d))
    oz = np.zeros(R)
    A1, A2 = f64(a1), f64(a2)
    for i in range(R):
        oa[i], oz[i] = O.merge(A1[i], float(z1[i]), A2[i], float(z2[i]))
    assert max_abs(f64(a), oa) <= TOL[a1.dtype]
    assert max_abs(f64(z), oz) <= TOL[a1.dtype]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_prefix_chunks_split_emulated_on_one_gpu(dt):
    """The split over ranks, on one GPU: each 'rank' encodes its run of the
    prefix chunks into its own buffers (asm_build_states), then the runs are
    folded in chunk order (asm_merge_states); the result is the single-pass
    oracle state."""
    from long_prefix_attention_b200 import sharding
    cfg = dict(inputs.CONFIGS[3], dtype=dt, Hq=8, Hkv=2, n_mix=8)
    bi = inputs.build_inputs(cfg, seed=77, N=300, L=1000, K=4)
    q = dev(bi["q"])
    bounds = [0, 128, 300, 301, 700, 1000]
    kc = [dev(bi["k"][:, b0:b1]) for b0, b1 in zip(bounds, bounds[1:])]
    vc = [dev(bi["v"][:, b0:b1]) for b0, b1 in zip(bounds, bounds[1:])]
    world = 3
    parts = []
    for r in range(world):
        c0, c1 = sharding.chunk_shard(len(kc), world, r)
        a = torch.empty_like(q)
        z = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
        for i in range(c0, c1):
            ops.asm_build_states(q, kc[i], vc[i], bi["scale"], a, z, accumulate=i > c0)
        parts.append((a, z))
    a, z = parts[0]
    for a_in, z_in in parts[1:]:
        ops.asm_merge_states(a, z, a_in, z_in)
    torch.cuda.synchronize()
    oa, oz = O.build_states(bi["q"], bi["k"], bi["v"], bi["scale"])
    tol = TOL[bi["q"].dtype]
    assert max_abs(f64(a), oa) <= tol
    assert max_abs(f64(z), oz) <= tol
