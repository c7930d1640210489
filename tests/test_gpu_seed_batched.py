"""Batched k-means++ seeding on the GPU (asm_kmeanspp_seed_batched) against
the oracle's batched seeding, draw for draw.

Up to `batch` centres are drawn per round from one D2 distribution before
D2 is updated, so the seeds differ from sequential k-means++ (except with
batch = 1, where they are the same); the oracle implements the same rule.
"""
import numpy as np
import pytest
import torch

from long_prefix_attention_b200 import inputs, ops
from oracle import asm_oracle as O

pytestmark = pytest.mark.gpu


def gpu_seed_batched(x, u, K, batch):
    H, N, d = x.shape
    ws = ops.alloc_workspace(ops.asm_kmeanspp_batched_workspace_size(H, N, d, K, batch), "cuda", zero=False)
    idx = torch.empty(H, K, dtype=torch.int32, device="cuda")
    ops.asm_kmeanspp_seed_batched(x.cuda(), u.cuda(), idx, batch, ws)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    return idx.cpu().numpy()


@pytest.mark.parametrize("dt,d,N,K", [("bf16", 128, 3001, 300), ("f32", 64, 2500, 256)])
def test_batch_of_one_is_kmeanspp(dt, d, N, K):
    """batch = 1 on the GPU gives the oracle's sequential k-means++ picks."""
    x = inputs.mixture(inputs.BASE_SEED + 60 + d, "bseed_q", 2, N, d, 48, 0.3, dt)
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 61, 2, K)
    np.testing.assert_array_equal(gpu_seed_batched(x, u, K, 1), O.kmeanspp_seed(x, u))


@pytest.mark.parametrize("dt,d,N,K,batch", [("bf16", 128, 8192, 1024, 128), ("bf16", 128, 5000, 700, 32),
                                             ("bf16", 128, 3001, 900, 200), ("bf16", 128, 2600, 800, 256),
                                             ("f32", 64, 4097, 500, 64), ("bf16", 64, 2048, 256, 256),
                                             ("f32", 128, 1500, 300, 7)])
def test_batched_seeding_matches_the_oracle(dt, d, N, K, batch):
    """Clustered points, ragged N and K, batches from 7 to 256 draws, both
    storage types and head dims: every pick equals the oracle's, and every
    head gets K distinct points.  bf16 with d = 128 runs the fused rounds
    (one or two centre tiles, the second ragged at 200 draws)."""
    x = inputs.mixture(inputs.BASE_SEED + 62 + N, "bseed_q", 2, N, d, 64, 0.3, dt)
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 63 + K, 2, 2 * K)
    got = gpu_seed_batched(x, u, K, batch)
    np.testing.assert_array_equal(got, O.kmeanspp_seed_batched(x, u, K, batch))
    assert all(len(set(r.tolist())) == K for r in got)


@pytest.mark.parametrize("batch", [128, 200])
def test_batched_many_tiles_per_cta(batch):
    """32 heads of 4096 points: each CTA of a fused round takes several
    128-point tiles in turn (four accumulators at 128 draws, two at 200)."""
    x = inputs.mixture(inputs.BASE_SEED + 69, "bseed_q", 32, 4096, 128, 64, 0.3, "bf16")
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 70, 32, 1200)
    got = gpu_seed_batched(x, u, 600, batch)
    np.testing.assert_array_equal(got, O.kmeanspp_seed_batched(x, u, 600, batch))


@pytest.mark.parametrize("dt,d", [("f32", 64), ("bf16", 128)])
def test_batched_repeats_and_exhausted_points(dt, d):
    """Fewer distinct points than centres (sum(D2) reaches 0, then the
    smallest unchosen indices), and draws that repeat within a round."""
    base = inputs.mixture(inputs.BASE_SEED + 64, "bseed_q", 1, 100, d, 4, 0.3, dt)
    x = base.repeat(1, 5, 1).contiguous()  # 500 points, 100 distinct
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 65, 1, 600)
    u[:, 1:9] = 0.37                        # round 1: eight equal draws, one kept
    got = gpu_seed_batched(x, u, 450, 16)
    np.testing.assert_array_equal(got, O.kmeanspp_seed_batched(x, u, 450, 16))
    assert len(set(got[0].tolist())) == 450


def test_batched_k_equals_n_and_k_one():
    x = inputs.mixture(inputs.BASE_SEED + 66, "bseed_q", 1, 300, 128, 8, 0.3, "bf16")
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 67, 1, 400)
    got = gpu_seed_batched(x, u, 300, 64)
    np.testing.assert_array_equal(got, O.kmeanspp_seed_batched(x, u, 300, 64))
    assert sorted(got[0].tolist()) == list(range(300))
    one = gpu_seed_batched(x, u, 1, 64)
    assert one[0, 0] == int(float(u[0, 0]) * 300)


def test_batched_build_shape_prefix():
    """The build shape (32 heads, N = 65536, d = 128, bf16, K = 8192) with 128
    draws per round.  The oracle's run with K = 1025 makes the same first
    eight rounds (each draws 128 while at least 128 centres are missing), so
    the picks agree up to the count after round 8: 1025 less the repeats,
    of which a few are expected; the first 1000 are compared."""
    cfg = inputs.CONFIGS[3]
    bi = inputs.build_inputs(cfg)
    H, N, d = bi["q"].shape
    K, batch = cfg["K"], 128
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 68, H, 2 * K)
    got = gpu_seed_batched(bi["q"], u, K, batch)
    assert all(len(set(r.tolist())) == K for r in got[[0, H - 1]])
    ref = O.kmeanspp_seed_batched(bi["q"][:1], u[:1], 1025, batch)
    np.testing.assert_array_equal(got[0, :1000], ref[0, :1000])


def test_batched_seeds_feed_lloyd_like_kmeanspp():
    """The free-running k-means rule applied to batched seeds (bf16, d = 128,
    the fused rounds): ten Lloyd iterations from the GPU's batched seeds end
    within 1e-3 relative inertia of the oracle's k-means from the same seeds,
    with the same number of non-empty clusters.  The seeds' own potential
    (sum of D2 to the nearest seed, by the oracle's assignment) is within 10%
    of sequential k-means++'s on the same points."""
    H, N, d, K, batch = 2, 4096, 128, 256, 32
    x = inputs.mixture(inputs.BASE_SEED + 71, "bseed_q", H, N, d, 64, 0.3, "bf16")
    u = inputs.kmeanspp_uniforms(inputs.BASE_SEED + 72, H, 2 * K)
    seeds = gpu_seed_batched(x, u, K, batch)
    np.testing.assert_array_equal(seeds, O.kmeanspp_seed_batched(x, u, K, batch))

    xd = x.cuda()
    c = torch.empty(H, K, d, dtype=torch.float32, device="cuda")
    cdt = torch.empty(H, K, d, dtype=x.dtype, device="cuda")
    assign = torch.empty(H, N, dtype=torch.int32, device="cuda")
    counts = torch.empty(H, K, dtype=torch.int32, device="cuda")
    perm = torch.empty(H, N, dtype=torch.int32, device="cuda")
    seg = torch.empty(H, K + 1, dtype=torch.int32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, N, d, K), "cuda", zero=False)
    ops.asm_kmeans(xd, torch.from_numpy(seeds).cuda(), 10, c, cdt, assign, counts, perm, seg, ws)
    torch.cuda.synchronize()
    oC, _, oa, ocounts, _ = O.kmeans(x, seeds, 10, O.L2, O.BF16)
    xs = x.to(torch.float64).numpy()
    ga, gc = assign.cpu().numpy(), c.cpu().to(torch.float64).numpy()
    for h in range(H):
        g_in = ((xs[h] - gc[h][ga[h]]) ** 2).sum()
        o_in = ((xs[h] - oC[h][oa[h]]) ** 2).sum()
        assert abs(g_in - o_in) <= 1e-3 * o_in
        assert (counts.cpu().numpy()[h] > 0).sum() == (ocounts[h] > 0).sum()

    seq = O.kmeanspp_seed(x, u[:, :K].contiguous())
    for h in range(H):
        pot = []
        for idx in (seeds[h], seq[h]):
            a, _ = O.assign(xs[h], xs[h][idx])
            pot.append(((xs[h] - xs[h][idx][a]) ** 2).sum())
        assert pot[0] <= 1.1 * pot[1], pot
