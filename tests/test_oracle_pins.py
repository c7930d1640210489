"""Pins of the fp64 oracle against facts fixed outside it.

Each test ties one oracle function to something the oracle does not compute
itself: a library routine (torch's fp64 scaled-dot-product attention, scipy's
logsumexp and cdist, sklearn's Lloyd k-means, torch's bf16 rounding), a
closed form, an invariant the pages assert (lossless composition of attention
states across key blocks, "Metodologia" of "Context Memorization for
Efficient Long Context Generation"), or brute force on tiny inputs.  They run
on the CPU (no ``gpu`` mark).
"""
import math

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist
from scipy.special import logsumexp

from oracle import asm_oracle as O

TOL = 1e-12


def sdpa_f64(q, K, V, scale):
    """torch's scaled-dot-product attention in fp64: q[d], K,V[L,d] -> [d]."""
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64)).view(1, 1, 1, -1)
    Kt = torch.from_numpy(np.asarray(K, dtype=np.float64)).view(1, 1, len(K), -1)
    Vt = torch.from_numpy(np.asarray(V, dtype=np.float64)).view(1, 1, len(V), -1)
    out = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return out.view(-1).numpy()


# ----------------------------------------------------------------- state ----

def test_state_two_keys_closed_form():
    # q = e1, keys e1 and e2, scale s: logits (s, 0), so Z = e^s + 1 and
    # a = (e^s v0 + v1) / (e^s + 1).
    s = 0.75
    q = np.array([1.0, 0.0])
    K = np.eye(2)
    V = np.array([[1.0, 2.0], [3.0, 4.0]])
    a, z = O.state(q, K, V, s)
    es = math.exp(s)
    assert z == pytest.approx(math.log(es + 1.0), abs=TOL)
    np.testing.assert_allclose(a, (es * V[0] + V[1]) / (es + 1.0), atol=TOL)


@pytest.mark.parametrize("L", [1, 2, 7, 64])
def test_state_matches_library_attention(L):
    g = np.random.default_rng(L)
    d = 16
    q, K, V = g.standard_normal(d), g.standard_normal((L, d)), g.standard_normal((L, d))
    s = 1.0 / math.sqrt(d)
    a, z = O.state(q, K, V, s)
    np.testing.assert_allclose(a, sdpa_f64(q, K, V, s), atol=TOL, rtol=0)
    assert z == pytest.approx(logsumexp(s * (K @ q)), abs=TOL)


def test_state_special_cases():
    g = np.random.default_rng(1)
    d = 8
    K, V = g.standard_normal((5, d)), g.standard_normal((5, d))
    # one key: a is that value row exactly, logZ its logit
    a, z = O.state(g.standard_normal(d) * 0 + 1.0, K[:1], V[:1], 0.5)
    np.testing.assert_array_equal(a, V[0])
    assert z == pytest.approx(0.5 * K[0].sum(), abs=TOL)
    # zero query: uniform weights, a = mean of V, Z = L
    a, z = O.state(np.zeros(d), K, V, 0.3)
    np.testing.assert_allclose(a, V.mean(axis=0), atol=TOL)
    assert z == pytest.approx(math.log(5.0), abs=TOL)
    # empty block
    a, z = O.state(np.ones(d), K[:0], V[:0], 0.3)
    assert z == -math.inf and not a.any()
    # large logits: max subtraction keeps it finite
    a, z = O.state(np.full(d, 40.0), K, V, 1.0)
    assert np.isfinite(z) and np.isfinite(a).all()
    np.testing.assert_allclose(a, sdpa_f64(np.full(d, 40.0), K, V, 1.0), atol=1e-10)


# ----------------------------------------------------------------- merge ----

@pytest.mark.parametrize("seed", range(6))
def test_merge_equals_attention_over_concatenation(seed):
    g = np.random.default_rng(100 + seed)
    d = 12
    L = int(g.integers(0, 40))
    cut = int(g.integers(0, L + 1))  # includes empty left or right blocks
    q, K, V = g.standard_normal(d), g.standard_normal((L, d)), g.standard_normal((L, d))
    s = 0.4
    a1, z1 = O.state(q, K[:cut], V[:cut], s)
    a2, z2 = O.state(q, K[cut:], V[cut:], s)
    a, z = O.merge(a1, z1, a2, z2)
    if L == 0:
        assert z == -math.inf and not a.any()
        return
    np.testing.assert_allclose(a, sdpa_f64(q, K, V, s), atol=TOL)
    assert z == pytest.approx(logsumexp(s * (K @ q)), abs=TOL)


def test_merge_algebra():
    g = np.random.default_rng(7)
    d = 6
    st = [(g.standard_normal(d), float(g.uniform(-3, 3))) for _ in range(3)]
    ab, zb = O.merge(*st[0], *st[1])
    ba, zba = O.merge(*st[1], *st[0])
    np.testing.assert_allclose(ab, ba, atol=TOL)
    assert zb == pytest.approx(zba, abs=TOL)
    l, zl = O.merge(*O.merge(*st[0], *st[1]), *st[2])
    r, zr = O.merge(*st[0], *O.merge(*st[1], *st[2]))
    np.testing.assert_allclose(l, r, atol=TOL)
    assert zl == pytest.approx(zr, abs=TOL)
    # Z adds: exp(z) = exp(z1) + exp(z2)
    assert math.exp(zb) == pytest.approx(math.exp(st[0][1]) + math.exp(st[1][1]), rel=1e-13)
    # the empty state is the identity
    e, ze = O.merge(*st[0], np.zeros(d), -math.inf)
    np.testing.assert_array_equal(e, st[0][0])
    assert ze == st[0][1]


# ------------------------------------------------------------ build states ---

def test_build_states_gqa_and_chunks():
    g = np.random.default_rng(3)
    Hq, Hkv, N, L, d = 4, 2, 5, 37, 16
    s = 1.0 / math.sqrt(d)
    Q = g.standard_normal((Hq, N, d))
    K, V = g.standard_normal((Hkv, L, d)), g.standard_normal((Hkv, L, d))
    A, lz = O.build_states(Q, K, V, s)
    # head h reads KV head h // (Hq // Hkv): torch SDPA with repeat_interleave
    Kr = torch.from_numpy(K).repeat_interleave(Hq // Hkv, dim=0)
    Vr = torch.from_numpy(V).repeat_interleave(Hq // Hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), Kr, Vr, scale=s).numpy()
    np.testing.assert_allclose(A, ref, atol=TOL)
    ref_lz = logsumexp(s * np.einsum("hnd,hld->hnl", Q, Kr.numpy()), axis=-1)
    np.testing.assert_allclose(lz, ref_lz, atol=TOL)
    # chunked encoding merged in memory equals the single pass (uneven chunks)
    A2, lz2 = None, None
    for lo, hi in [(0, 10), (10, 11), (11, 30), (30, 37)]:
        A2, lz2 = O.build_states(Q, K[:, lo:hi], V[:, lo:hi], s, A2, lz2, accumulate=A2 is not None)
    np.testing.assert_allclose(A2, A, atol=TOL)
    np.testing.assert_allclose(lz2, lz, atol=TOL)
    # accumulating into the empty state is the single pass
    A3, lz3 = O.build_states(Q, K, V, s, np.zeros_like(A), np.full_like(lz, -np.inf), accumulate=True)
    np.testing.assert_allclose(A3, A, atol=TOL)
    np.testing.assert_allclose(lz3, lz, atol=TOL)


# -------------------------------------------------------------- k-means++ ---

def test_kmeanspp_first_pick_and_full_permutation():
    g = np.random.default_rng(11)
    N, d = 23, 5
    X = g.standard_normal((1, N, d))
    u = g.random((1, N))
    idx = O.kmeanspp_seed(X, u)[0]
    assert idx[0] == int(u[0, 0] * N)
    # with K = N, D2 of every chosen point is 0, so every point is chosen once
    assert sorted(idx.tolist()) == list(range(N))


def test_kmeanspp_second_pick_is_d2_inverse_cdf():
    """For u on a fine grid, the second pick hits point i in proportion to D2_i."""
    g = np.random.default_rng(12)
    N, d, M = 9, 3, 20000
    X = g.standard_normal((N, d))
    first = 4
    D2 = cdist(X, X[first:first + 1], "sqeuclidean")[:, 0]
    p = D2 / D2.sum()
    u1 = (np.arange(M) + 0.5) / M
    Xs = np.broadcast_to(X, (M, N, d))
    u = np.stack([np.full(M, (first + 0.5) / N), u1], axis=1)
    picks = O.kmeanspp_seed(Xs, u)[:, 1]
    counts = np.bincount(picks, minlength=N)
    np.testing.assert_allclose(counts / M, p, atol=2.0 / M)
    assert counts[first] == 0
    # inverse CDF is monotone in u
    assert np.all(np.diff(picks) >= 0)


def test_kmeanspp_all_duplicate_points():
    X = np.ones((1, 6, 4))
    u = np.array([[0.5, 0.1, 0.9, 0.3]])
    idx = O.kmeanspp_seed(X, u)[0]
    # round 0 takes floor(0.5 * 6) = 3; then sum(D2) = 0 -> smallest unchosen
    assert idx.tolist() == [3, 0, 1, 2]


# ------------------------------------------------- batched k-means++ ------

@pytest.mark.parametrize("dup", [False, True])
def test_kmeanspp_batched_one_draw_per_round_is_kmeanspp(dup):
    """b = 1: one draw per round, D2 updated after each, is k-means++ itself
    (clustered points, and points repeated so that sum(D2) reaches 0)."""
    g = np.random.default_rng(31 + dup)
    base = g.standard_normal((2, 40, 6))
    X = np.concatenate([base, base], axis=1) if dup else g.standard_normal((2, 80, 6))
    K = 60
    u = g.random((2, K))
    np.testing.assert_array_equal(O.kmeanspp_seed_batched(X, u, K, 1), O.kmeanspp_seed(X, u))


def test_kmeanspp_batched_hand_case_with_a_repeated_draw():
    """Four points on a line at 0, 1, 10, 11, K = 3, two draws per round.
    Round 0: u = 0 takes point 0; D2 = 0, 1, 100, 121 (sum 222).  Round 1:
    both draws are 0.5 -> thresholds 111: the running sums 0, 1, 101, 222
    first exceed it at point 3, twice, so the second draw is dropped.  D2
    becomes 0, 1, 1, 0 (sum 2).  Round 2 (one centre left): u = 0.75 ->
    threshold 1.5, first exceeded at point 2 (running sum 2)."""
    X = np.array([[[0.0], [1.0], [10.0], [11.0]]])
    u = np.array([[0.0, 0.5, 0.5, 0.75]])
    assert O.kmeanspp_seed_batched(X, u, 3, 2)[0].tolist() == [0, 3, 2]


def test_kmeanspp_batched_all_duplicates_take_the_smallest_unchosen():
    """Six equal points: round 0 takes floor(0.6 * 6) = 3, then sum(D2) = 0 and
    the three draws of round 1 take the 1st, 2nd and 3rd smallest unchosen
    indices."""
    X = np.ones((1, 6, 4))
    u = np.array([[0.6, 0.9, 0.1, 0.5]])
    assert O.kmeanspp_seed_batched(X, u, 4, 3)[0].tolist() == [3, 0, 1, 2]


def test_kmeanspp_batched_k_equals_n_is_a_permutation():
    g = np.random.default_rng(33)
    N = 50
    X = g.standard_normal((1, N, 3))
    u = g.random((1, 2 * N))
    idx = O.kmeanspp_seed_batched(X, u, N, 8)[0]
    assert idx[0] == int(u[0, 0] * N)
    assert sorted(idx.tolist()) == list(range(N))


def test_kmeanspp_batched_first_round_draws_follow_d2():
    """All draws of round 1 come from the same D2 distribution (the round-0
    centre's): over a fine grid of u, the picks of each draw position hit
    point i in proportion to D2_i (repeats within a round dropped only when
    two draws hit the same point, which a grid of distinct u spreads out)."""
    g = np.random.default_rng(34)
    N, d, M, b = 9, 3, 4000, 4
    X = g.standard_normal((N, d))
    first = 4
    D2 = cdist(X, X[first:first + 1], "sqeuclidean")[:, 0]
    p = D2 / D2.sum()
    grid = (np.arange(M) + 0.5) / M
    # case m: K = b + 1, so round 1 makes b draws, all equal to grid[m]: they
    # hit the same point and the round keeps one, the inverse CDF of grid[m]
    u = np.concatenate([np.full((M, 1), (first + 0.5) / N), np.repeat(grid[:, None], b, axis=1)], axis=1)
    picks = O.kmeanspp_seed_batched(np.broadcast_to(X, (M, N, d)), u, b + 1, b)[:, 1]
    counts = np.bincount(picks, minlength=N)
    np.testing.assert_allclose(counts / M, p, atol=2.0 / M)


# ---------------------------------------------------------------- assign ----

@pytest.mark.parametrize("metric", [O.L2, O.COSINE])
def test_assign_matches_cdist(metric):
    g = np.random.default_rng(20 + metric)
    X, C = g.standard_normal((300, 8)), g.standard_normal((17, 8))
    a, gap = O.assign(X, C, metric)
    D = cdist(X, C, "sqeuclidean" if metric == O.L2 else "cosine")
    np.testing.assert_array_equal(a, D.argmin(axis=1))
    Ds = np.sort(D, axis=1)
    if metric == O.L2:
        np.testing.assert_allclose(gap, (Ds[:, 1] - Ds[:, 0]) / Ds[:, 0], rtol=1e-9)
    else:
        assert (gap >= 0).all()


def test_assign_ties_and_single_centre():
    C = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 0.0]])
    X = np.array([[2.0, 0.0], [0.5, 0.5]])
    a, gap = O.assign(X, C, O.L2)
    assert a.tolist() == [0, 0]  # duplicate centre 2 and the equidistant point
    assert gap[0] == 0.0 and gap[1] == 0.0
    a, gap = O.assign(X, C[:1], O.L2)
    assert a.tolist() == [0, 0] and np.isinf(gap).all()


# --------------------------------------------------------- update / Lloyd ---

def test_update_is_member_mean_and_keeps_empty():
    g = np.random.default_rng(30)
    X = g.standard_normal((40, 6))
    a = g.integers(0, 4, 40).astype(np.int32)
    a[a == 2] = 3  # cluster 2 empty
    Cin = g.standard_normal((5, 6))
    Cout, counts = O.update(X, a, Cin)
    for c in range(5):
        m = a == c
        assert counts[c] == m.sum()
        np.testing.assert_allclose(Cout[c], X[m].mean(axis=0) if m.any() else Cin[c], atol=TOL)


def test_lloyd_matches_sklearn():
    from sklearn.cluster import KMeans
    g = np.random.default_rng(31)
    means = 6.0 * g.standard_normal((6, 4))
    X = (means[g.integers(0, 6, 600)] + 0.7 * g.standard_normal((600, 4))).astype(np.float32)
    X = X.astype(np.float64)  # exact fp32 values
    init = np.array([[0, 100, 200, 300, 400, 500]], dtype=np.int32)
    for iters in (1, 3, 10):
        C, Cq, a, counts, inertia = O.kmeans(X[None], init, iters, O.L2, O.F32)
        km = KMeans(n_clusters=6, init=X[init[0]], n_init=1, max_iter=iters, tol=0.0,
                    algorithm="lloyd").fit(X)
        np.testing.assert_allclose(C[0], km.cluster_centers_, atol=1e-9)
        assert (np.diff(inertia[0]) <= 1e-9 * inertia[0, 0]).all()  # Lloyd never goes up
        np.testing.assert_allclose(Cq[0], C[0].astype(np.float32), atol=0)
        assert counts[0].sum() == 600


def test_lloyd_identity_when_every_point_is_a_centre():
    g = np.random.default_rng(32)
    X = g.standard_normal((1, 15, 3))
    init = np.arange(15, dtype=np.int32)[None]
    C, Cq, a, counts, _ = O.kmeans(X, init, 3, O.L2, O.F32)
    assert a[0].tolist() == list(range(15))
    assert (counts == 1).all()
    np.testing.assert_array_equal(C[0], X[0])


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(33)
    x = np.concatenate([g.standard_normal(5000) * 10.0, [0.0, -0.0, 1e-30, 3.0e38]])
    y = O.round_storage(x, O.BF16)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(y, ref)
    np.testing.assert_array_equal(O.round_storage(x, O.F32), x.astype(np.float32).astype(np.float64))


# ------------------------------------------------------------- aggregate ----

def test_aggregate_singleton_equal_and_modes():
    g = np.random.default_rng(40)
    N, d, K = 9, 5, 4
    A = g.standard_normal((N, d))
    lz = g.uniform(-2, 6, N)
    a = np.array([0, 1, 1, 1, 2, 2, 0, 0, 1], dtype=np.int32)  # cluster 3 empty
    Ab_m, lz_m = O.aggregate(A, lz, a, K, O.ZBAR_MEAN)
    Ab_s, lz_s = O.aggregate(A, lz, a, K, O.ZBAR_SUM)
    np.testing.assert_allclose(Ab_m, Ab_s, atol=0)
    for c in range(3):
        n = (a == c).sum()
        assert lz_s[c] - lz_m[c] == pytest.approx(math.log(n), abs=TOL)
        assert lz_s[c] == pytest.approx(logsumexp(lz[a == c]), abs=TOL)
    assert lz_m[3] == -math.inf and not Ab_m[3].any()
    # a singleton cluster returns exactly its member's state
    Ab1, lz1 = O.aggregate(A[:1], lz[:1], np.zeros(1, np.int32), 1, O.ZBAR_MEAN)
    np.testing.assert_array_equal(Ab1[0], A[0])
    assert lz1[0] == lz[0]
    # members with identical states: the mean mode returns that state
    Ab2, lz2 = O.aggregate(np.repeat(A[:1], 4, 0), np.repeat(lz[:1], 4), np.zeros(4, np.int32), 1)
    np.testing.assert_allclose(Ab2[0], A[0], atol=TOL)
    assert lz2[0] == pytest.approx(lz[0], abs=TOL)


def test_aggregate_is_brute_force_pooled_attention():
    """Sum mode: Z_bar = sum_i sum_j e^{s q_i.k_j}, Z_bar a_bar = sum_i sum_j e^{..} v_j."""
    g = np.random.default_rng(41)
    M, L, d = 6, 11, 4
    s = 0.5
    Q, K, V = g.standard_normal((M, d)), g.standard_normal((L, d)), g.standard_normal((L, d))
    A, lz = O.build_states(Q[None], K[None], V[None], s)
    Ab, lzb = O.aggregate(A[0], lz[0], np.zeros(M, np.int32), 1, O.ZBAR_SUM)
    W = np.exp(s * Q @ K.T)  # [M, L]
    Z = W.sum()
    assert lzb[0] == pytest.approx(math.log(Z), abs=1e-12)
    np.testing.assert_allclose(Ab[0], (W.sum(axis=0) @ V) / Z, atol=1e-12)


# ---------------------------------------------------------------- decode ----

def _tiny_decode_case(g, B=2, Hq=4, Hkv=2, K=6, T=5, d=8, Lp=9):
    return dict(
        q=g.standard_normal((B, Hq, d)), C=g.standard_normal((Hq, K, d)),
        Kp=g.standard_normal((Hkv, Lp, d)), Vp=g.standard_normal((Hkv, Lp, d)),
        Kc=g.standard_normal((B, Hkv, T, d)), Vc=g.standard_normal((B, Hkv, T, d)),
    )


def test_full_attention_matches_library():
    g = np.random.default_rng(50)
    t = _tiny_decode_case(g)
    ll = np.array([5, 2], np.int32)
    s = 0.35
    out, lse = O.full_attention(t["q"], t["Kp"], t["Vp"], t["Kc"], t["Vc"], ll, s)
    for b in range(2):
        for h in range(4):
            gg = h // 2
            Kcat = np.concatenate([t["Kp"][gg], t["Kc"][b, gg, :ll[b]]])
            Vcat = np.concatenate([t["Vp"][gg], t["Vc"][b, gg, :ll[b]]])
            np.testing.assert_allclose(out[b, h], sdpa_f64(t["q"][b, h], Kcat, Vcat, s), atol=TOL)
            assert lse[b, h] == pytest.approx(logsumexp(s * Kcat @ t["q"][b, h]), abs=TOL)


def test_decode_identity_memory_recovers_full_attention():
    """K = N, centres = calibration queries, states = their exact prefix states:
    a decode query equal to calibration query i selects i, and the merged
    output is attention over prefix + local ("Fusion" bullet)."""
    g = np.random.default_rng(51)
    B, Hq, Hkv, N, T, d, Lp = 3, 4, 2, 10, 6, 8, 13
    s = 1 / math.sqrt(d)
    calib = g.standard_normal((Hq, N, d))
    Kp, Vp = g.standard_normal((Hkv, Lp, d)), g.standard_normal((Hkv, Lp, d))
    Abar, lzbar = O.build_states(calib, Kp, Vp, s)
    pick = g.integers(0, N, (B, Hq))
    q = np.stack([[calib[h, pick[b, h]] for h in range(Hq)] for b in range(B)])
    Kc, Vc = g.standard_normal((B, Hkv, T, d)), g.standard_normal((B, Hkv, T, d))
    ll = np.array([6, 0, 3], np.int32)
    out, lse, idx, gap = O.decode(q, calib, Abar, lzbar, Kc, Vc, ll, s)
    np.testing.assert_array_equal(idx, pick)
    ref, ref_lse = O.full_attention(q, Kp, Vp, Kc, Vc, ll, s)
    for b in range(B):
        for h in range(Hq):
            gg = h // 2
            Kcat = np.concatenate([Kp[gg], Kc[b, gg, :ll[b]]])
            Vcat = np.concatenate([Vp[gg], Vc[b, gg, :ll[b]]])
            np.testing.assert_allclose(out[b, h], sdpa_f64(q[b, h], Kcat, Vcat, s), atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)
    # local length 0 returns the retrieved state itself
    np.testing.assert_allclose(out[1], Abar[np.arange(Hq), pick[1]], atol=TOL)


def test_decode_search_and_local_only_cases():
    g = np.random.default_rng(52)
    B, Hq, Hkv, K, T, d = 2, 4, 1, 7, 5, 8
    s = 0.3
    q = g.standard_normal((B, Hq, d))
    C = g.standard_normal((Hq, K, d))
    Kc, Vc = g.standard_normal((B, Hkv, T, d)), g.standard_normal((B, Hkv, T, d))
    ll = np.array([5, 4], np.int32)
    # empty memory states: the output is plain attention over the local tokens
    out, lse, idx, _ = O.decode(q, C, np.zeros((Hq, K, d)), np.full((Hq, K), -np.inf), Kc, Vc, ll, s)
    for b in range(B):
        for h in range(Hq):
            np.testing.assert_allclose(out[b, h], sdpa_f64(q[b, h], Kc[b, 0, :ll[b]], Vc[b, 0, :ll[b]], s),
                                       atol=TOL)
            assert idx[b, h] == cdist(q[b, h][None], C[h], "sqeuclidean").argmin()
    # cosine retrieval follows cdist's cosine distance
    _, _, idx_c, _ = O.decode(q, C, np.zeros((Hq, K, d)), np.zeros((Hq, K)), Kc, Vc, ll, s, O.COSINE)
    for b in range(B):
        for h in range(Hq):
            assert idx_c[b, h] == cdist(q[b, h][None], C[h], "cosine").argmin()
    # a given index overrides the search
    forced = np.zeros((B, Hq), np.int32) + 3
    _, _, idx_f, _ = O.decode(q, C, np.zeros((Hq, K, d)), np.zeros((Hq, K)), Kc, Vc, ll, s, idx_in=forced)
    assert (idx_f == 3).all()


# ------------------------------------------------- two-level (hierarchical) search

def test_index_search_hand_case():
    """Centres on a line: clusters {0, 4} (super-centre 2) and {6, 100}
    (super-centre 53).  The query 5.2 is nearest to the super-centre 2, so
    with one cluster kept the search returns 4 (row 1) although 6 (row 2) is
    the nearest centre; keeping both clusters returns 6.  Distances by hand:
    super 10.24 vs 2284.84; members 27.04, 1.44 | 0.64, 9063.04."""
    C = np.array([[[0, 0], [4, 0], [6, 0], [100, 0]]], float)
    S = np.array([[[2, 0], [53, 0]]], float)
    so = np.array([[0, 2, 4]], np.int32)
    q = np.array([[[5.2, 0]]], float)
    idx, sel, gs, gi = O.index_search(q, S, so, C, 1)
    assert idx[0, 0] == 1 and sel[0, 0, 0] == 0
    assert gs[0, 0] == pytest.approx((2284.84 - 10.24) / 10.24)
    assert gi[0, 0] == pytest.approx((27.04 - 1.44) / 1.44)
    idx, sel, gs, gi = O.index_search(q, S, so, C, 2)
    assert idx[0, 0] == 2 and list(sel[0, 0]) == [0, 1]
    assert np.isinf(gs[0, 0])
    assert gi[0, 0] == pytest.approx((1.44 - 0.64) / 0.64)


def _clustered(rng, H, K, K1, d):
    """Centres ordered by an arbitrary partition into K1 non-empty clusters."""
    sizes = rng.multinomial(K - K1, np.ones(K1) / K1) + 1
    so = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    C = rng.standard_normal((H, K, d))
    S = rng.standard_normal((H, K1, d))
    return C, S, np.tile(so, (H, 1))


@pytest.mark.parametrize("metric", [O.L2, O.COSINE])
def test_index_search_keeping_every_cluster_is_the_flat_search(metric):
    rng = np.random.default_rng(3)
    H, K, K1, d, B = 3, 97, 9, 16, 5
    C, S, so = _clustered(rng, H, K, K1, d)
    q = rng.standard_normal((B, H, d))
    idx, sel, gs, gi = O.index_search(q, S, so, C, K1, metric)
    for h in range(H):
        flat, gap = O.assign(q[:, h], C[h], metric)
        np.testing.assert_array_equal(idx[:, h], flat)
        np.testing.assert_allclose(gi[:, h], gap)
        assert all(sorted(s) == list(range(K1)) for s in sel[:, h])


def test_index_search_singleton_clusters_is_the_flat_search():
    """K1 = K, every centre its own cluster and super-centre, one cluster
    kept: the first level alone is the flat search."""
    rng = np.random.default_rng(4)
    H, K, d, B = 2, 40, 8, 7
    C = rng.standard_normal((H, K, d))
    so = np.tile(np.arange(K + 1, dtype=np.int32), (H, 1))
    q = rng.standard_normal((B, H, d))
    idx, sel, gs, gi = O.index_search(q, C, so, C, 1)
    for h in range(H):
        flat, gap = O.assign(q[:, h], C[h])
        np.testing.assert_array_equal(idx[:, h], flat)
        np.testing.assert_array_equal(sel[:, h, 0], flat)
        np.testing.assert_allclose(gs[:, h], gap)


# ----------------------------------------------------------- whitening ---

def test_whitening_diagonal_closed_form():
    """Rows +-s_i e_i: mean 0 and covariance exactly diag(2 s_i^2 / N), so W
    is diag((2 s_i^2 / N + eps)^-1/2) with eps = eps_rel * trace / d."""
    d = 6
    s = np.array([0.5, 1.0, 2.0, 3.0, 0.25, 1.5])
    rows = np.concatenate([np.diag(s), -np.diag(s)])[None]  # N = 2d
    N = 2 * d
    mu, W = O.whitening(rows, eps_rel=1e-3)
    var = 2 * s ** 2 / N
    eps = 1e-3 * var.sum() / d
    np.testing.assert_allclose(mu[0], 0.0, atol=1e-15)
    np.testing.assert_allclose(W[0], np.diag((var + eps) ** -0.5), rtol=1e-12, atol=1e-12)


def test_whitening_inverts_the_regularised_covariance():
    """W is symmetric and W (C + eps I) W = I, C from numpy's own covariance."""
    g = np.random.default_rng(3)
    A = g.standard_normal((16, 16))
    X = (g.standard_normal((2, 500, 16)) @ A) + 3.0
    mu, W = O.whitening(X, eps_rel=1e-4)
    for h in range(2):
        C = np.cov(X[h], rowvar=False, bias=True)
        eps = 1e-4 * np.trace(C) / 16
        np.testing.assert_allclose(W[h], W[h].T, atol=1e-12)
        np.testing.assert_allclose(W[h] @ (C + eps * np.eye(16)) @ W[h], np.eye(16), atol=1e-9)
        np.testing.assert_allclose(mu[h], X[h].mean(0), atol=1e-12)


def test_whitening_is_rotation_equivariant():
    """ZCA (not PCA) whitening: rotating the data rotates W the same way."""
    g = np.random.default_rng(4)
    X = g.standard_normal((1, 400, 8)) @ g.standard_normal((8, 8))
    Q, _ = np.linalg.qr(g.standard_normal((8, 8)))
    _, W = O.whitening(X)
    _, Wq = O.whitening(X @ Q)
    np.testing.assert_allclose(Wq[0], Q.T @ W[0] @ Q, atol=1e-9)


def test_whiten_gives_identity_covariance():
    g = np.random.default_rng(5)
    X = g.standard_normal((2, 1000, 12)) @ g.standard_normal((12, 12)) - 1.0
    mu, W = O.whitening(X, eps_rel=0.0)
    Y = O.whiten(X, mu, W)
    for h in range(2):
        np.testing.assert_allclose(Y[h].mean(0), 0.0, atol=1e-10)
        np.testing.assert_allclose(np.cov(Y[h], rowvar=False, bias=True), np.eye(12), atol=1e-9)


def test_decode_search_with_the_same_query_is_decode():
    g = np.random.default_rng(6)
    B, Hq, Hkv, d, K, T = 2, 4, 2, 16, 9, 5
    q = g.standard_normal((B, Hq, d))
    C = g.standard_normal((Hq, K, d))
    Ab = g.standard_normal((Hq, K, d))
    lz = g.uniform(5, 10, (Hq, K))
    Kc = g.standard_normal((B, Hkv, T, d))
    Vc = g.standard_normal((B, Hkv, T, d))
    ll = np.array([T, 3], dtype=np.int32)
    a = O.decode(q, C, Ab, lz, Kc, Vc, ll, 0.25)
    b = O.decode_search(q, q, C, Ab, lz, Kc, Vc, ll, 0.25)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
