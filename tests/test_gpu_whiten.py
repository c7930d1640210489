"""Parity of the whitened retrieval (CUDA, through the C ABI) with the fp64
oracle: the ZCA whitening of each head's calibration queries, the row
transform in both layouts, and the decode step whose centroid search uses
the whitened query.

The pages name whitening before retrieval without a recipe ("Recuperacion"
in "Fase de Inferencia Online" of "Context Memorization for Efficient Long
Context Generation"); the reading implemented is ZCA from the calibration
covariance, W = (C + eps I)^(-1/2).
"""
import numpy as np
import pytest
import torch

from long_prefix_attention_b200 import inputs, ops
from oracle import asm_oracle as O

from gpu_common import GAP, TOL, dev, f64, host, max_abs

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def correlated(H, N, d, dt, seed):
    """Points with a strongly non-isotropic covariance and a non-zero mean."""
    g = np.random.default_rng(seed)
    out = np.empty((H, N, d), dtype=np.float32)
    for h in range(H):
        A = g.standard_normal((d, d)) * np.linspace(0.05, 2.0, d)[:, None]
        out[h] = g.standard_normal((N, d)) @ A + g.standard_normal(d)
    return torch.from_numpy(out).to(DT[dt])


def gpu_whitening(x, eps_rel=1e-5):
    H, N, d = x.shape
    mu = torch.empty(H, d, dtype=torch.float32, device="cuda")
    W = torch.empty(H, d, d, dtype=torch.float32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_whitening_workspace_size(H, d), "cuda")
    ops.asm_whitening(x, mu, W, ws, eps_rel=eps_rel)
    torch.cuda.synchronize()
    return mu, W, ops.asm_workspace_error(ws)


@pytest.mark.parametrize("dt,d,N", [("bf16", 128, 5000), ("f32", 64, 3001), ("bf16", 64, 20000), ("f32", 128, 700)])
def test_whitening_matches_the_oracle(dt, d, N):
    x = correlated(2, N, d, dt, seed=d + N)
    mu, W, err = gpu_whitening(dev(x))
    assert err == 0
    o_mu, o_W = O.whitening(x, eps_rel=1e-5)
    assert max_abs(f64(mu), o_mu) <= 1e-5 * max(1.0, np.abs(o_mu).max())
    # fp32 output of an fp64 computation
    assert max_abs(f64(W), o_W) <= 1e-5 * np.abs(o_W).max()


def test_whitened_points_have_identity_covariance():
    x = correlated(2, 20000, 128, "f32", seed=3)
    xd = dev(x)
    mu, W, err = gpu_whitening(xd, eps_rel=0.0)
    assert err == 0
    y = torch.empty_like(xd)
    ops.asm_whiten(xd, mu, W, y)
    torch.cuda.synchronize()
    yh = host(y).numpy().astype(np.float64)
    for h in range(2):
        np.testing.assert_allclose(yh[h].mean(0), 0.0, atol=1e-3)
        np.testing.assert_allclose(np.cov(yh[h], rowvar=False, bias=True), np.eye(128), atol=2e-3)


def test_singular_covariance_without_regularisation_is_flagged():
    """A coordinate that is zero in every point: its row and column of C are
    exactly zero, so with eps_rel = 0 the inverse square root does not exist
    and the bounded iteration reports it instead of returning W.  (A
    covariance that is singular only up to rounding has tiny positive
    eigenvalues instead, and its exact inverse square root is returned.)"""
    x = correlated(1, 400, 64, "f32", seed=4)
    x[:, :, 5] = 0.0
    _, _, err = gpu_whitening(dev(x), eps_rel=0.0)
    assert err == ops.ASM_ERR_TIMEOUT
    # with the default regularisation the same points whiten fine
    _, W, err = gpu_whitening(dev(x), eps_rel=1e-5)
    assert err == 0
    _, o_W = O.whitening(x, eps_rel=1e-5)
    assert max_abs(f64(W), o_W) <= 1e-5 * np.abs(o_W).max()


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_whiten_rows_in_both_layouts(dt):
    H, N, d, B = 4, 777, 128, 5
    x = correlated(H, N, d, dt, seed=7)
    mu, W, _ = gpu_whitening(dev(x))
    # calibration layout [H, N, d]
    y = torch.empty_like(dev(x))
    ops.asm_whiten(dev(x), mu, W, y)
    ref = O.whiten(x, f64(mu), f64(W))
    assert max_abs(f64(y), ref) <= TOL[DT[dt]] * max(1.0, np.abs(ref).max())
    # decode layout [B, H, d]
    q = x[:, :B].transpose(0, 1).contiguous()
    yq = torch.empty_like(dev(q))
    ops.asm_whiten(dev(q), mu, W, yq)
    torch.cuda.synchronize()
    refq = O.whiten(q.transpose(0, 1), f64(mu), f64(W)).transpose(1, 0, 2)
    assert max_abs(f64(yq), refq) <= TOL[DT[dt]] * max(1.0, np.abs(refq).max())


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_decode_with_whitened_search_matches_the_oracle(dt):
    """Centres and queries whitened on the GPU; the search uses the whitened
    query, the attention and merge the original one."""
    Hq, Hkv, d, K, B, T = 8, 2, 128, 300, 3, 90
    cfg = dict(inputs.CONFIGS[1], dtype=dt, Hq=Hq, Hkv=Hkv, d=d, n_mix=16)
    ins = inputs.decode_inputs(cfg, seed=31, B=B, K=K, T=T, local_len=[90, 41, 0])
    calib = correlated(Hq, 4000, d, dt, seed=32)
    mu, W, _ = gpu_whitening(dev(calib))
    cw = torch.empty_like(dev(ins["centroids"]))
    ops.asm_whiten(dev(ins["centroids"]), mu, W, cw)
    q = dev(ins["q"])
    qs = torch.empty_like(q)
    ops.asm_whiten(q, mu, W, qs)
    kc, vc, ll = dev(ins["k_cache"]), dev(ins["v_cache"]), dev(ins["local_len"])
    ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, d, q.dtype), "cuda")
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, Hq, dtype=torch.int32, device="cuda")
    ops.asm_decode_step_search(q, qs, cw, dev(ins["a_bar"]), dev(ins["logz_bar"]), kc, vc, ll, ins["scale"],
                               out, ws, lse_out=lse, idx_out=idx)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    o_out, o_lse, o_idx, o_gap = O.decode_search(ins["q"], host(qs), host(cw), ins["a_bar"], ins["logz_bar"],
                                                 ins["k_cache"], ins["v_cache"], ins["local_len"], ins["scale"])
    g_idx = host(idx).numpy()
    bad = g_idx != o_idx
    assert not (bad & (o_gap >= GAP)).any()
    if bad.any():  # near-ties: the oracle at the GPU's choice
        o_out, o_lse, _, _ = O.decode(ins["q"], host(cw), ins["a_bar"], ins["logz_bar"], ins["k_cache"],
                                      ins["v_cache"], ins["local_len"], ins["scale"], idx_in=g_idx)
    tol = TOL[q.dtype]
    assert max_abs(f64(out), o_out) <= tol
    assert max_abs(f64(lse), o_lse) <= tol
    # the whitened search differs from the plain one somewhere (it is used)
    plain = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"], ins["k_cache"], ins["v_cache"],
                     ins["local_len"], ins["scale"])[2]
    assert (plain != o_idx).any()
