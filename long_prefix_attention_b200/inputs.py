"""Seeded synthetic inputs for the ASM hot path.

This module draws random tensors and rounds them to the storage dtype; it
holds none of the method's arithmetic.  The tests hand the same tensors to the
CUDA path and to the fp64 oracle, and the benchmark uses them as its workload.

The pages' workloads (LLaMA-3.1-8B activations on ManyICLBench, NBA,
RuleArena) are not available; these recipes stand in for them with the
LLaMA-3.1-8B attention shape (32 query heads, 8 KV heads, head dim 128):

* queries: a Gaussian mixture per head -- component means ~ N(0, I_d), member
  = mean + sigma * N(0, I_d) with a uniformly drawn component;
* prefix and local keys/values: N(0, 1);
* decode-time memories: centroids ~ N(0, 1), states a ~ N(0, 1) and
  logZ ~ U(5, 10) (fp32);
* k-means++ draws: U[0, 1) per head and round, passed to both sides.

Every tensor comes from its own PCG64 stream keyed by (seed, name), so the
tensors do not depend on the order in which they are requested.
"""
from __future__ import annotations

import math
import zlib

import numpy as np
import torch

# Workload descriptions, in the order they are numbered (C0 .. C4).
CONFIGS = [
    dict(name="tiny-fp32", dtype="f32", Hq=2, Hkv=1, d=64, L=512, N=2048, n_mix=32,
         sigma=0.3, K=64, iters=10, B=1, T=16, n_decode=8),
    dict(name="llama31-8b-layer-decode-K1024-T2048-B1", dtype="bf16", Hq=32, Hkv=8, d=128,
         K=1024, T=2048, B=1, n_mix=256, sigma=0.3, logz_lo=5.0, logz_hi=10.0),
    dict(name="llama31-8b-layer-decode-K8192-T4096-B16", dtype="bf16", Hq=32, Hkv=8, d=128,
         K=8192, T=4096, B=16, n_mix=256, sigma=0.3, logz_lo=5.0, logz_hi=10.0),
    dict(name="llama31-8b-layer-build-L16384x4-N65536-K8192", dtype="bf16", Hq=32, Hkv=8,
         d=128, L=16384, chunks=4, N=65536, n_mix=1024, sigma=0.3, K=8192, iters=10),
    dict(name="llama31-8b-32layer-sweep", dtype="bf16", Hq=32, Hkv=8, d=128, layers=32,
         B=(1, 4, 16, 64), K=(1024, 4096, 8192), T=(1024, 8192, 32768), Lp=32768,
         n_mix=256, sigma=0.3, logz_lo=5.0, logz_hi=10.0),
]

BASE_SEED = 0xA5A50000

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _rng(seed: int, name: str) -> np.random.Generator:
    key = zlib.crc32(name.encode())
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed & 0xFFFFFFFF, key])))


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round an fp32/fp64 array to the storage dtype (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(TORCH_DTYPE[dtype])


def normal(seed: int, name: str, shape, dtype: str) -> torch.Tensor:
    return to_storage(_rng(seed, name).standard_normal(shape, dtype=np.float32), dtype)


def uniform(seed: int, name: str, shape, lo: float, hi: float) -> torch.Tensor:
    u = _rng(seed, name).random(shape, dtype=np.float64)
    return torch.from_numpy((lo + (hi - lo) * u).astype(np.float32))


def mixture(seed: int, name: str, H: int, n: int, d: int, n_comp: int, sigma: float,
            dtype: str) -> torch.Tensor:
    """[H, n, d] queries; head h draws from its own n_comp-component mixture."""
    out = np.empty((H, n, d), dtype=np.float32)
    for h in range(H):
        g = _rng(seed, f"{name}/head{h}")
        means = g.standard_normal((n_comp, d), dtype=np.float32)
        z = g.integers(0, n_comp, size=n)
        out[h] = means[z] + np.float32(sigma) * g.standard_normal((n, d), dtype=np.float32)
    return to_storage(out, dtype)


def kmeanspp_uniforms(seed: int, H: int, K: int) -> torch.Tensor:
    """U[0,1) draws [H, K] consumed by the k-means++ seeding rounds (fp64)."""
    return torch.from_numpy(_rng(seed, "kmeanspp_u").random((H, K), dtype=np.float64))


def decode_inputs(cfg: dict, seed: int | None = None, B: int | None = None,
                  K: int | None = None, T: int | None = None, local_len=None) -> dict:
    """Memory (centroids, a_bar, logz_bar), local KV cache and queries of one layer."""
    seed = BASE_SEED + 1 if seed is None else seed
    dt = cfg["dtype"]
    Hq, Hkv, d = cfg["Hq"], cfg["Hkv"], cfg["d"]
    B = cfg["B"] if B is None else B
    K = cfg["K"] if K is None else K
    T = cfg["T"] if T is None else T
    q = mixture(seed, "q", Hq, B, d, cfg["n_mix"], cfg["sigma"], dt).transpose(0, 1).contiguous()
    ins = dict(
        q=q,
        centroids=normal(seed, "centroids", (Hq, K, d), dt),
        a_bar=normal(seed, "a_bar", (Hq, K, d), dt),
        logz_bar=uniform(seed, "logz_bar", (Hq, K), cfg.get("logz_lo", 5.0), cfg.get("logz_hi", 10.0)),
        k_cache=normal(seed, "k_cache", (B, Hkv, T, d), dt),
        v_cache=normal(seed, "v_cache", (B, Hkv, T, d), dt),
        local_len=torch.full((B,), T, dtype=torch.int32) if local_len is None
        else torch.as_tensor(local_len, dtype=torch.int32),
        scale=1.0 / math.sqrt(d),
    )
    return ins


def decode_layer_device(cfg: dict, seed: int, B: int, K: int, T: int, device="cuda", Lp: int = 0) -> dict:
    """One decode layer's inputs generated directly on the device (timing
    workloads of gigabytes, where host generation would dominate): the same
    distributions as :func:`decode_inputs` (N(0,1) centroids, states and
    cache; logZ_bar ~ U(lo, hi); queries from a Gaussian mixture), drawn from
    a seeded device generator, so the values differ from the host ones.
    With Lp > 0 also an explicit prefix K/V [Hkv, Lp, d]."""
    Hq, Hkv, d = cfg["Hq"], cfg["Hkv"], cfg["d"]
    dt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)

    def nrm(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dt)

    means = torch.randn(Hq, cfg["n_mix"], d, generator=g, device=device)
    comp = torch.randint(0, cfg["n_mix"], (Hq, B), generator=g, device=device)
    q = means[torch.arange(Hq, device=device)[:, None], comp] + cfg["sigma"] * torch.randn(
        Hq, B, d, generator=g, device=device)
    lo, hi = cfg.get("logz_lo", 5.0), cfg.get("logz_hi", 10.0)
    out = dict(
        q=q.transpose(0, 1).contiguous().to(dt),
        centroids=nrm(Hq, K, d),
        a_bar=nrm(Hq, K, d),
        logz_bar=lo + (hi - lo) * torch.rand(Hq, K, generator=g, device=device),
        k_cache=nrm(B, Hkv, T, d),
        v_cache=nrm(B, Hkv, T, d),
        local_len=torch.full((B,), T, dtype=torch.int32, device=device),
        scale=1.0 / math.sqrt(d),
    )
    if Lp > 0:
        out["k_prefix"] = nrm(Hkv, Lp, d)
        out["v_prefix"] = nrm(Hkv, Lp, d)
    return out


def build_inputs(cfg: dict, seed: int | None = None, N: int | None = None,
                 L: int | None = None, K: int | None = None, H: int | None = None) -> dict:
    """Calibration queries, prefix K/V and k-means++ draws of the memory build."""
    seed = BASE_SEED + 3 if seed is None else seed
    dt = cfg["dtype"]
    Hq = cfg["Hq"] if H is None else H
    Hkv = max(1, Hq * cfg["Hkv"] // cfg["Hq"])
    d = cfg["d"]
    N = cfg["N"] if N is None else N
    L = cfg["L"] if L is None else L
    K = cfg["K"] if K is None else K
    return dict(
        q=mixture(seed, "calib_q", Hq, N, d, cfg["n_mix"], cfg["sigma"], dt),
        k=normal(seed, "prefix_k", (Hkv, L, d), dt),
        v=normal(seed, "prefix_v", (Hkv, L, d), dt),
        u=kmeanspp_uniforms(seed, Hq, K),
        scale=1.0 / math.sqrt(d),
        K=K,
        iters=cfg.get("iters", 10),
    )
