"""fp64 CPU oracle for Attention State Memory (ASM): Python side.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the package smoke
check and the benchmark's CPU-baseline leg may import this module.  It loads
``liboracle.so`` (built from ``asm_oracle.c`` by :func:`build`) with ctypes and
marshals numpy arrays; every computation happens in the C file, in double
precision, on the exact storage-dtype values the caller passes (bf16 inputs
are upcast exactly), except the whitening functions, which are numpy in
fp64 (with numpy's symmetric eigensolver as a library step).  Nothing here
imports or calls the CUDA package.

Method source: "Context Memorization for Efficient Long Context Generation"
(gist.science summary of arXiv 2605.18226), section "Metodologia".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "asm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

L2 = 0
COSINE = 1
F32 = 0
BF16 = 1
ZBAR_MEAN = 0
ZBAR_SUM = 1


def build(force: bool = False) -> str:
    """Compile asm_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_max_threads.restype = I
        lib.oracle_state.argtypes = [P, P, P, I, I, D, P, P]
        lib.oracle_merge.argtypes = [P, D, P, D, I, P, P]
        lib.oracle_build_states.argtypes = [P, P, P, I, I, I, I, I, D, I, P, P]
        lib.oracle_kmeanspp_seed.argtypes = [P, I, I, I, I, P, P]
        lib.oracle_kmeanspp_seed_batched.argtypes = [P, I, I, I, I, I, P, I, P]
        lib.oracle_assign.argtypes = [P, P, I, I, I, I, P, P]
        lib.oracle_update.argtypes = [P, P, I, I, I, P, P, P]
        lib.oracle_round_storage.argtypes = [P, ctypes.c_long, I, P]
        lib.oracle_kmeans.argtypes = [P, I, I, I, I, I, I, I, P, P, P, P, P, P]
        lib.oracle_aggregate.argtypes = [P, P, P, I, I, I, I, P, P]
        lib.oracle_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, D, I,
                                      P, P, P, P, P]
        lib.oracle_full_attention.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, D,
                                              P, P]
        lib.oracle_index_search.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P, P]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or a CPU torch tensor (bf16 included)."""
    if hasattr(x, "detach"):  # torch tensor: upcast exactly on the torch side
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def state(q, K, V, scale: float):
    """(a, logZ) of one query q[d] over the block K,V[L,d]."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    d = q.shape[-1]
    L = K.shape[0]
    a = np.zeros(d)
    z = ctypes.c_double()
    _load().oracle_state(_p(q), _p(K), _p(V), L, d, float(scale), _p(a), ctypes.byref(z))
    return a, z.value


def merge(a1, z1: float, a2, z2: float):
    """Online-softmax merge of two states over disjoint key blocks."""
    a1, a2 = _f64(a1), _f64(a2)
    d = a1.shape[-1]
    a = np.zeros(d)
    z = ctypes.c_double()
    _load().oracle_merge(_p(a1), float(z1), _p(a2), float(z2), d, _p(a), ctypes.byref(z))
    return a, z.value


def build_states(Q, K, V, scale: float, A=None, logZ=None, accumulate: bool = False):
    """States of Q[Hq,N,d] over K,V[Hkv,L,d]; merges into (A, logZ) if accumulate."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Hq, N, d = Q.shape
    Hkv, L, _ = K.shape
    A = np.zeros((Hq, N, d)) if A is None else _f64(A).copy()
    logZ = np.full((Hq, N), -np.inf) if logZ is None else _f64(logZ).copy()
    _load().oracle_build_states(_p(Q), _p(K), _p(V), Hq, Hkv, N, L, d, float(scale),
                                int(bool(accumulate)), _p(A), _p(logZ))
    return A, logZ


def kmeanspp_seed(X, u):
    """k-means++ seed indices [H,K] of X[H,N,d] with uniform draws u[H,K]."""
    X, u = _f64(X), _f64(u)
    H, N, d = X.shape
    K = u.shape[1]
    idx = np.zeros((H, K), dtype=np.int32)
    _load().oracle_kmeanspp_seed(_p(X), H, N, d, K, _p(u), _p(idx))
    return idx


def kmeanspp_seed_batched(X, u, K: int, b: int):
    """Batched k-means++ seed indices [H,K] of X[H,N,d]: up to b draws per
    round from the same D2 distribution (uniform draws u[H,U], in order)."""
    X, u = _f64(X), _f64(u)
    H, N, d = X.shape
    U = u.shape[1]
    idx = np.zeros((H, K), dtype=np.int32)
    _load().oracle_kmeanspp_seed_batched(_p(X), H, N, d, int(K), int(b), _p(u), U, _p(idx))
    return idx


def assign(X, C, metric: int = L2):
    """Nearest centre (and relative top-2 gap) of every row of X[N,d] in C[K,d]."""
    X, C = _f64(X), _f64(C)
    N, d = X.shape
    K = C.shape[0]
    out = np.zeros(N, dtype=np.int32)
    gap = np.zeros(N)
    _load().oracle_assign(_p(X), _p(C), N, K, d, int(metric), _p(out), _p(gap))
    return out, gap


def update(X, assign_, Cin):
    """Mean of each cluster's members (an empty cluster keeps Cin's row)."""
    X, a, Cin = _f64(X), _i32(assign_), _f64(Cin)
    N, d = X.shape
    K = Cin.shape[0]
    Cout = np.zeros((K, d))
    counts = np.zeros(K, dtype=np.int32)
    _load().oracle_update(_p(X), _p(a), N, K, d, _p(Cin), _p(Cout), _p(counts))
    return Cout, counts


def round_storage(x, dtype: int):
    """Round fp64 values to fp32 (dtype F32) or to fp32 then bf16 (dtype BF16)."""
    x = _f64(x)
    y = np.zeros_like(x)
    _load().oracle_round_storage(_p(x), x.size, int(dtype), _p(y))
    return y


def kmeans(X, init_idx, iters: int, metric: int = L2, dtype: int = F32):
    """Lloyd iterations per head from X[h, init_idx[h]].

    Returns (C fp64 master [H,K,d], Cq storage-rounded [H,K,d], assign [H,N],
    counts [H,K], inertia [H,iters]).
    """
    X, init = _f64(X), _i32(init_idx)
    H, N, d = X.shape
    K = init.shape[1]
    C = np.zeros((H, K, d))
    Cq = np.zeros((H, K, d))
    a = np.zeros((H, N), dtype=np.int32)
    counts = np.zeros((H, K), dtype=np.int32)
    inertia = np.zeros((H, max(iters, 1)))
    _load().oracle_kmeans(_p(X), H, N, d, K, int(iters), int(metric), int(dtype), _p(init),
                          _p(C), _p(Cq), _p(a), _p(counts), _p(inertia))
    return C, Cq, a, counts, inertia[:, :iters]


def aggregate(A, logZ, assign_, K: int, zmode: int = ZBAR_MEAN):
    """Per-cluster Z-weighted state aggregation of A[N,d], logZ[N]."""
    A, lz, a = _f64(A), _f64(logZ), _i32(assign_)
    N, d = A.shape
    Abar = np.zeros((K, d))
    lzb = np.zeros(K)
    _load().oracle_aggregate(_p(A), _p(lz), _p(a), N, K, d, int(zmode), _p(Abar), _p(lzb))
    return Abar, lzb


def decode(q, C, Abar, logZbar, Kc, Vc, local_len, scale: float, metric: int = L2,
           idx_in=None):
    """One decode step: lookup + merge with local attention.

    q[B,Hq,d], C/Abar[Hq,K,d], logZbar[Hq,K], Kc/Vc[B,Hkv,Tmax,d], local_len[B].
    Returns (out[B,Hq,d], lse[B,Hq], idx[B,Hq], gap[B,Hq]).
    """
    q, C, Abar, lzb = _f64(q), _f64(C), _f64(Abar), _f64(logZbar)
    Kc, Vc, ll = _f64(Kc), _f64(Vc), _i32(local_len)
    B, Hq, d = q.shape
    K = C.shape[1]
    _, Hkv, Tmax, _ = Kc.shape
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    idx = np.zeros((B, Hq), dtype=np.int32)
    gap = np.zeros((B, Hq))
    idx_p = None
    if idx_in is not None:
        idx_in = _i32(idx_in)
        idx_p = _p(idx_in)
    _load().oracle_decode(_p(q), _p(C), _p(Abar), _p(lzb), _p(Kc), _p(Vc), _p(ll), B, Hq, Hkv,
                          K, Tmax, d, float(scale), int(metric), idx_p, _p(out), _p(lse),
                          _p(idx), _p(gap))
    return out, lse, idx, gap


def index_search(q, S, seg_off, C, P: int, metric: int = L2):
    """Two-level centroid search (C oracle ``oracle_index_search``).
    q[B,Hq,d], S[Hq,K1,d], seg_off[Hq,K1+1] int32, C[Hq,K,d] (rows ordered by
    cluster) -> idx[B,Hq], sel[B,Hq,P], gap_sel[B,Hq], gap_idx[B,Hq]."""
    q, S, C = _f64(q), _f64(S), _f64(C)
    so = _i32(seg_off)
    B, Hq, d = q.shape
    K1 = S.shape[1]
    K = C.shape[1]
    idx = np.zeros((B, Hq), dtype=np.int32)
    sel = np.zeros((B, Hq, P), dtype=np.int32)
    gs = np.zeros((B, Hq))
    gi = np.zeros((B, Hq))
    _load().oracle_index_search(_p(q), _p(S), _p(so), _p(C), B, Hq, K, K1, d, int(P), int(metric), _p(idx),
                                _p(sel), _p(gs), _p(gi))
    return idx, sel, gs, gi


def full_attention(q, Kp, Vp, Kc, Vc, local_len, scale: float):
    """Attention of q[B,Hq,d] over the prefix Kp,Vp[Hkv,Lp,d] then the local tokens."""
    q, Kp, Vp = _f64(q), _f64(Kp), _f64(Vp)
    Kc, Vc, ll = _f64(Kc), _f64(Vc), _i32(local_len)
    B, Hq, d = q.shape
    Hkv, Lp, _ = Kp.shape
    Tmax = Kc.shape[2]
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    _load().oracle_full_attention(_p(q), _p(Kp), _p(Vp), Lp, _p(Kc), _p(Vc), _p(ll), B, Hq,
                                  Hkv, Tmax, d, float(scale), _p(out), _p(lse))
    return out, lse


# ------------------------------------------------------------ whitening ---
#
# "Context Memorization for Efficient Long Context Generation", Fase de
# Inferencia Online, Recuperacion: retrieval may whiten the vectors first; the
# pages give no recipe.  Reading: ZCA whitening from the calibration queries'
# covariance, W = (C + eps I)^(-1/2) with C the (1/N) covariance of a head's
# points and eps = eps_rel * trace(C) / d, applied as y = W (x - mu).


def whitening(X, eps_rel: float = 1e-5):
    """ZCA whitening of each head: X[H,N,d] -> mu[H,d], W[H,d,d] (symmetric)."""
    X = _f64(X)
    H, N, d = X.shape
    mu = X.mean(axis=1)
    W = np.empty((H, d, d))
    for h in range(H):
        Xc = X[h] - mu[h]
        C = Xc.T @ Xc / N
        eps = eps_rel * np.trace(C) / d
        lam, V = np.linalg.eigh(C)
        W[h] = (V * (lam + eps) ** -0.5) @ V.T
    return mu, W


def whiten(X, mu, W):
    """y = W (x - mu) for every row of X[H,R,d] (W symmetric): (X - mu) @ W."""
    X, mu, W = _f64(X), _f64(mu), _f64(W)
    return np.einsum("hrd,hde->hre", X - mu[:, None, :], W)


def decode_search(q, qs, C, Abar, logZbar, Kc, Vc, local_len, scale: float, metric: int = L2):
    """One decode step whose centroid search uses qs[B,Hq,d] (for instance the
    whitened queries against whitened centroids C) while the local attention
    and the merge use q.  Returns (out, lse, idx, gap) as :func:`decode`."""
    qs = _f64(qs)
    B, Hq, _ = qs.shape
    idx = np.zeros((B, Hq), dtype=np.int32)
    gap = np.zeros((B, Hq))
    for h in range(Hq):
        idx[:, h], gap[:, h] = assign(qs[:, h], _f64(C)[h], metric)
    out, lse, _, _ = decode(q, C, Abar, logZbar, Kc, Vc, local_len, scale, metric, idx_in=idx)
    return out, lse, idx, gap
