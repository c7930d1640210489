"""Python binding of the ASM C ABI (include/asm.h) for torch CUDA tensors.

Each function has the name of the C entry point it calls and only marshals
arguments: shapes are read from the tensors, pointers and the current CUDA
stream are passed through, and a non-OK status raises :class:`AsmError`.
Every computation runs in the library's sm_100a kernels; outputs are written
into the tensors the caller passes.  The ``alloc_*`` helpers only allocate
correctly sized (and, for decode workspaces, zeroed) buffers.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

ASM_OK, ASM_ERR_INVALID_ARG, ASM_ERR_UNSUPPORTED, ASM_ERR_WORKSPACE, ASM_ERR_CUDA, ASM_ERR_TIMEOUT = range(6)
ASM_F32, ASM_BF16 = 0, 1
ASM_L2, ASM_COSINE = 0, 1
ASM_ZBAR_MEAN, ASM_ZBAR_SUM = 0, 1
ASM_DECODE_PREFETCH_CENTROIDS = 1

_DT = {torch.float32: ASM_F32, torch.bfloat16: ASM_BF16}


class AsmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = _lib.load()
        msg = lib.asm_status_string(status).decode()
        if status == ASM_ERR_CUDA:
            msg += ": " + lib.asm_last_cuda_error().decode()
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AsmError(fn, status)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"storage dtype must be float32 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def status_string(status: int) -> str:
    return _lib.load().asm_status_string(int(status)).decode()


def version() -> str:
    return _lib.load().asm_version().decode()


# ------------------------------------------------------------------ build --

def asm_build_states(q, k, v, scale: float, a, logz, accumulate: bool = False, stream=None):
    """States of q[Hq,N,d] over the prefix block k,v[Hkv,L,d] into a, logz."""
    _contig(q, k, v, a, logz)
    Hq, N, d = q.shape
    Hkv, L, _ = k.shape
    _check("asm_build_states", _lib.load().asm_build_states(
        _p(q), _p(k), _p(v), Hq, Hkv, N, L, d, float(scale), _dt(q), int(bool(accumulate)),
        _p(a), _p(logz), _stream(stream)))


def asm_merge_states(a_acc, logz_acc, a_in, logz_in, stream=None):
    """Fold the states (a_in, logz_in) into (a_acc, logz_acc) by the
    online-softmax identity, row by row (any leading shape, d innermost)."""
    _contig(a_acc, logz_acc, a_in, logz_in)
    if a_acc.shape != a_in.shape or logz_acc.shape != logz_in.shape or a_acc.dtype != a_in.dtype:
        raise AsmError("asm_merge_states", ASM_ERR_INVALID_ARG)
    d = a_acc.shape[-1]
    R = a_acc.numel() // d
    if logz_acc.numel() != R:
        raise AsmError("asm_merge_states", ASM_ERR_INVALID_ARG)
    _check("asm_merge_states", _lib.load().asm_merge_states(
        _p(a_acc), _p(logz_acc), _p(a_in), _p(logz_in), R, d, _dt(a_acc), _stream(stream)))


def asm_kmeanspp_workspace_size(H: int, N: int, d: int, K: int) -> int:
    return int(_lib.load().asm_kmeanspp_workspace_size(H, N, d, K))


def asm_kmeanspp_seed(x, u, init_idx, ws, stream=None):
    """k-means++ indices init_idx[H,K] of x[H,N,d] from the draws u[H,K] (fp64)."""
    _contig(x, u, init_idx)
    H, N, d = x.shape
    K = u.shape[1]
    _check("asm_kmeanspp_seed", _lib.load().asm_kmeanspp_seed(
        _p(x), H, N, d, K, _p(u), _dt(x), _p(init_idx), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def asm_kmeanspp_batched_workspace_size(H: int, N: int, d: int, K: int, batch: int) -> int:
    return int(_lib.load().asm_kmeanspp_batched_workspace_size(H, N, d, K, batch))


def asm_kmeanspp_seed_batched(x, u, init_idx, batch: int, ws, stream=None):
    """Batched k-means++ indices init_idx[H,K] of x[H,N,d]: up to `batch`
    draws per round from the same D2 distribution, draws u[H,U] (fp64) used
    in order."""
    _contig(x, u, init_idx)
    H, N, d = x.shape
    K = init_idx.shape[1]
    _check("asm_kmeanspp_seed_batched", _lib.load().asm_kmeanspp_seed_batched(
        _p(x), H, N, d, K, int(batch), _p(u), u.shape[1], _dt(x), _p(init_idx), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def asm_kmeans_workspace_size(H: int, N: int, d: int, K: int) -> int:
    return int(_lib.load().asm_kmeans_workspace_size(H, N, d, K))


def asm_kmeans_assign(x, centroids_dt, assign, ws, metric: int = ASM_L2, stream=None):
    _contig(x, centroids_dt, assign)
    H, N, d = x.shape
    K = centroids_dt.shape[1]
    _check("asm_kmeans_assign", _lib.load().asm_kmeans_assign(
        _p(x), _p(centroids_dt), H, N, d, K, int(metric), _dt(x), _p(assign), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def asm_kmeans_update(x, assign, centroids, centroids_dt, counts, perm, seg_off, ws, stream=None):
    _contig(x, assign, centroids, centroids_dt, counts, perm, seg_off)
    H, N, d = x.shape
    K = centroids.shape[1]
    _check("asm_kmeans_update", _lib.load().asm_kmeans_update(
        _p(x), _p(assign), H, N, d, K, _dt(x), _p(centroids), _p(centroids_dt), _p(counts),
        _p(perm), _p(seg_off), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def asm_kmeans(x, init_idx, iters: int, centroids, centroids_dt, assign, counts, perm, seg_off,
               ws, metric: int = ASM_L2, stream=None):
    _contig(x, init_idx, centroids, centroids_dt, assign, counts, perm, seg_off)
    H, N, d = x.shape
    K = init_idx.shape[1]
    _check("asm_kmeans", _lib.load().asm_kmeans(
        _p(x), H, N, d, K, int(iters), int(metric), _dt(x), _p(init_idx), _p(centroids),
        _p(centroids_dt), _p(assign), _p(counts), _p(perm), _p(seg_off), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def asm_aggregate(a, logz, perm, seg_off, a_bar, logz_bar, zmode: int = ASM_ZBAR_MEAN,
                  stream=None):
    _contig(a, logz, perm, seg_off, a_bar, logz_bar)
    H, N, d = a.shape
    K = a_bar.shape[1]
    _check("asm_aggregate", _lib.load().asm_aggregate(
        _p(a), _p(logz), _p(perm), _p(seg_off), H, N, d, K, int(zmode), _dt(a), _p(a_bar),
        _p(logz_bar), _stream(stream)))


# ----------------------------------------------------------------- decode --

def asm_decode_workspace_size(B, Hq, Hkv, K, Tmax, d, dtype) -> int:
    return int(_lib.load().asm_decode_workspace_size(B, Hq, Hkv, K, Tmax, d, _DT[dtype]))


def asm_decode_step_launches(B, Hq, Hkv, K, Tmax, d, dtype) -> int:
    """Kernel launches of one asm_decode_step with these sizes on the current device."""
    return int(_lib.load().asm_decode_step_launches(B, Hq, Hkv, K, Tmax, d, _DT[dtype]))


def asm_flash_decode_workspace_size(B, Hq, Hkv, Lp, Tmax, d, dtype) -> int:
    return int(_lib.load().asm_flash_decode_workspace_size(B, Hq, Hkv, Lp, Tmax, d, _DT[dtype]))


def asm_workspace_init(ws, stream=None):
    _check("asm_workspace_init", _lib.load().asm_workspace_init(
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def asm_workspace_error(ws, stream=None) -> int:
    code = ctypes.c_int(0)
    _check("asm_workspace_error", _lib.load().asm_workspace_error(
        _p(ws), ws.numel() * ws.element_size(), ctypes.byref(code), _stream(stream)))
    return code.value


def asm_wait_spin_limit() -> int:
    """Unsuccessful try_wait polls after which any library wait gives up."""
    return int(_lib.load().asm_wait_spin_limit())


def asm_wait_selftest(polls: int, ws, stream=None) -> int:
    """Run a bounded wait that nothing completes (polls try_wait polls, 0 =
    the library's own bound); returns its duration in ns.  The workspace's
    error word then holds ASM_ERR_TIMEOUT (read with asm_workspace_error)."""
    ns = ctypes.c_uint64(0)
    _check("asm_wait_selftest", _lib.load().asm_wait_selftest(
        int(polls), _p(ws), ws.numel() * ws.element_size(), ctypes.byref(ns), _stream(stream)))
    return int(ns.value)


def asm_decode_step(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, scale: float,
                    out, ws, lse_out=None, idx_out=None, metric: int = ASM_L2, flags: int = 0,
                    stream=None):
    """One decode step: lookup + merge with local attention, into out[B,Hq,d]."""
    _contig(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, out, lse_out, idx_out)
    B, Hq, d = q.shape
    K = centroids.shape[1]
    _, Hkv, Tmax, _ = k_cache.shape
    _check("asm_decode_step", _lib.load().asm_decode_step(
        _p(q), _p(centroids), _p(a_bar), _p(logz_bar), _p(k_cache), _p(v_cache), _p(local_len),
        B, Hq, Hkv, K, Tmax, d, float(scale), int(metric), _dt(q), _p(out), _p(lse_out),
        _p(idx_out), int(flags), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def asm_decode_step_search(q, q_search, centroids, a_bar, logz_bar, k_cache, v_cache, local_len,
                           scale: float, out, ws, lse_out=None, idx_out=None, metric: int = ASM_L2,
                           flags: int = 0, stream=None):
    """asm_decode_step whose centroid search uses q_search[B,Hq,d] (e.g. the
    whitened queries) while the local attention and the merge use q."""
    _contig(q, q_search, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, out, lse_out, idx_out)
    if q_search.shape != q.shape or q_search.dtype != q.dtype:
        raise AsmError("asm_decode_step_search", ASM_ERR_INVALID_ARG)
    B, Hq, d = q.shape
    K = centroids.shape[1]
    _, Hkv, Tmax, _ = k_cache.shape
    _check("asm_decode_step_search", _lib.load().asm_decode_step_search(
        _p(q), _p(q_search), _p(centroids), _p(a_bar), _p(logz_bar), _p(k_cache), _p(v_cache),
        _p(local_len), B, Hq, Hkv, K, Tmax, d, float(scale), int(metric), _dt(q), _p(out), _p(lse_out),
        _p(idx_out), int(flags), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def asm_whitening_workspace_size(H: int, d: int) -> int:
    return int(_lib.load().asm_whitening_workspace_size(H, d))


def asm_whitening(x, mu, W, ws, eps_rel: float = 1e-5, stream=None):
    """ZCA whitening of each head of x[H,N,d]: mu[H,d] and W[H,d,d] (fp32)."""
    _contig(x, mu, W)
    H, N, d = x.shape
    _check("asm_whitening", _lib.load().asm_whitening(
        _p(x), H, N, d, _dt(x), float(eps_rel), _p(mu), _p(W), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def asm_whiten(x, mu, W, y, layout: str | None = None, stream=None):
    """y = W[h] (x - mu[h]) row by row.  layout "heads": x, y are [H, R, d]
    (calibration points, centres); "batch": [R, H, d] (decode queries).  When
    omitted it is inferred from which dimension equals H = mu.shape[0], and
    must then be unambiguous."""
    _contig(x, mu, W, y)
    H, d = mu.shape
    if x.shape != y.shape or x.dtype != y.dtype or x.dim() != 3 or x.shape[2] != d:
        raise AsmError("asm_whiten", ASM_ERR_INVALID_ARG)
    if layout is None:
        if (x.shape[0] == H) == (x.shape[1] == H):
            raise AsmError("asm_whiten", ASM_ERR_INVALID_ARG)
        layout = "heads" if x.shape[0] == H else "batch"
    if layout == "heads" and x.shape[0] == H:
        R, sh, sr = x.shape[1], x.shape[1] * d, d
    elif layout == "batch" and x.shape[1] == H:
        R, sh, sr = x.shape[0], d, H * d
    else:
        raise AsmError("asm_whiten", ASM_ERR_INVALID_ARG)
    _check("asm_whiten", _lib.load().asm_whiten(
        _p(x), H, R, d, _dt(x), sh, sr, _p(mu), _p(W), _p(y), sh, sr, _stream(stream)))


def asm_decode_step_noalloc(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len,
                            scale: float, out, lse_out=None, idx_out=None, metric: int = ASM_L2,
                            flags: int = 0, stream=None):
    """asm_decode_step using the library's built-in scratch (no workspace argument)."""
    _contig(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, out, lse_out, idx_out)
    B, Hq, d = q.shape
    K = centroids.shape[1]
    _, Hkv, Tmax, _ = k_cache.shape
    _check("asm_decode_step_noalloc", _lib.load().asm_decode_step_noalloc(
        _p(q), _p(centroids), _p(a_bar), _p(logz_bar), _p(k_cache), _p(v_cache), _p(local_len),
        B, Hq, Hkv, K, Tmax, d, float(scale), int(metric), _dt(q), _p(out), _p(lse_out),
        _p(idx_out), int(flags), _stream(stream)))


def asm_decode_noalloc_error(stream=None) -> int:
    """Device-side status of the last asm_decode_step_noalloc call on the current device."""
    code = ctypes.c_int(0)
    _check("asm_decode_noalloc_error", _lib.load().asm_decode_noalloc_error(ctypes.byref(code), _stream(stream)))
    return code.value


def asm_flash_decode(q, k_prefix, v_prefix, k_cache, v_cache, local_len, scale: float, out, ws,
                     lse_out=None, stream=None):
    """Full attention over a shared explicit prefix plus each row's local tokens."""
    _contig(q, k_prefix, v_prefix, k_cache, v_cache, local_len, out, lse_out)
    B, Hq, d = q.shape
    Hkv, Lp, _ = k_prefix.shape
    Tmax = k_cache.shape[2]
    _check("asm_flash_decode", _lib.load().asm_flash_decode(
        _p(q), _p(k_prefix), _p(v_prefix), Lp, _p(k_cache), _p(v_cache), _p(local_len), B, Hq, Hkv,
        Tmax, d, float(scale), _dt(q), _p(out), _p(lse_out), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


# ---------------------------------------------------------------- helpers --

def asm_index_reorder(perm, centroids, a_bar, logz_bar, centroids_ord, a_bar_ord, logz_bar_ord, stream=None):
    """Lay a memory out by cluster: row i of head h <- row perm[h, i]."""
    _contig(perm, centroids, a_bar, logz_bar, centroids_ord, a_bar_ord, logz_bar_ord)
    H, K, d = centroids.shape
    _check("asm_index_reorder", _lib.load().asm_index_reorder(
        _p(perm), H, K, d, _dt(centroids), _p(centroids), _p(a_bar), _p(logz_bar), _p(centroids_ord),
        _p(a_bar_ord), _p(logz_bar_ord), _stream(stream)))


def asm_decode_indexed_workspace_size(B, Hq, Hkv, K1, P, max_seg, Tmax, d, dtype) -> int:
    return int(_lib.load().asm_decode_indexed_workspace_size(B, Hq, Hkv, K1, P, max_seg, Tmax, d, _DT[dtype]))


def asm_decode_step_indexed(q, supers, seg_off, P: int, max_seg: int, centroids, a_bar, logz_bar, k_cache,
                            v_cache, local_len, scale: float, out, ws, lse_out=None, idx_out=None,
                            metric: int = ASM_L2, stream=None):
    """Decode step with the two-level search over a memory ordered by cluster."""
    _contig(q, supers, seg_off, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, out, lse_out, idx_out)
    B, Hq, d = q.shape
    K1 = supers.shape[1]
    K = centroids.shape[1]
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    _check("asm_decode_step_indexed", _lib.load().asm_decode_step_indexed(
        _p(q), _p(supers), _p(seg_off), K1, int(P), int(max_seg), _p(centroids), _p(a_bar), _p(logz_bar),
        _p(k_cache), _p(v_cache), _p(local_len), B, Hq, Hkv, K, Tmax, d, float(scale), int(metric), _dt(q),
        _p(out), _p(lse_out), _p(idx_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def alloc_workspace(nbytes: int, device, zero: bool = True) -> torch.Tensor:
    """A 256-byte-granular device buffer (zeroed: ready for decode calls)."""
    n = max(256, (int(nbytes) + 255) // 256 * 256)
    t = torch.empty(n, dtype=torch.uint8, device=device)
    if zero:
        asm_workspace_init(t)
    return t
