// api.cu -- the C ABI declared in include/asm.h: host-side validation (no
// CUDA call happens before every argument has been checked), workspace
// sizing and dispatch to the kernel files.
#include <cuda_runtime.h>
#include <stdint.h>

#include "asm.h"
#include "launch.h"

namespace {

bool aligned(const void *p, size_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool dt_ok(asm_dtype dt) { return dt == ASM_F32 || dt == ASM_BF16; }
bool d_ok(int d) { return d == 64 || d == 128; }
bool group_ok(int Hq, int Hkv) {
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return false;
    const int G = Hq / Hkv;
    return G == 1 || G == 2 || G == 4 || G == 8;
}

// Multiprocessor count of the current device (cached per device ordinal).
int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// The last CUDA error this thread's library calls observed (cudaSuccess if none).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

asm_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return ASM_OK;
    t_last_cuda_error = e;
    return ASM_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *asm_last_cuda_error(void) {
    return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

const char *asm_status_string(asm_status s) {
    switch (s) {
        case ASM_OK: return "ok";
        case ASM_ERR_INVALID_ARG: return "invalid argument";
        case ASM_ERR_UNSUPPORTED: return "unsupported shape";
        case ASM_ERR_WORKSPACE: return "workspace missing or too small";
        case ASM_ERR_CUDA: return "CUDA error";
        case ASM_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

const char *asm_version(void) { return "0.1.0"; }

asm_status asm_build_states(const void *q, const void *k, const void *v, int Hq, int Hkv, int N,
                            int L, int d, float scale, asm_dtype dt, int accumulate, void *a,
                            float *logz, cudaStream_t stream) {
    if (!dt_ok(dt) || N < 0 || L < 0 || !(scale == scale)) return ASM_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || !group_ok(Hq, Hkv)) return ASM_ERR_UNSUPPORTED;
    if (N == 0) return ASM_OK;
    if (!aligned(q, 16) || !aligned(a, 16) || !aligned(logz, 4)) return ASM_ERR_INVALID_ARG;
    if (L > 0 && (!aligned(k, 16) || !aligned(v, 16))) return ASM_ERR_INVALID_ARG;
    return cuda_status(asm_build_states_launch(q, k, v, Hq, Hkv, N, L, d, scale, dt, accumulate ? 1 : 0,
                                               a, logz, num_sms(), stream));
}

asm_status asm_merge_states(void *a_acc, float *logz_acc, const void *a_in, const float *logz_in, int64_t R,
                            int d, asm_dtype dt, cudaStream_t stream) {
    if (!dt_ok(dt) || R < 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (R == 0) return ASM_OK;
    if (!aligned(a_acc, 16) || !aligned(a_in, 16) || !aligned(logz_acc, 4) || !aligned(logz_in, 4))
        return ASM_ERR_INVALID_ARG;
    // the two sets must not overlap (the accumulator is written in place)
    const size_t es = dt == ASM_BF16 ? 2 : 4, ab = (size_t)R * d * es, zb = (size_t)R * sizeof(float);
    const char *pa = static_cast<const char *>(a_acc), *pb = static_cast<const char *>(a_in);
    const char *za = reinterpret_cast<const char *>(logz_acc), *zb2 = reinterpret_cast<const char *>(logz_in);
    if ((pa < pb + ab && pb < pa + ab) || (za < zb2 + zb && zb2 < za + zb)) return ASM_ERR_INVALID_ARG;
    return cuda_status(asm_merge_states_launch(a_acc, logz_acc, a_in, logz_in, (long long)R, d, dt, num_sms(),
                                               stream));
}

size_t asm_kmeanspp_workspace_size(int H, int N, int d, int K) {
    if (H < 1 || N < 1 || K < 1) return 0;
    return asm_kmeanspp_ws_bytes(H, N, d, K);
}

asm_status asm_kmeanspp_seed(const void *x, int H, int N, int d, int K, const double *u,
                             asm_dtype dt, int32_t *init_idx, void *ws, size_t ws_bytes,
                             cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1 || K > N) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || N > (1 << 24)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(u, 8) || !aligned(init_idx, 4)) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_kmeanspp_ws_bytes(H, N, d, K)) return ASM_ERR_WORKSPACE;
    return cuda_status(asm_kmeanspp_launch(x, H, N, d, K, u, dt, init_idx, ws, stream));
}

size_t asm_kmeanspp_batched_workspace_size(int H, int N, int d, int K, int batch) {
    if (H < 1 || N < 1 || K < 1 || batch < 1 || batch > 256 || !d_ok(d)) return 0;
    return asm_kmeanspp_batched_ws_bytes(H, N, d, K, batch);
}

asm_status asm_kmeanspp_seed_batched(const void *x, int H, int N, int d, int K, int batch, const double *u,
                                     int U, asm_dtype dt, int32_t *init_idx, void *ws, size_t ws_bytes,
                                     cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1 || K > N || batch < 1 || U < 1) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || batch > 256 || N > (1 << 21)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(u, 8) || !aligned(init_idx, 4)) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_kmeanspp_batched_ws_bytes(H, N, d, K, batch)) return ASM_ERR_WORKSPACE;
    return cuda_status(asm_kmeanspp_batched_launch(x, H, N, d, K, batch, u, U, dt, init_idx, ws, num_sms(), stream));
}

size_t asm_kmeans_workspace_size(int H, int N, int d, int K) {
    if (H < 1 || N < 1 || K < 1) return 0;
    return asm_kmeans_ws_bytes(H, N, d, K);
}

asm_status asm_kmeans_assign(const void *x, const void *centroids_dt, int H, int N, int d, int K,
                             asm_metric metric, asm_dtype dt, int32_t *assign, void *ws,
                             size_t ws_bytes, cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1) return ASM_ERR_INVALID_ARG;
    if (metric != ASM_L2 && metric != ASM_COSINE) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(centroids_dt, 16) || !aligned(assign, 4)) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_kmeans_ws_bytes(H, N, d, K)) return ASM_ERR_WORKSPACE;
    return cuda_status(asm_kmeans_assign_launch(x, centroids_dt, H, N, d, K, (int)metric, dt, assign,
                                                ws, num_sms(), stream));
}

asm_status asm_kmeans_update(const void *x, const int32_t *assign, int H, int N, int d, int K,
                             asm_dtype dt, float *centroids, void *centroids_dt, int32_t *counts,
                             int32_t *perm, int32_t *seg_off, void *ws, size_t ws_bytes,
                             cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(assign, 4) || !aligned(centroids, 16) || !aligned(centroids_dt, 16) ||
        !aligned(counts, 4) || !aligned(perm, 4) || !aligned(seg_off, 4))
        return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_kmeans_ws_bytes(H, N, d, K)) return ASM_ERR_WORKSPACE;
    return cuda_status(asm_kmeans_update_launch(x, assign, H, N, d, K, dt, centroids, centroids_dt,
                                                counts, perm, seg_off, ws, stream));
}

asm_status asm_kmeans(const void *x, int H, int N, int d, int K, int iters, asm_metric metric,
                      asm_dtype dt, const int32_t *init_idx, float *centroids, void *centroids_dt,
                      int32_t *assign, int32_t *counts, int32_t *perm, int32_t *seg_off, void *ws,
                      size_t ws_bytes, cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1 || K > N || iters < 1) return ASM_ERR_INVALID_ARG;
    if (metric != ASM_L2 && metric != ASM_COSINE) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(init_idx, 4) || !aligned(centroids, 16) || !aligned(centroids_dt, 16) ||
        !aligned(assign, 4) || !aligned(counts, 4) || !aligned(perm, 4) || !aligned(seg_off, 4))
        return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_kmeans_ws_bytes(H, N, d, K)) return ASM_ERR_WORKSPACE;
    cudaError_t e = asm_kmeans_init_launch(x, H, N, d, K, dt, init_idx, centroids, centroids_dt, stream);
    const int sms = num_sms();
    for (int t = 0; t < iters && e == cudaSuccess; ++t) {
        e = asm_kmeans_assign_launch(x, centroids_dt, H, N, d, K, (int)metric, dt, assign, ws, sms, stream);
        if (e == cudaSuccess)
            e = asm_kmeans_update_launch(x, assign, H, N, d, K, dt, centroids, centroids_dt, counts, perm,
                                         seg_off, ws, stream);
    }
    return cuda_status(e);
}

asm_status asm_aggregate(const void *a, const float *logz, const int32_t *perm,
                         const int32_t *seg_off, int H, int N, int d, int K, asm_zbar_mode zmode,
                         asm_dtype dt, void *a_bar, float *logz_bar, cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || K < 1) return ASM_ERR_INVALID_ARG;
    if (zmode != ASM_ZBAR_MEAN && zmode != ASM_ZBAR_SUM) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(a, 16) || !aligned(logz, 4) || !aligned(perm, 4) || !aligned(seg_off, 4) ||
        !aligned(a_bar, 16) || !aligned(logz_bar, 4))
        return ASM_ERR_INVALID_ARG;
    return cuda_status(asm_aggregate_launch(a, logz, perm, seg_off, H, N, d, K, (int)zmode, dt, a_bar,
                                            logz_bar, stream));
}

size_t asm_decode_workspace_size(int B, int Hq, int Hkv, int K, int Tmax, int d, asm_dtype dt) {
    if (B < 1 || Hq < 1 || Hkv < 1 || K < 1 || Tmax < 0 || !d_ok(d) || !dt_ok(dt)) return 0;
    return asm_decode_ws_bytes(0, B, Hq, Hkv, K, 0, Tmax, d, dt);
}

int asm_decode_step_launches(int B, int Hq, int Hkv, int K, int Tmax, int d, asm_dtype dt) {
    if (!dt_ok(dt) || B < 1 || B > 4096 || K < 1 || Tmax < 0 || !d_ok(d) || !group_ok(Hq, Hkv)) return -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return dt == ASM_F32 ? 1 : 2;
}

}  // extern "C"

// Every check of asm_decode_step except the workspace's.
asm_status asm_decode_check_args(const void *q, const void *centroids, const void *a_bar, const float *logz_bar,
                                 const void *k_cache, const void *v_cache, const int32_t *local_len, int B, int Hq,
                                 int Hkv, int K, int Tmax, int d, float scale, int metric, asm_dtype dt,
                                 const void *out, const float *lse_out, const int32_t *idx_out, unsigned flags) {
    if (!dt_ok(dt) || B < 1 || B > 4096 || K < 1 || Tmax < 0 || !(scale == scale)) return ASM_ERR_INVALID_ARG;
    if (metric != ASM_L2 && metric != ASM_COSINE) return ASM_ERR_INVALID_ARG;
    if ((flags & ~ASM_DECODE_PREFETCH_CENTROIDS) != 0) return ASM_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || !group_ok(Hq, Hkv)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(centroids, 16) || !aligned(a_bar, 16) || !aligned(logz_bar, 4) ||
        !aligned(local_len, 4) || !aligned(out, 16))
        return ASM_ERR_INVALID_ARG;
    if (Tmax > 0 && (!aligned(k_cache, 16) || !aligned(v_cache, 16))) return ASM_ERR_INVALID_ARG;
    if ((lse_out && !aligned(lse_out, 4)) || (idx_out && !aligned(idx_out, 4))) return ASM_ERR_INVALID_ARG;
    return ASM_OK;
}

extern "C" {

asm_status asm_decode_step(const void *q, const void *centroids, const void *a_bar,
                           const float *logz_bar, const void *k_cache, const void *v_cache,
                           const int32_t *local_len, int B, int Hq, int Hkv, int K, int Tmax, int d,
                           float scale, asm_metric metric, asm_dtype dt, void *out, float *lse_out,
                           int32_t *idx_out, unsigned flags, void *ws, size_t ws_bytes,
                           cudaStream_t stream) {
    const asm_status v = asm_decode_check_args(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, B, Hq,
                                               Hkv, K, Tmax, d, scale, (int)metric, dt, out, lse_out, idx_out, flags);
    if (v != ASM_OK) return v;
    if (!aligned(ws, 16) || ws_bytes < asm_decode_ws_bytes(0, B, Hq, Hkv, K, 0, Tmax, d, dt))
        return ASM_ERR_WORKSPACE;
    return cuda_status(asm_decode_launch(0, q, centroids, a_bar, logz_bar, nullptr, nullptr, 0, k_cache,
                                         v_cache, local_len, B, Hq, Hkv, K, Tmax, d, scale, (int)metric,
                                         dt, out, lse_out, idx_out, flags, ws, num_sms(), stream));
}

asm_status asm_decode_step_search(const void *q, const void *q_search, const void *centroids, const void *a_bar,
                                  const float *logz_bar, const void *k_cache, const void *v_cache,
                                  const int32_t *local_len, int B, int Hq, int Hkv, int K, int Tmax, int d,
                                  float scale, asm_metric metric, asm_dtype dt, void *out, float *lse_out,
                                  int32_t *idx_out, unsigned flags, void *ws, size_t ws_bytes,
                                  cudaStream_t stream) {
    if (!aligned(q_search, 16)) return ASM_ERR_INVALID_ARG;
    if (!dt_ok(dt) || B < 1 || B > 4096 || K < 1 || Tmax < 0 || !(scale == scale)) return ASM_ERR_INVALID_ARG;
    if (metric != ASM_L2 && metric != ASM_COSINE) return ASM_ERR_INVALID_ARG;
    if ((flags & ~ASM_DECODE_PREFETCH_CENTROIDS) != 0) return ASM_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || !group_ok(Hq, Hkv)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(centroids, 16) || !aligned(a_bar, 16) || !aligned(logz_bar, 4) ||
        !aligned(local_len, 4) || !aligned(out, 16))
        return ASM_ERR_INVALID_ARG;
    if (Tmax > 0 && (!aligned(k_cache, 16) || !aligned(v_cache, 16))) return ASM_ERR_INVALID_ARG;
    if ((lse_out && !aligned(lse_out, 4)) || (idx_out && !aligned(idx_out, 4))) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_decode_ws_bytes(0, B, Hq, Hkv, K, 0, Tmax, d, dt))
        return ASM_ERR_WORKSPACE;
    return cuda_status(asm_decode_launch(0, q, centroids, a_bar, logz_bar, nullptr, nullptr, 0, k_cache,
                                         v_cache, local_len, B, Hq, Hkv, K, Tmax, d, scale, (int)metric,
                                         dt, out, lse_out, idx_out, flags, ws, num_sms(), stream, q_search));
}

size_t asm_whitening_workspace_size(int H, int d) {
    if (H < 1 || !d_ok(d)) return 0;
    return asm_whitening_ws_bytes(H, d);
}

asm_status asm_whitening(const void *x, int H, int N, int d, asm_dtype dt, float eps_rel, float *mu, float *W,
                         void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || N < 1 || !(eps_rel >= 0.f) || !(eps_rel < 1e30f)) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(mu, 4) || !aligned(W, 4)) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_whitening_ws_bytes(H, d)) return ASM_ERR_WORKSPACE;
    return cuda_status(asm_whitening_launch(x, H, N, d, dt, eps_rel, mu, W, ws, stream));
}

asm_status asm_whiten(const void *x, int H, int R, int d, asm_dtype dt, int64_t head_stride, int64_t row_stride,
                      const float *mu, const float *W, void *y, int64_t y_head_stride, int64_t y_row_stride,
                      cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || R < 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (head_stride < 0 || row_stride < 0 || y_head_stride < 0 || y_row_stride < 0) return ASM_ERR_INVALID_ARG;
    const size_t es = dt == ASM_BF16 ? 2 : 4;
    if (!aligned(x, es) || !aligned(y, es) || !aligned(mu, 4) || !aligned(W, 4)) return ASM_ERR_INVALID_ARG;
    if (R == 0) return ASM_OK;
    return cuda_status(asm_whiten_launch(x, H, R, d, dt, (long long)head_stride, (long long)row_stride, mu, W, y,
                                         (long long)y_head_stride, (long long)y_row_stride, stream));
}

asm_status asm_index_reorder(const int32_t *perm, int H, int K, int d, asm_dtype dt, const void *centroids,
                             const void *a_bar, const float *logz_bar, void *centroids_ord, void *a_bar_ord,
                             float *logz_bar_ord, cudaStream_t stream) {
    if (!dt_ok(dt) || H < 1 || K < 1) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(perm, 4) || !aligned(centroids, 16) || !aligned(a_bar, 16) || !aligned(logz_bar, 4) ||
        !aligned(centroids_ord, 16) || !aligned(a_bar_ord, 16) || !aligned(logz_bar_ord, 4))
        return ASM_ERR_INVALID_ARG;
    if (centroids_ord == centroids || a_bar_ord == a_bar || logz_bar_ord == logz_bar) return ASM_ERR_INVALID_ARG;
    return cuda_status(asm_index_reorder_launch(perm, H, K, d, dt, centroids, a_bar, logz_bar, centroids_ord,
                                                a_bar_ord, logz_bar_ord, stream));
}

size_t asm_decode_indexed_workspace_size(int B, int Hq, int Hkv, int K1, int P, int max_seg, int Tmax, int d,
                                         asm_dtype dt) {
    if (B < 1 || Hq < 1 || Hkv < 1 || K1 < 1 || P < 1 || max_seg < 1 || Tmax < 0 || !d_ok(d) || dt != ASM_BF16)
        return 0;
    return asm_decode_indexed_tc_ws_bytes(B, Hq, P, max_seg, Tmax, d);
}

asm_status asm_decode_step_indexed(const void *q, const void *supers, const int32_t *seg_off, int K1, int P,
                                   int max_seg, const void *centroids, const void *a_bar, const float *logz_bar,
                                   const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                                   int Hq, int Hkv, int K, int Tmax, int d, float scale, asm_metric metric,
                                   asm_dtype dt, void *out, float *lse_out, int32_t *idx_out, void *ws,
                                   size_t ws_bytes, cudaStream_t stream) {
    if (!dt_ok(dt) || B < 1 || B > 4096 || K < 1 || Tmax < 0 || !(scale == scale)) return ASM_ERR_INVALID_ARG;
    if (metric != ASM_L2 && metric != ASM_COSINE) return ASM_ERR_INVALID_ARG;
    if (K1 < 1 || K1 > K || K1 > 4096 || P < 1 || P > K1 || P > 32 || max_seg < 1 || max_seg > K)
        return ASM_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ASM_ERR_INVALID_ARG;
    if (dt != ASM_BF16 || !d_ok(d) || !group_ok(Hq, Hkv)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(supers, 16) || !aligned(seg_off, 4) || !aligned(centroids, 16) ||
        !aligned(a_bar, 16) || !aligned(logz_bar, 4) || !aligned(local_len, 4) || !aligned(out, 16))
        return ASM_ERR_INVALID_ARG;
    if (Tmax > 0 && (!aligned(k_cache, 16) || !aligned(v_cache, 16))) return ASM_ERR_INVALID_ARG;
    if ((lse_out && !aligned(lse_out, 4)) || (idx_out && !aligned(idx_out, 4))) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_decode_indexed_tc_ws_bytes(B, Hq, P, max_seg, Tmax, d))
        return ASM_ERR_WORKSPACE;
    return cuda_status(asm_decode_indexed_tc_launch(q, supers, seg_off, K1, P, max_seg, centroids, a_bar, logz_bar,
                                                    k_cache, v_cache, local_len, B, Hq, Hkv, K, Tmax, d, scale,
                                                    (int)metric, out, lse_out, idx_out, ws, stream));
}

size_t asm_flash_decode_workspace_size(int B, int Hq, int Hkv, int Lp, int Tmax, int d, asm_dtype dt) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Lp < 0 || Tmax < 0 || !d_ok(d) || !dt_ok(dt)) return 0;
    return asm_decode_ws_bytes(1, B, Hq, Hkv, 0, Lp, Tmax, d, dt);
}

asm_status asm_flash_decode(const void *q, const void *k_prefix, const void *v_prefix, int Lp,
                            const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                            int Hq, int Hkv, int Tmax, int d, float scale, asm_dtype dt, void *out,
                            float *lse_out, void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (!dt_ok(dt) || B < 1 || B > 4096 || Lp < 0 || Tmax < 0 || Lp + Tmax < 1 || !(scale == scale))
        return ASM_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ASM_ERR_INVALID_ARG;
    if (!d_ok(d) || !group_ok(Hq, Hkv)) return ASM_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(local_len, 4) || !aligned(out, 16)) return ASM_ERR_INVALID_ARG;
    if (Lp > 0 && (!aligned(k_prefix, 16) || !aligned(v_prefix, 16))) return ASM_ERR_INVALID_ARG;
    if (Tmax > 0 && (!aligned(k_cache, 16) || !aligned(v_cache, 16))) return ASM_ERR_INVALID_ARG;
    if (lse_out && !aligned(lse_out, 4)) return ASM_ERR_INVALID_ARG;
    if (!aligned(ws, 16) || ws_bytes < asm_decode_ws_bytes(1, B, Hq, Hkv, 0, Lp, Tmax, d, dt))
        return ASM_ERR_WORKSPACE;
    return cuda_status(asm_decode_launch(1, q, nullptr, nullptr, nullptr, k_prefix, v_prefix, Lp, k_cache,
                                         v_cache, local_len, B, Hq, Hkv, 1, Tmax, d, scale, 0, dt, out,
                                         lse_out, nullptr, 0u, ws, num_sms(), stream));
}

asm_status asm_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (!aligned(ws, 16) || ws_bytes == 0) return ASM_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

uint32_t asm_wait_spin_limit(void) { return asm_wait_spin_limit_value(); }

asm_status asm_wait_selftest(int polls, void *ws, size_t ws_bytes, uint64_t *elapsed_ns, cudaStream_t stream) {
    if (polls < 0 || !aligned(ws, 16) || ws_bytes < 256 || elapsed_ns == nullptr) return ASM_ERR_INVALID_ARG;
    char *b = static_cast<char *>(ws);
    unsigned long long *dev_ns = reinterpret_cast<unsigned long long *>(b + 8);
    cudaError_t e = cudaMemsetAsync(ws, 0, 16, stream);
    if (e == cudaSuccess) e = asm_selftest_wait_launch(polls, reinterpret_cast<int *>(b), dev_ns, stream);
    unsigned long long v = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, dev_ns, sizeof(v), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_status(e);
    *elapsed_ns = v;
    return ASM_OK;
}

asm_status asm_workspace_error(const void *ws, size_t ws_bytes, int *code, cudaStream_t stream) {
    if (!aligned(ws, 16) || ws_bytes < 256 || code == nullptr) return ASM_ERR_INVALID_ARG;
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return ASM_ERR_CUDA;
    *code = v;
    return ASM_OK;
}

}  // extern "C"
