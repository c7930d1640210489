// launch.h -- internal launch entry points between the C ABI (api.cu) and the
// kernel files.  Arguments are validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "asm.h"

// decode.cu: mode 0 = memory lookup + local attention, 1 = explicit prefix + local.
size_t asm_decode_ws_bytes(int mode, int B, int Hq, int Hkv, int K, int Lp, int Tmax, int d,
                           asm_dtype dt);
cudaError_t asm_decode_launch(int mode, const void *q, const void *centroids, const void *a_bar,
                              const float *logz_bar, const void *k_prefix, const void *v_prefix,
                              int Lp, const void *k_cache, const void *v_cache,
                              const int32_t *local_len, int B, int Hq, int Hkv, int K, int Tmax,
                              int d, float scale, int metric, asm_dtype dt, void *out,
                              float *lse_out, int32_t *idx_out, unsigned flags, void *ws,
                              int num_sms, cudaStream_t st, const void *q_search = nullptr);

// Bytes at the start of a decode workspace that must be zero before a call:
// the error word, and for fp32 the (b, g) arrival counters.
size_t asm_decode_ws_header_bytes(int B, int Hkv, asm_dtype dt);

// api.cu: every argument check of asm_decode_step except the workspace's
asm_status asm_decode_check_args(const void *q, const void *centroids, const void *a_bar, const float *logz_bar,
                                 const void *k_cache, const void *v_cache, const int32_t *local_len, int B, int Hq,
                                 int Hkv, int K, int Tmax, int d, float scale, int metric, asm_dtype dt,
                                 const void *out, const float *lse_out, const int32_t *idx_out, unsigned flags);

// decode_tc.cu: the bf16 path (split units on tensor cores, then a merge kernel)
size_t asm_decode_tc_ws_bytes(int mode, int B, int Hq, int K, int Lp, int Tmax, int d);
cudaError_t asm_decode_tc_launch(int mode, const void *q, const void *centroids, const void *a_bar,
                                 const float *logz_bar, const void *k_prefix, const void *v_prefix, int Lp,
                                 const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                                 int Hq, int Hkv, int K, int Tmax, int d, float scale, int metric, void *out,
                                 float *lse_out, int32_t *idx_out, unsigned flags, void *ws, cudaStream_t st,
                                 const void *q_search = nullptr);

// decode_tc.cu: two-level search decode (bf16)
size_t asm_decode_indexed_tc_ws_bytes(int B, int Hq, int P, int max_seg, int Tmax, int d);
cudaError_t asm_decode_indexed_tc_launch(const void *q, const void *supers, const int32_t *seg_off, int K1, int P,
                                         int max_seg, const void *centroids, const void *a_bar, const float *logz_bar,
                                         const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                                         int Hq, int Hkv, int K, int Tmax, int d, float scale, int metric, void *out,
                                         float *lse_out, int32_t *idx_out, void *ws, cudaStream_t st);

// index.cu: order a memory by cluster
cudaError_t asm_index_reorder_launch(const int32_t *perm, int H, int K, int d, asm_dtype dt, const void *c,
                                     const void *abar, const float *lz, void *c_out, void *abar_out, float *lz_out,
                                     cudaStream_t st);

// build_states.cu
cudaError_t asm_build_states_launch(const void *q, const void *k, const void *v, int Hq, int Hkv,
                                    int N, int L, int d, float scale, asm_dtype dt,
                                    int accumulate, void *a, float *logz, int num_sms,
                                    cudaStream_t st);

// build_states_tc.cu: bf16, d = 128, L > 0 on tcgen05
cudaError_t asm_build_states_tc_launch(const void *q, const void *k, const void *v, int Hq, int Hkv, int N, int L,
                                       float scale, int accumulate, void *a, float *logz, cudaStream_t st);

// build_states_tc.cu: decode partials of a shared prefix for all B rows (bf16, d = 128)
cudaError_t asm_prefix_partials_tc_launch(const void *q, const void *k_prefix, const void *v_prefix, int B, int Hq,
                                          int Hkv, int Lp, int chunk, float scale, float2 *ws_ml, float *ws_o,
                                          int nslots, cudaStream_t st);

// kmeans.cu
size_t asm_kmeanspp_ws_bytes(int H, int N, int d, int K);
cudaError_t asm_kmeanspp_launch(const void *x, int H, int N, int d, int K, const double *u,
                                asm_dtype dt, int32_t *init_idx, void *ws, cudaStream_t st);
size_t asm_kmeans_ws_bytes(int H, int N, int d, int K);
cudaError_t asm_kmeans_init_launch(const void *x, int H, int N, int d, int K, asm_dtype dt,
                                   const int32_t *init_idx, float *centroids, void *centroids_dt,
                                   cudaStream_t st);
size_t asm_kmeanspp_batched_ws_bytes(int H, int N, int d, int K, int batch);
cudaError_t asm_kmeanspp_batched_launch(const void *x, int H, int N, int d, int K, int batch, const double *u,
                                        int U, asm_dtype dt, int32_t *init_idx, void *ws, int num_sms,
                                        cudaStream_t st);
cudaError_t asm_kmeans_assign_launch(const void *x, const void *centroids_dt, int H, int N, int d,
                                     int K, int metric, asm_dtype dt, int32_t *assign, void *ws,
                                     int num_sms, cudaStream_t st);
cudaError_t asm_kmeans_update_launch(const void *x, const int32_t *assign, int H, int N, int d,
                                     int K, asm_dtype dt, float *centroids, void *centroids_dt,
                                     int32_t *counts, int32_t *perm, int32_t *seg_off, void *ws,
                                     cudaStream_t st);

// assign_tc.cu: bf16, d = 128 assignment on tcgen05; `err` is the workspace error word
cudaError_t asm_assign_tc_launch(const void *x, const void *c, const float *norms, const void *bias, int H, int N,
                                 int K, int metric, int32_t *assign, int *err, cudaStream_t st);

// assign_tc.cu: one fused round of batched k-means++ seeding (bf16, d = 128, B <= 256)
cudaError_t asm_bseed_round_tc_launch(const void *x, const void *c, const void *bias,
                                      const float *xn, double *d2, double *bs1, const int *st, int H, int N,
                                      int B, int NR1, int num_sms, int *err, cudaStream_t stream);

// merge.cu: online-softmax merge of two state arrays, row by row
cudaError_t asm_selftest_wait_launch(int polls, int *err, unsigned long long *elapsed_ns, cudaStream_t st);
uint32_t asm_wait_spin_limit_value();
cudaError_t asm_merge_states_launch(void *a, float *z, const void *a2, const float *z2, long long R, int d,
                                    asm_dtype dt, int num_sms, cudaStream_t st);

// aggregate.cu
cudaError_t asm_aggregate_launch(const void *a, const float *logz, const int32_t *perm,
                                 const int32_t *seg_off, int H, int N, int d, int K, int zmode,
                                 asm_dtype dt, void *a_bar, float *logz_bar, cudaStream_t st);

// whiten.cu: ZCA whitening (moments, inverse square root, row transform)
size_t asm_whitening_ws_bytes(int H, int d);
cudaError_t asm_whitening_launch(const void *x, int H, int N, int d, asm_dtype dt, float eps_rel, float *mu,
                                 float *W, void *ws, cudaStream_t st);
cudaError_t asm_whiten_launch(const void *x, int H, int R, int d, asm_dtype dt, long long sh_in, long long sr_in,
                              const float *mu, const float *W, void *y, long long sh_out, long long sr_out,
                              cudaStream_t st);
