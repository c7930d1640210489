// aggregate.cu -- attention-aware aggregation of each cluster's states.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Agregacion": the states (a_i, Z_i) of a cluster's members are fused with
// the online-softmax update rule into one entry (a_bar, Z_bar):
//   m = max_i logZ_i,  w_i = exp(logZ_i - m)
//   a_bar = sum_i w_i a_i / sum_i w_i
//   logZ_bar = m + ln sum_i w_i  [- ln |members| for the mean of Z]
// One warp per cluster walks its member list (perm / seg_off of the k-means
// update) once for the maximum and once for the weighted sum; lanes own
// head-dim slices, so each member row is one coalesced read.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

template <typename T, int D>
__global__ void aggregate_kernel(const T *__restrict__ a, const float *__restrict__ logz,
                                 const int32_t *__restrict__ perm, const int32_t *__restrict__ seg_off,
                                 int H, int N, int K, int zmode, T *a_bar, float *logz_bar) {
    constexpr int EPL = D / 32;
    const size_t w = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (size_t)H * K) return;
    const int h = (int)(w / K), c = (int)(w % K);
    const int lo = seg_off[(size_t)h * (K + 1) + c], hi = seg_off[(size_t)h * (K + 1) + c + 1];
    const int32_t *pm = perm + (size_t)h * N;
    const float *lz = logz + (size_t)h * N;
    float m = kNegInf;
    for (int i = lo + lane; i < hi; i += 32) m = fmaxf(m, lz[pm[i]]);
    m = warp_max(m);
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float out_z = kNegInf;
    if (hi > lo && m != kNegInf) {
        float S = 0.f;
        for (int i = lo; i < hi; ++i) {
            const int p = pm[i];
            const float wi = expf(lz[p] - m);
            S += wi;
            float f[EPL];
            load_vec<T, EPL>(a + ((size_t)h * N + p) * D + lane * EPL, f);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wi, f[e], acc[e]);
        }
        const float inv = 1.f / S;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] *= inv;
        out_z = m + logf(S) - (zmode == 0 ? logf((float)(hi - lo)) : 0.f);
    }
    store_vec<T, EPL>(a_bar + w * D + lane * EPL, acc);
    if (lane == 0) logz_bar[w] = out_z;
}

}  // namespace asmk

cudaError_t asm_aggregate_launch(const void *a, const float *logz, const int32_t *perm,
                                 const int32_t *seg_off, int H, int N, int d, int K, int zmode,
                                 asm_dtype dt, void *a_bar, float *logz_bar, cudaStream_t st) {
    using namespace asmk;
    const size_t HK = (size_t)H * K;
    const unsigned nb = (unsigned)((HK * 32 + 255) / 256);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) aggregate_kernel<T, 128><<<nb, 256, 0, st>>>((const T *)a, logz, perm, seg_off, H, N, K, zmode, (T *)a_bar, logz_bar);
        else aggregate_kernel<T, 64><<<nb, 256, 0, st>>>((const T *)a, logz, perm, seg_off, H, N, K, zmode, (T *)a_bar, logz_bar);
    } else {
        if (d == 128) aggregate_kernel<float, 128><<<nb, 256, 0, st>>>((const float *)a, logz, perm, seg_off, H, N, K, zmode, (float *)a_bar, logz_bar);
        else aggregate_kernel<float, 64><<<nb, 256, 0, st>>>((const float *)a, logz, perm, seg_off, H, N, K, zmode, (float *)a_bar, logz_bar);
    }
    return cudaGetLastError();
}
