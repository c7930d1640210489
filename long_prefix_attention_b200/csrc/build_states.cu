// build_states.cu -- attention state (a, logZ) of every calibration query
// over a block of the prefix, with the chunk-merge epilogue.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia:
// "Recoleccion" (each query's attention state over the prefix is recorded)
// and "Eficiencia" (a long prefix is encoded in chunks whose states are
// merged with the online-softmax identity).
//
// This file holds the portable CUDA-core kernel, used for fp32 storage and
// for head dim 64; bf16 with head dim 128 is dispatched to the tcgen05
// kernel in build_states_tc.cu.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

constexpr int kBsWarps = 4;
constexpr int kBsQPerWarp = 8;
constexpr int kBsQ = kBsWarps * kBsQPerWarp;  // queries per CTA
constexpr int kBsKT = 32;                     // keys per smem tile

// Online-softmax merge of a stored state with a new one, natural-log Z.
__device__ __forceinline__ void merge_state(float za, float zb, float &wa, float &wb, float &z) {
    if (za == kNegInf && zb == kNegInf) {
        wa = 0.f; wb = 0.f; z = kNegInf;
        return;
    }
    const float m = fmaxf(za, zb);
    const float ea = expf(za - m), eb = expf(zb - m);
    z = m + logf(ea + eb);
    wa = ea / (ea + eb);
    wb = eb / (ea + eb);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBsWarps * 32)
build_states_simple(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    int Hq, int Hkv, int N, int L, float qscale, int accumulate, T *a,
                    float *logz) {
    constexpr int EPL = D / 32;
    __shared__ __align__(16) T ks[kBsKT * D];
    __shared__ __align__(16) T vs[kBsKT * D];
    const int h = blockIdx.y, g = h / (Hq / Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kBsQ + warp * kBsQPerWarp;

    float qr[kBsQPerWarp][EPL], o[kBsQPerWarp][EPL], m[kBsQPerWarp], l[kBsQPerWarp];
#pragma unroll
    for (int j = 0; j < kBsQPerWarp; ++j) {
        const int n = min(n0 + j, N - 1);
        load_vec<T, EPL>(q + ((size_t)h * N + n) * D + lane * EPL, qr[j]);
#pragma unroll
        for (int e = 0; e < EPL; ++e) { qr[j][e] *= qscale; o[j][e] = 0.f; }
        m[j] = kNegInf;
        l[j] = 0.f;
    }
    const T *kg = k + (size_t)g * L * D;
    const T *vg = v + (size_t)g * L * D;
    constexpr int VEC = 16 / sizeof(T);
    for (int t0 = 0; t0 < L; t0 += kBsKT) {
        const int nk = min(kBsKT, L - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < kBsKT * D / VEC; i += blockDim.x) {
            const int row = (i * VEC) / D;
            uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (row < nk) {
                kv = *reinterpret_cast<const uint4 *>(kg + (size_t)t0 * D + (size_t)i * VEC);
                vv = *reinterpret_cast<const uint4 *>(vg + (size_t)t0 * D + (size_t)i * VEC);
            }
            reinterpret_cast<uint4 *>(ks)[i] = kv;
            reinterpret_cast<uint4 *>(vs)[i] = vv;
        }
        __syncthreads();
#pragma unroll 1
        for (int j = 0; j < kBsQPerWarp; ++j) {
            float part[kBsKT];
#pragma unroll
            for (int t = 0; t < kBsKT; ++t) {
                float kf[EPL];
                load_vec<T, EPL>(ks + t * D + lane * EPL, kf);
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc = fmaf(qr[j][e], kf[e], acc);
                part[t] = acc;
            }
            float s = transpose_reduce<kBsKT>(part, lane);  // lane = key
            if (lane >= nk) s = kNegInf;
            const float mnew = fmaxf(m[j], warp_max(s));
            const float alpha = (m[j] == kNegInf) ? 0.f : exp2f(m[j] - mnew);
            const float p = (s == kNegInf) ? 0.f : exp2f(s - mnew);
            l[j] = l[j] * alpha + warp_sum(p);
            m[j] = mnew;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[j][e] *= alpha;
            for (int t = 0; t < nk; ++t) {
                const float pt = __shfl_sync(0xffffffffu, p, t);
                float vf[EPL];
                load_vec<T, EPL>(vs + t * D + lane * EPL, vf);
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[j][e] = fmaf(pt, vf[e], o[j][e]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kBsQPerWarp; ++j) {
        const int n = n0 + j;
        if (n >= N) break;
        const size_t row = (size_t)h * N + n;
        float z = (l[j] > 0.f) ? (m[j] + log2f(l[j])) * kLn2 : kNegInf;
        float res[EPL];
        const float inv = (l[j] > 0.f) ? 1.f / l[j] : 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) res[e] = o[j][e] * inv;
        if (accumulate) {
            float prev[EPL];
            load_vec<T, EPL>(a + row * D + lane * EPL, prev);
            const float zp = logz[row];
            float wa, wb, zz;
            merge_state(zp, z, wa, wb, zz);
#pragma unroll
            for (int e = 0; e < EPL; ++e) res[e] = wa * prev[e] + wb * res[e];
            z = zz;
        }
        store_vec<T, EPL>(a + row * D + lane * EPL, res);
        if (lane == 0) logz[row] = z;
    }
}

}  // namespace asmk


cudaError_t asm_build_states_launch(const void *q, const void *k, const void *v, int Hq, int Hkv,
                                    int N, int L, int d, float scale, asm_dtype dt,
                                    int accumulate, void *a, float *logz, int num_sms,
                                    cudaStream_t st) {
    using namespace asmk;
    (void)num_sms;
    if (dt == ASM_BF16 && d == 128 && L > 0)
        return asm_build_states_tc_launch(q, k, v, Hq, Hkv, N, L, scale, accumulate, a, logz, st);
    dim3 grid((N + kBsQ - 1) / kBsQ, Hq);
    const float qs = scale * kLog2e;
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128)
            build_states_simple<T, 128><<<grid, kBsWarps * 32, 0, st>>>(
                (const T *)q, (const T *)k, (const T *)v, Hq, Hkv, N, L, qs, accumulate, (T *)a, logz);
        else
            build_states_simple<T, 64><<<grid, kBsWarps * 32, 0, st>>>(
                (const T *)q, (const T *)k, (const T *)v, Hq, Hkv, N, L, qs, accumulate, (T *)a, logz);
    } else {
        if (d == 128)
            build_states_simple<float, 128><<<grid, kBsWarps * 32, 0, st>>>(
                (const float *)q, (const float *)k, (const float *)v, Hq, Hkv, N, L, qs, accumulate,
                (float *)a, logz);
        else
            build_states_simple<float, 64><<<grid, kBsWarps * 32, 0, st>>>(
                (const float *)q, (const float *)k, (const float *)v, Hq, Hkv, N, L, qs, accumulate,
                (float *)a, logz);
    }
    return cudaGetLastError();
}
