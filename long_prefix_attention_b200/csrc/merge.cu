// merge.cu -- online-softmax merge of two sets of attention states, row by row.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Eficiencia": a long prefix is encoded chunk by chunk and the chunk states
// are combined with the online-softmax identity.  When the chunks are encoded
// on different GPUs, each GPU holds the states of its chunks; once they are
// gathered, this call folds them in chunk order:
//   z = logaddexp(z, z'),  a = e^(z_old - z) a + e^(z' - z) a'
// (the empty state (0, -inf) is the identity).  HBM-bound: per row, two reads
// of d values, one write, and the two logZ.  A row is D / E lanes of 16-byte
// accesses (E = elements per 16 bytes); each warp takes 32 / (D / E) rows at a
// time, so a row's lanes sit in one warp and its first lane computes the
// weights once and shares them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

template <typename T, int D>
__global__ void __launch_bounds__(256)
merge_states_kernel(T *__restrict__ a, float *__restrict__ z, const T *__restrict__ a2,
                    const float *__restrict__ z2, long long R) {
    constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte access
    constexpr int LPR = D / E;              // lanes per row
    constexpr int RPW = 32 / LPR;           // rows per warp and step
    static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row lanes");
    const int lane = threadIdx.x & 31, c = lane % LPR, lead = lane - c;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long base = warp * RPW; base < R; base += nwarps * RPW) {
        const long long row = base + lane / LPR;
        const bool valid = row < R;
        float wa = 0.f, wb = 0.f, zz = kNegInf;
        if (c == 0 && valid) {
            const float za = z[row], zb = z2[row];
            if (!(za == kNegInf && zb == kNegInf)) {
                const float m = fmaxf(za, zb);
                const float ea = expf(za - m), eb = expf(zb - m), s = ea + eb;
                zz = m + logf(s);
                wa = ea / s;
                wb = eb / s;
            }
        }
        wa = __shfl_sync(0xffffffffu, wa, lead);
        wb = __shfl_sync(0xffffffffu, wb, lead);
        if (valid) {
            T *pa = a + row * D + c * E;
            float x[E], y[E];
            if constexpr (E == 8) {
                load_vec<T, 4>(pa, *reinterpret_cast<float(*)[4]>(x));
                load_vec<T, 4>(pa + 4, *reinterpret_cast<float(*)[4]>(x + 4));
                load_vec<T, 4>(a2 + row * D + c * E, *reinterpret_cast<float(*)[4]>(y));
                load_vec<T, 4>(a2 + row * D + c * E + 4, *reinterpret_cast<float(*)[4]>(y + 4));
            } else {
                load_vec<T, 4>(pa, x);
                load_vec<T, 4>(a2 + row * D + c * E, y);
            }
#pragma unroll
            for (int e = 0; e < E; ++e) x[e] = fmaf(wa, x[e], wb * y[e]);
            if constexpr (E == 8) {
                store_vec<T, 4>(pa, *reinterpret_cast<float(*)[4]>(x));
                store_vec<T, 4>(pa + 4, *reinterpret_cast<float(*)[4]>(x + 4));
            } else {
                store_vec<T, 4>(pa, x);
            }
            if (c == 0) z[row] = zz;
        }
    }
}

template <typename T, int D>
static cudaError_t merge_launch_t(void *a, float *z, const void *a2, const float *z2, long long R, int num_sms,
                                  cudaStream_t st) {
    constexpr int RPW = 32 / (D / (16 / (int)sizeof(T)));
    const long long warps = (R + RPW - 1) / RPW;
    long long blocks = (warps + 7) / 8;
    blocks = blocks < (long long)num_sms * 8 ? blocks : (long long)num_sms * 8;
    if (blocks < 1) return cudaSuccess;
    merge_states_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>((T *)a, z, (const T *)a2, z2, R);
    return cudaGetLastError();
}

}  // namespace asmk

cudaError_t asm_merge_states_launch(void *a, float *z, const void *a2, const float *z2, long long R, int d,
                                    asm_dtype dt, int num_sms, cudaStream_t st) {
    using namespace asmk;
    if (dt == ASM_BF16)
        return d == 128 ? merge_launch_t<__nv_bfloat16, 128>(a, z, a2, z2, R, num_sms, st)
                        : merge_launch_t<__nv_bfloat16, 64>(a, z, a2, z2, R, num_sms, st);
    return d == 128 ? merge_launch_t<float, 128>(a, z, a2, z2, R, num_sms, st)
                    : merge_launch_t<float, 64>(a, z, a2, z2, R, num_sms, st);
}
