// common.cuh -- device helpers shared by the ASM kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "asm.h"

namespace asmk {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -__builtin_huge_valf();

// Bounded spins: a wait that has not completed after this many polls gives
// up and raises ASM_ERR_TIMEOUT in the caller's error word.  A poll of an
// mbarrier that does not complete suspends the thread for about 4 us on
// this part (measured by the timeout self-test), so the bound is about one
// second, thousands of times any wait of a working kernel.
constexpr uint32_t kSpinLimit = 1u << 18;

// ---------------------------------------------------------------- dtypes --

template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static float to_f(float x) { return x; }
    __device__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load / store N consecutive elements of T (N * sizeof(T) in {4, 8, 16}
// bytes, naturally aligned) as fp32.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T *p, float (&out)[N]) {
    if constexpr (sizeof(T) == 4) {
        static_assert(N == 2 || N == 4, "fp32 vector");
        if constexpr (N == 4) {
            float4 v = *reinterpret_cast<const float4 *>(p);
            out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
        } else {
            float2 v = *reinterpret_cast<const float2 *>(p);
            out[0] = v.x; out[1] = v.y;
        }
    } else {
        static_assert(N == 2 || N == 4, "bf16 vector");
        if constexpr (N == 4) {
            uint2 v = *reinterpret_cast<const uint2 *>(p);
            __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&v.x);
            __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v.y);
            float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
            out[0] = fa.x; out[1] = fa.y; out[2] = fb.x; out[3] = fb.y;
        } else {
            uint32_t v = *reinterpret_cast<const uint32_t *>(p);
            __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&v);
            float2 fa = __bfloat1622float2(a);
            out[0] = fa.x; out[1] = fa.y;
        }
    }
}

template <typename T, int N>
__device__ __forceinline__ void store_vec(T *p, const float (&in)[N]) {
    if constexpr (sizeof(T) == 4) {
        if constexpr (N == 4) {
            *reinterpret_cast<float4 *>(p) = make_float4(in[0], in[1], in[2], in[3]);
        } else {
            *reinterpret_cast<float2 *>(p) = make_float2(in[0], in[1]);
        }
    } else {
        if constexpr (N == 4) {
            __nv_bfloat162 a = __floats2bfloat162_rn(in[0], in[1]);
            __nv_bfloat162 b = __floats2bfloat162_rn(in[2], in[3]);
            uint2 v;
            v.x = *reinterpret_cast<uint32_t *>(&a);
            v.y = *reinterpret_cast<uint32_t *>(&b);
            *reinterpret_cast<uint2 *>(p) = v;
        } else {
            __nv_bfloat162 a = __floats2bfloat162_rn(in[0], in[1]);
            *reinterpret_cast<__nv_bfloat162 *>(p) = a;
        }
    }
}

// ------------------------------------------------------------- reductions --

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
    return v;
}

// Reduce NV per-lane partial sums across the warp so that every lane ends up
// holding one full sum: lane l holds the total of value index l / (32 / NV).
// NV must be a power of two <= 32.  Uses (NV - 1) + log2(32 / NV) shuffles.
template <int NV>
__device__ __forceinline__ float transpose_reduce(float (&v)[NV], int lane) {
    static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "NV");
    int mask = 16;
#pragma unroll
    for (int n = NV; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            float send = up ? v[i] : v[i + half];
            float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
        mask >>= 1;
    }
    float r = v[0];
    for (; mask >= 1; mask >>= 1) r += __shfl_xor_sync(0xffffffffu, r, mask);
    return r;
}

// Arg-max over lanes: larger score wins, ties go to the smaller index.
__device__ __forceinline__ bool better(float s, int i, float bs, int bi) {
    return s > bs || (s == bs && (unsigned)i < (unsigned)bi);
}
__device__ __forceinline__ void warp_argmax(float &s, int &i) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        float os = __shfl_xor_sync(0xffffffffu, s, m);
        int oi = __shfl_xor_sync(0xffffffffu, i, m);
        if (better(os, oi, s, i)) { s = os; i = oi; }
    }
}

// ------------------------------------------------- mbarrier / bulk copies --

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase; returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 1-D bulk copy global -> shared, completing `bytes` on `bar`.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

// Hardware base-2 exponential and logarithm (approximate, flush-to-zero;
// relative error about 2^-22): single instructions, used where code size and
// latency matter more than the last bits (softmax weights, merge weights).
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2f(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float ld_cg(const float *p) { return __ldcg(p); }
__device__ __forceinline__ int ld_cg(const int *p) { return __ldcg(p); }

}  // namespace asmk

// ------------------------------------------- warp-level tensor-core MMA ----
namespace asmk {

// D += A * B for one m16n8k16 tile, bf16 inputs, fp32 accumulation.  It
// reads and writes registers only, so the compiler may interleave
// independent accumulation chains.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of the 16-byte chunk `c` (0..7) of row `r` in a tile written by
// a TMA load with 128-byte swizzling (rows of 128 bytes, 1024-byte aligned).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// 3-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int c0, int c1, int c2,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4}], [%5];"
        ::"r"(smem_addr(dst)), "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

// 4-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4, %5}], [%6];"
        ::"r"(smem_addr(dst)), "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
        : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's memory, and
// let the next grid in the stream begin launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace asmk
