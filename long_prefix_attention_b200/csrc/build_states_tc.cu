// build_states_tc.cu -- attention states of the calibration queries on the
// 5th-generation tensor cores (bf16, head dim 128).
//
// "Context Memorization for Efficient Long Context Generation", Metodologia:
// "Recoleccion" (each calibration query's attention state over the prefix)
// and "Eficiencia" (the prefix is encoded in chunks whose states merge by the
// online-softmax identity).  The state of query q over keys K, values V is
//   a = softmax(s q K^T) V,   logZ = ln sum_j exp(s <q, k_j>),
// computed flash-attention style: S = Q K^T and O += P V on tcgen05.mma with
// fp32 accumulators in tensor memory, the softmax in registers.
//
// One CTA owns two 128-query tiles (X = 0, 1) of one query head and sweeps the
// L keys of its KV head in tiles of 64.  Warp roles:
//   warp 0     TMA producer: both Q tiles once, then K and V tiles (128-byte
//              swizzle) through two 3-slot rings;
//   warp 1     allocates 512 TMEM columns; one lane issues the MMAs in the
//              order S_0(j), S_1(j), PV_0(j-1), PV_1(j-1), so that the
//              tensor core multiplies while the softmax warps work;
//   warps 2-5  softmax of tile 0, warps 6-9 softmax of tile 1: one thread
//              per query row (TMEM lane), which reads its 64 scores, forms
//              P = exp2(t - m) in bf16 into one of two shared-memory buffers
//              (so it never waits for the previous P V product unless it
//              has to rescale), and rescales its
//              O row in TMEM on the rare tiles where the running maximum
//              rises by more than 8 (base-2 units; below that the stale
//              maximum is kept, which is exact since numerator and
//              denominator share it).
// TMEM columns: O_0 [0,128) O_1 [128,256) S_0 double buffer [256,384)
// S_1 double buffer [384,512).  Every wait is bounded; a timeout writes NaN
// into logZ of the CTA's rows.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {
namespace stc {

constexpr int kQT = 128;              // queries per tile (MMA M)
constexpr int kKT = 64;               // keys per tile
constexpr int kD = 128;
constexpr int kRing = 3;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescale = 8.f;       // lazy-rescale threshold (base-2 units)

constexpr int kQBox = kQT * 128;      // 128 rows x 64 columns bf16 (16 KB)
constexpr int kKBox = kKT * 128;      // 64 rows x 64 columns bf16 (8 KB)
constexpr int kKVBytes = 2 * kKBox;   // one K or V tile

struct Smem {
    unsigned char q[2][2][kQBox];     // [tile][d-half]
    unsigned char k[kRing][kKVBytes]; // [slot][d-half box]
    unsigned char v[kRing][kKVBytes];
    unsigned char p[2][2][kQBox];     // P [tile][buffer]: 128 rows x 64 keys
    uint64_t q_full, k_full[kRing], k_empty[kRing], v_full[kRing], v_empty[kRing];
    // [tile][buffer]; a barrier per buffer, so no wait can be overtaken by
    // the phase after the one it waits for
    uint64_t s_full[2][2], s_free[2][2], p_full[2][2], pv_done[2][2];
    uint32_t tmem_base;
};

// K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major operand, 128-byte swizzle: 64-element MN blocks `lbo` bytes apart,
// 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Three-input maximum and paired fp32 arithmetic (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
    return v;
}
__device__ __forceinline__ float lo_f32(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo;
}
__device__ __forceinline__ float hi_f32(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return hi;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

struct Maps {
    CUtensorMap q, k, v;
};

// Online-softmax merge of a stored state (za) with a new one (zb), natural log.
__device__ __forceinline__ void merge_weights(float za, float zb, float &wa, float &wb, float &z) {
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

__global__ void __launch_bounds__(kThreads, 1)
states_tc_kernel(const __grid_constant__ Maps maps, int Hq, int Hkv, int N, int L, float sl2, int accumulate,
                 __nv_bfloat16 *__restrict__ a, float *__restrict__ logz) {
    extern __shared__ unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, g = h / (Hq / Hkv);
    const int n0 = blockIdx.x * (2 * kQT);
    const int J = (L + kKT - 1) / kKT;

    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x)
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sm.s_full[x][b], 1);
                mbar_init(&sm.s_free[x][b], kQT);
                mbar_init(&sm.p_full[x][b], kQT);
                mbar_init(&sm.pv_done[x][b], 1);
            }
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&sm.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&sm.q_full, 4 * kQBox);
            for (int x = 0; x < 2; ++x)
                for (int dh = 0; dh < 2; ++dh)
                    tma_load_3d(sm.q[x][dh], &maps.q, dh * 64, n0 + x * kQT, h, &sm.q_full);
            for (int j = 0; j < J; ++j) {
                const int s = j % kRing;
                const uint32_t par = ((j / kRing) - 1) & 1;
                if (j >= kRing) ok &= mbar_wait(&sm.k_empty[s], par);
                mbar_arrive_expect_tx(&sm.k_full[s], kKVBytes);
                tma_load_3d(sm.k[s], &maps.k, 0, j * kKT, g, &sm.k_full[s]);
                tma_load_3d(sm.k[s] + kKBox, &maps.k, 64, j * kKT, g, &sm.k_full[s]);
                if (j >= kRing) ok &= mbar_wait(&sm.v_empty[s], par);
                mbar_arrive_expect_tx(&sm.v_full[s], kKVBytes);
                tma_load_3d(sm.v[s], &maps.v, 0, j * kKT, g, &sm.v_full[s]);
                tma_load_3d(sm.v[s] + kKBox, &maps.v, 64, j * kKT, g, &sm.v_full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer
        if (lane == 0) {
            // S = Q K^T: M = 128, N = 64, both operands K-major
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKT >> 3) << 17) |
                                     ((uint32_t)(kQT >> 4) << 24);
            // O += P V: M = 128, N = 128; P K-major, V MN-major (d contiguous)
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                     ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kQT >> 4) << 24);
            ok &= mbar_wait(&sm.q_full, 0);
            for (int j = 0; j <= J; ++j) {
                if (j < J) {
                    const int s = j % kRing, b = j & 1;
                    ok &= mbar_wait(&sm.k_full[s], (j / kRing) & 1);
                    const uint32_t kb = smem_addr(sm.k[s]);
                    for (int x = 0; x < 2; ++x) {
                        if (j >= 2) ok &= mbar_wait(&sm.s_free[x][b], ((j >> 1) - 1) & 1);
                        tc_fence_after();
                        const uint32_t qb = smem_addr(sm.q[x][0]);
                        const uint32_t td = tmem + 256 + (uint32_t)(x * 128 + b * 64);
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk) {
                            const uint32_t off = (uint32_t)((kk & 3) * 32);
                            umma_bf16(td, desc_k_sw128(qb + (kk >> 2) * kQBox + off),
                                      desc_k_sw128(kb + (kk >> 2) * kKBox + off), idesc_s, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&sm.s_full[x][b]);
                    }
                    umma_commit(&sm.k_empty[s]);
                }
                if (j >= 1) {
                    const int jj = j - 1, s = jj % kRing, pb = jj & 1;
                    ok &= mbar_wait(&sm.v_full[s], (jj / kRing) & 1);
                    const uint32_t vb = smem_addr(sm.v[s]);
                    for (int x = 0; x < 2; ++x) {
                        ok &= mbar_wait(&sm.p_full[x][pb], (jj >> 1) & 1);
                        tc_fence_after();
                        const uint32_t pa = smem_addr(sm.p[x][pb]);
#pragma unroll
                        for (int kk = 0; kk < kKT / 16; ++kk) {
                            // 16 keys per step: +32 bytes along P's rows, +2 K-groups of V
                            umma_bf16(tmem + (uint32_t)(x * 128), desc_k_sw128(pa + kk * 32),
                                      desc_mn_sw128(vb + kk * 2048, kKBox), idesc_o,
                                      (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&sm.pv_done[x][pb]);
                    }
                    umma_commit(&sm.v_empty[s]);
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- softmax
        const int x = (warp - 2) >> 2;      // query tile
        const int qd = warp & 3;            // TMEM lane quarter
        const int row = qd * 32 + lane;     // row within the tile
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const uint32_t t_o = tmem + lane_off + (uint32_t)(x * 128);
        float m_used = kNegInf, l = 0.f;
        for (int j = 0; j < J; ++j) {
            const int b = j & 1;
            ok &= mbar_wait(&sm.s_full[x][b], (j >> 1) & 1);
            tc_fence_after();
            uint32_t r[64];
            const uint32_t t_s = tmem + lane_off + 256 + (uint32_t)(x * 128 + b * 64);
            tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.s_free[x][b]);

            const int valid = L - j * kKT;  // keys of this tile inside the block
            if (valid < kKT) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c >= valid) r[c] = 0xff800000u;  // -inf
            }
            // row maximum of the raw scores (the scale is positive)
            float m21[22];
#pragma unroll
            for (int i = 0; i < 21; ++i)
                m21[i] = max3f(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
            m21[21] = __uint_as_float(r[63]);
            float m7[8];
#pragma unroll
            for (int i = 0; i < 7; ++i) m7[i] = max3f(m21[3 * i], m21[3 * i + 1], m21[3 * i + 2]);
            m7[7] = m21[21];
            const float mt = max3f(max3f(m7[0], m7[1], m7[2]), max3f(m7[3], m7[4], m7[5]), fmaxf(m7[6], m7[7])) * sl2;
            bool rescale = false;
            float alpha = 1.f;
            if (mt > m_used + kRescale) {
                alpha = (m_used == kNegInf) ? 0.f : ex2f(m_used - mt);
                rescale = j > 0;
                m_used = mt;
                l *= alpha;
            }
            // p = 2^(s * scale * log2(e) - m), paired fp32 arithmetic
            const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
            const uint64_t negm2 = pack_f32x2(-m_used, -m_used);
            uint32_t pk[32];
            uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const uint64_t t2 = fma_f32x2(pack_u32x2(r[2 * c], r[2 * c + 1]), sl2x2, negm2);
                const float p0 = ex2f(lo_f32(t2)), p1 = ex2f(hi_f32(t2));
                acc[c & 3] = add_f32x2(acc[c & 3], pack_f32x2(p0, p1));
                pk[c] = pack_bf16(p0, p1);
            }
            const uint64_t a01 = add_f32x2(add_f32x2(acc[0], acc[1]), add_f32x2(acc[2], acc[3]));
            l += lo_f32(a01) + hi_f32(a01);
            // TMEM loads and stores are warp-collective: the warp rescales
            // together, rows that keep their maximum by a factor of 1; O
            // must hold PV(j-1) first
            if (__any_sync(0xffffffffu, rescale)) {
                ok &= mbar_wait(&sm.pv_done[x][(j - 1) & 1], ((j - 1) >> 1) & 1);
                tc_fence_after();
                const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c0 = 0; c0 < kD; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(t_o + (uint32_t)c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(t_o + (uint32_t)c0, o);
                }
                tmem_wait_st();
            }
            // P buffer b is free once PV(j-2) has finished
            if (j >= 2) ok &= mbar_wait(&sm.pv_done[x][b], ((j >> 1) - 1) & 1);
            const uint32_t p_row = smem_addr(sm.p[x][b]) + (uint32_t)row * 128;
            // row of P: eight 16-byte chunks, 128-byte swizzle
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_v4(p_row + (uint32_t)((c ^ (row & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                             pk[4 * c + 3]);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.p_full[x][b]);
        }
        // ------------------------------------------------------ epilogue
        ok &= mbar_wait(&sm.pv_done[x][(J - 1) & 1], ((J - 1) >> 1) & 1);
        tc_fence_after();
        const int n = n0 + x * kQT + row;
        const bool live = n < N;
        const size_t grow = (size_t)h * N + (size_t)(live ? n : 0);
        float z = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : kNegInf;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        float wa = 0.f, wb = 1.f;
        if (accumulate && live) {
            float zz;
            merge_weights(logz[grow], z, wa, wb, zz);
            z = zz;
        }
        __nv_bfloat16 *arow = a + grow * kD;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(t_o + (uint32_t)c0, o);
            tmem_wait_ld();
            if (live) {
                float prev[32];
                if (accumulate) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(arow + c0 + i);
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            prev[i + 2 * e] = __uint_as_float(w[e] << 16);
                            prev[i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                        }
                    }
                }
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float v0 = __uint_as_float(o[i]) * inv, v1 = __uint_as_float(o[i + 1]) * inv;
                    if (accumulate) {
                        v0 = wa * prev[i] + wb * v0;
                        v1 = wa * prev[i + 1] + wb * v1;
                    }
                    packed[i / 2] = pack_bf16(v0, v1);
                }
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<uint4 *>(arow + c0 + 2 * i) =
                        make_uint4(packed[i], packed[i + 1], packed[i + 2], packed[i + 3]);
            }
        }
        if (live) logz[grow] = ok ? z : __int_as_float(0x7fc00000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace stc

bool make_map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows);

}  // namespace asmk

cudaError_t asm_build_states_tc_launch(const void *q, const void *k, const void *v, int Hq, int Hkv, int N, int L,
                                       float scale, int accumulate, void *a, float *logz, cudaStream_t st) {
    using namespace asmk;
    stc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!make_map_3d(&maps.q, q, stc::kD, N, Hq, stc::kQT) || !make_map_3d(&maps.k, k, stc::kD, L, Hkv, stc::kKT) ||
        !make_map_3d(&maps.v, v, stc::kD, L, Hkv, stc::kKT))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(stc::Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(stc::states_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((N + 2 * stc::kQT - 1) / (2 * stc::kQT), Hq);
    stc::states_tc_kernel<<<grid, stc::kThreads, smem, st>>>(maps, Hq, Hkv, N, L, scale * kLog2e, accumulate,
                                                             static_cast<__nv_bfloat16 *>(a), logz);
    return cudaGetLastError();
}
