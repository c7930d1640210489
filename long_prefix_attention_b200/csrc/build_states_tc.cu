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
// One CTA owns two 128-query tiles (x = 0, 1) of one query head and sweeps the
// L keys of its KV head in tiles of 128.  Warp roles:
//   warp 0     TMA producer: both Q tiles once, then K_0, V_0, K_1, V_1, ...
//              (128-byte swizzle) through a 4-slot ring;
//   warp 1     allocates 512 TMEM columns; one lane issues the MMAs in the
//              order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while one tile's
//              softmax works, the tensor core multiplies the other tile;
//   warps 2-5  softmax of tile 0, warps 6-9 softmax of tile 1: one thread
//              per query row (TMEM lane).  It loads its 128 scores, forms
//              P = exp2(t - m) (three quarters on the MUFU unit, one quarter
//              by a cubic on the FMA pipe) and stores P as bf16 over the
//              first 64 columns of its own S region, from where the P V
//              product reads it as the A operand; only V comes from shared
//              memory.  Its O row is rescaled in TMEM on the rare tiles where
//              the running maximum rises by more than 8 (base-2 units; below
//              that the stale maximum is kept, which is exact since
//              numerator and denominator share it).
// The tensor pipe completes MMAs in issue order, so S_x(j+1) (issued after
// PV_x(j)) overwrites P_x(j) only after it was read, and the completion of
// S_x(j) also means PV_x(j-1) is done: O_x is stable when softmax x starts.
// TMEM columns: O_0 [0,128) O_1 [128,256) S_0 / P_0 [256,384) S_1 / P_1 [384,512).
// Every wait is bounded; a timeout writes NaN into logZ of the CTA's rows.
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
constexpr int kKT = 128;              // keys per tile (MMA N of S = Q K^T)
constexpr int kD = 128;
constexpr int kRing = 4;              // K/V slots
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescale = 8.f;       // lazy-rescale threshold (base-2 units)

constexpr int kBox = 128 * 128;       // 128 rows x 64 columns bf16 (16 KB)
constexpr int kTile = 2 * kBox;       // a 128 x 128 bf16 tile as two 64-column boxes

struct Smem {
    unsigned char q[2][kTile];        // [query tile]: d-halves
    unsigned char kv[kRing][kTile];   // K or V tile: d-halves, rows = keys
    uint64_t q_full, kv_full[kRing], kv_empty[kRing];
    uint64_t s_full[2], p_full[2], o_full[2];
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
// D[tmem] (+)= A[tmem] * B^T: A (M x 16, bf16 pairs per column) from tensor memory
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

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
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


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
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
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

// 2^t for two arguments on the FMA pipe: t = n + f with n = round(t),
// f in [-1/2, 1/2]; 2^f by a cubic fitted to 2^f over that interval
// (relative error below 7.5e-5, under a quarter of a bf16 half-unit), and
// 2^n added into the exponent field.  t is clamped at -125 (2^-125 counts as
// 0 next to the row maximum's 2^0).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t t2) {
    const float t0 = fmaxf(lo_f32(t2), -125.f), t1 = fmaxf(hi_f32(t2), -125.f);
    const uint64_t t = pack_f32x2(t0, t1);
    const uint64_t y = add_f32x2(t, pack_f32x2(12582912.f, 12582912.f));   // 1.5 * 2^23: n in the low bits
    const uint64_t n = add_f32x2(y, pack_f32x2(-12582912.f, -12582912.f));
    const uint64_t f = fma_f32x2(n, pack_f32x2(-1.f, -1.f), t);
    uint64_t p = fma_f32x2(pack_f32x2(0.0551716685f, 0.0551716685f), f, pack_f32x2(0.2426111251f, 0.2426111251f));
    p = fma_f32x2(p, f, pack_f32x2(0.6932609678f, 0.6932609678f));
    p = fma_f32x2(p, f, pack_f32x2(0.9999280572f, 0.9999280572f));
    const uint32_t lo = (uint32_t)p + ((uint32_t)y << 23), hi = (uint32_t)(p >> 32) + ((uint32_t)(y >> 32) << 23);
    return pack_u32x2(lo, hi);
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

struct Params {
    int Hq, Hkv, N, L;            // states: queries [Hq][N][d], keys [Hkv][L][d]
    float sl2;                    // softmax scale * log2(e)
    int accumulate;
    __nv_bfloat16 *a;             // states: [Hq][N][d]
    float *logz;                  // states: [Hq][N]
    // decode partials: the (row b, head) pairs of KV group blockIdx.y against
    // prefix chunk blockIdx.z (keys [z * chunk, z * chunk + chunk) of L)
    int B, G, chunk, nslots;
    float2 *ws_ml;                // [B][Hq][nslots] (m in base 2, l)
    float *ws_o;                  // [B][Hq][nslots][d]
};

// MODE 0: prefix states of calibration queries (a, logZ), with the chunk merge.
// MODE 1: decode partials of a shared prefix chunk for the batch's query rows:
//         (m = log2 of the chunk's Z, l = 1, o = a), the form the decode merge reads.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
states_tc_kernel(const __grid_constant__ Maps maps, const Params p) {
    extern __shared__ unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hq = p.Hq, N = p.N, accumulate = p.accumulate;
    const float sl2 = p.sl2;
    const int h = blockIdx.y;
    const int g = MODE == 0 ? h / (Hq / p.Hkv) : blockIdx.y;
    const int n0 = blockIdx.x * (2 * kQT);
    const int k0 = MODE == 0 ? 0 : blockIdx.z * p.chunk;                // first key of this CTA
    const int L = MODE == 0 ? p.L : min(p.chunk, p.L - k0);             // keys of this CTA
    const int J = (L + kKT - 1) / kKT;

    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&sm.kv_full[i], 1);
            mbar_init(&sm.kv_empty[i], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sm.s_full[x], 1);
            mbar_init(&sm.p_full[x], kQT);
            mbar_init(&sm.o_full[x], 1);
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
            mbar_arrive_expect_tx(&sm.q_full, 2 * kTile);
            for (int x = 0; x < 2; ++x)
                for (int dh = 0; dh < 2; ++dh) {
                    if (MODE == 0)
                        tma_load_3d(sm.q[x] + dh * kBox, &maps.q, dh * 64, n0 + x * kQT, h, &sm.q_full);
                    else  // 128 (row, head) pairs of group g: rows (n0 + x * kQT) / G ..
                        tma_load_4d(sm.q[x] + dh * kBox, &maps.q, dh * 64, 0, g, (n0 + x * kQT) / p.G,
                                    &sm.q_full);
                }
            // ring item n: K_{n/2} for even n, V_{n/2} for odd n
            for (int n = 0; n < 2 * J; ++n) {
                const int slot = n % kRing;
                if (n >= kRing) ok &= mbar_wait(&sm.kv_empty[slot], ((n / kRing) - 1) & 1);
                mbar_arrive_expect_tx(&sm.kv_full[slot], kTile);
                const CUtensorMap *mp = (n & 1) ? &maps.v : &maps.k;
                tma_load_3d(sm.kv[slot], mp, 0, k0 + (n >> 1) * kKT, g, &sm.kv_full[slot]);
                tma_load_3d(sm.kv[slot] + kBox, mp, 64, k0 + (n >> 1) * kKT, g, &sm.kv_full[slot]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer
        if (lane == 0) {
            // S = Q K^T: M = 128, N = 128, both operands K-major (shared memory)
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKT >> 3) << 17) |
                                     ((uint32_t)(kQT >> 4) << 24);
            // O += P V: M = 128, N = 128; P K-major in TMEM, V MN-major (d contiguous)
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                     ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kQT >> 4) << 24);
            auto issue_s = [&](int x, uint32_t kb) {
                const uint32_t qb = smem_addr(sm.q[x]);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * kBox + (kk & 3) * 32);
                    umma_bf16(tmem + 256 + (uint32_t)(x * 128), desc_k_sw128(qb + off), desc_k_sw128(kb + off),
                              idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sm.s_full[x]);
            };
            auto issue_pv = [&](int x, uint32_t vb, int j) {
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    // 16 keys per step: 8 TMEM columns of P, 16 rows (2 K-groups) of V
                    umma_bf16_ts(tmem + (uint32_t)(x * 128), tmem + 256 + (uint32_t)(x * 128 + kk * 8),
                                 desc_mn_sw128(vb + (uint32_t)(kk * 2048), kBox), idesc_o,
                                 (j > 0 || kk > 0) ? 1u : 0u);
            };
            ok &= mbar_wait(&sm.q_full, 0);
            // scores of key tile 0
            ok &= mbar_wait(&sm.kv_full[0], 0);
            tc_fence_after();
            issue_s(0, smem_addr(sm.kv[0]));
            issue_s(1, smem_addr(sm.kv[0]));
            umma_commit(&sm.kv_empty[0]);
            for (int j = 0; j < J; ++j) {
                const int nv = 2 * j + 1, nk = 2 * j + 2;          // ring items V_j and K_{j+1}
                const int sv = nv % kRing, sk = nk % kRing;
                const bool more = j + 1 < J;
                ok &= mbar_wait(&sm.kv_full[sv], (nv / kRing) & 1);
                const uint32_t vb = smem_addr(sm.kv[sv]), kb = smem_addr(sm.kv[sk]);
                for (int x = 0; x < 2; ++x) {
                    ok &= mbar_wait(&sm.p_full[x], j & 1);
                    tc_fence_after();
                    issue_pv(x, vb, j);
                    if (more) {
                        if (x == 0) ok &= mbar_wait(&sm.kv_full[sk], (nk / kRing) & 1);
                        issue_s(x, kb);
                    } else {
                        umma_commit(&sm.o_full[x]);
                    }
                }
                umma_commit(&sm.kv_empty[sv]);
                if (more) umma_commit(&sm.kv_empty[sk]);
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
        const uint32_t t_s = tmem + lane_off + 256 + (uint32_t)(x * 128);
        float m_used = kNegInf, l = 0.f;
        for (int j = 0; j < J; ++j) {
            // S_x(j) done, and with it PV_x(j-1): O_x is stable, P_x's columns free
            ok &= mbar_wait(&sm.s_full[x], j & 1);
            tc_fence_after();
            const int valid = L - j * kKT;  // keys of this tile inside the block
            // pass 1: row maximum of the raw scores (the scale is positive),
            // 32 columns at a time
            float mraw = kNegInf;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(t_s + (uint32_t)(32 * c), r);
                tmem_wait_ld();
                if (valid < kKT) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i >= valid) r[i] = 0xff800000u;  // -inf
                }
                float m11[11];
#pragma unroll
                for (int i = 0; i < 10; ++i)
                    m11[i] = max3f(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
                m11[10] = fmaxf(__uint_as_float(r[30]), __uint_as_float(r[31]));
                mraw = max3f(mraw, max3f(max3f(m11[0], m11[1], m11[2]), max3f(m11[3], m11[4], m11[5]),
                                         max3f(m11[6], m11[7], m11[8])), fmaxf(m11[9], m11[10]));
            }
            const float mt = mraw * sl2;
            bool rescale = false;
            float alpha = 1.f;
            if (mt > m_used + kRescale) {
                alpha = (m_used == kNegInf) ? 0.f : ex2f(m_used - mt);
                rescale = j > 0;
                m_used = mt;
                l *= alpha;
            }
            // TMEM loads and stores are warp-collective: the warp rescales
            // together, rows that keep their maximum by a factor of 1
            if (__any_sync(0xffffffffu, rescale)) {
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
            }
            // pass 2: p = 2^(s * scale * log2(e) - m), packed to bf16 pairs;
            // chunk c's 16 columns of P land on S columns already read
            const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
            const uint64_t negm2 = pack_f32x2(-m_used, -m_used);
            uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(t_s + (uint32_t)(32 * c), r);
                tmem_wait_ld();
                if (valid < kKT) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i >= valid) r[i] = 0xff800000u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t t2 = fma_f32x2(pack_u32x2(r[2 * i], r[2 * i + 1]), sl2x2, negm2);
                    uint64_t p2;
                    if ((i & 3) == 3) {
                        p2 = exp2_poly_x2(t2);
                    } else {
                        p2 = pack_f32x2(ex2f(lo_f32(t2)), ex2f(hi_f32(t2)));
                    }
                    acc[i & 3] = add_f32x2(acc[i & 3], p2);
                    pk[i] = pack_bf16(lo_f32(p2), hi_f32(p2));
                }
                tmem_st16(t_s + (uint32_t)(16 * c), pk);
            }
            const uint64_t a01 = add_f32x2(add_f32x2(acc[0], acc[1]), add_f32x2(acc[2], acc[3]));
            l += lo_f32(a01) + hi_f32(a01);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[x]);
        }
        // ------------------------------------------------------ epilogue
        ok &= mbar_wait(&sm.o_full[x], 0);
        tc_fence_after();
        if (MODE == 1) {
            // row -> (batch row b, head g * G + hh); rows past the batch are padding
            const int r = n0 + x * kQT + row;
            const int b = r / p.G, hh = r - b * p.G;
            const bool live = b < p.B;
            const size_t bh = (size_t)b * Hq + (size_t)g * p.G + hh;
            const size_t slot = (size_t)blockIdx.z;
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            float *orow = p.ws_o + ((live ? bh : 0) * p.nslots + slot) * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(t_o + (uint32_t)c0, o);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(orow + c0 + i) =
                            make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                        __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                }
            }
            if (live)
                p.ws_ml[bh * p.nslots + slot] = (l > 0.f && ok) ? make_float2(m_used + log2f(l), 1.f)
                                                                : make_float2(ok ? kNegInf : __int_as_float(0x7fc00000), 0.f);
        } else {
        const int n = n0 + x * kQT + row;
        const bool live = n < N;
        const size_t grow = (size_t)h * N + (size_t)(live ? n : 0);
        float z = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : kNegInf;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        float wa = 0.f, wb = 1.f;
        if (accumulate && live) {
            float zz;
            merge_weights(p.logz[grow], z, wa, wb, zz);
            z = zz;
        }
        __nv_bfloat16 *arow = p.a + grow * kD;
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
        if (live) p.logz[grow] = ok ? z : __int_as_float(0x7fc00000);
        }
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
bool make_map_qgroups(CUtensorMap *m, const void *q, int B, int Hkv, int G, int d);

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
    cudaError_t e = cudaFuncSetAttribute(stc::states_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    stc::Params p{};
    p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.L = L;
    p.sl2 = scale * kLog2e;
    p.accumulate = accumulate;
    p.a = static_cast<__nv_bfloat16 *>(a);
    p.logz = logz;
    dim3 grid((N + 2 * stc::kQT - 1) / (2 * stc::kQT), Hq);
    stc::states_tc_kernel<0><<<grid, stc::kThreads, smem, st>>>(maps, p);
    return cudaGetLastError();
}

// Decode partials of a shared explicit prefix for all B rows of a batch:
// grid (row tiles, Hkv, chunks); partial slot z of pair (b, h) covers keys
// [z * chunk, z * chunk + chunk).  q [B][Hq][128] bf16, prefix [Hkv][Lp][128].
cudaError_t asm_prefix_partials_tc_launch(const void *q, const void *k_prefix, const void *v_prefix, int B, int Hq,
                                          int Hkv, int Lp, int chunk, float scale, float2 *ws_ml, float *ws_o,
                                          int nslots, cudaStream_t st) {
    using namespace asmk;
    const int G = Hq / Hkv;
    stc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!make_map_qgroups(&maps.q, q, B, Hkv, G, stc::kD) ||
        !make_map_3d(&maps.k, k_prefix, stc::kD, Lp, Hkv, stc::kKT) ||
        !make_map_3d(&maps.v, v_prefix, stc::kD, Lp, Hkv, stc::kKT))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(stc::Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(stc::states_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    stc::Params p{};
    p.Hq = Hq; p.Hkv = Hkv; p.N = B * G; p.L = Lp;
    p.sl2 = scale * kLog2e;
    p.B = B; p.G = G; p.chunk = chunk; p.nslots = nslots;
    p.ws_ml = ws_ml;
    p.ws_o = ws_o;
    dim3 grid((B * G + 2 * stc::kQT - 1) / (2 * stc::kQT), Hkv, (Lp + chunk - 1) / chunk);
    stc::states_tc_kernel<1><<<grid, stc::kThreads, smem, st>>>(maps, p);
    return cudaGetLastError();
}
