// assign_tc.cu -- k-means assignment on the 5th-generation tensor cores.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Agrupamiento": each calibration query joins its nearest centroid.  The L2
// arg-min over centroids is the arg-max of <x, c> - |c|^2 / 2 (cosine: the
// arg-max of <x, c> / |c|), so the work is a dense X C^T contraction (bf16
// in, fp32 accumulate) followed by a row-wise arg-max with a per-column term.
// For L2 the term rides on the contraction: a ninth K=16 step multiplies a
// constant tile of ones by three bf16 parts of -|c|^2 / 2 per centre (their
// sum is the fp32 value to within 2^-24 of it), so the accumulator already
// holds <x, c> - |c|^2 / 2 and the epilogue is the arg-max alone (with the
// term applied by the CUDA cores the epilogue, not the MMA, set the pace).
//
// One CTA owns 256 points of one head (two M=128 halves that share every
// centroid tile, which halves the L2 -> shared traffic per flop) and sweeps
// all K centroids in tiles of 128.  Warp roles:
//   warp 0     producer: TMA of the 256x128 point tile once, then the 128x128
//              centroid tiles (128-byte swizzle, 4 stages) with, for L2, the
//              128x16 tile of bias parts (32-byte swizzle); for cosine its
//              lanes copy the tile's |c| into a 4-deep shared ring;
//   warp 1     allocates 512 TMEM columns and one lane issues tcgen05.mma
//              (M=128, N=128, K=16 x 8 (+1 for L2), both halves) into two
//              ping-pong accumulator pairs, committing to mbarriers;
//   warps 2-9  epilogue: warp w reads TMEM lane quarter w%4 of one half,
//              (cosine: divides by |c|) and keeps a running arg-max (ties go
//              to the smaller index) while the next tile is multiplied.
// Every wait is bounded; a timeout sets the workspace error word to 5.
//
// The same contraction, against the few centres of one round, drives the
// fused round of batched k-means++ seeding further down (bseed_round_tc):
// nearest centre, screened exact D2 update and range sums in one pass.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace asmk {
namespace atc {

constexpr int kMH = 128;         // rows per MMA (one half)
constexpr int kM = 2 * kMH;      // points per CTA
constexpr int kN = 128;          // centroids per tile (MMA N)
constexpr int kD = 128;          // head dim (MMA K = 8 x 16)
constexpr int kStages = 4;
constexpr int kBias = 4;         // depth of the per-column term ring
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 512;   // 2 buffers x 2 halves x 128 fp32 columns

constexpr int kSub = 128 * 128;       // one 128-row x 64-column swizzled box (16 KB)
constexpr int kABytes = 4 * kSub;     // [half][k-half]
constexpr int kBBytes = 2 * kSub;     // [k-half]
constexpr int kEBytes = 128 * 32;     // 128 rows x 16 columns, 32-byte swizzle (the bias step)

struct Smem {
    unsigned char a[kABytes];
    unsigned char b[kStages][kBBytes];
    unsigned char be[kStages][kEBytes];  // bias parts of the centroid tile (L2)
    unsigned char ae[kEBytes];           // the ones they multiply (L2)
    float bias[kBias][kN];
    uint64_t a_full, b_full[kStages], b_empty[kStages], acc_full[2], acc_empty[2];
    uint64_t bias_full[kBias], bias_empty[kBias];
    uint32_t tmem_base;
};

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes in 8-row groups 1024 bytes apart; Blackwell descriptor version 1.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// The same for 32-byte rows (K = 16 bf16) with the 32-byte swizzle: 8-row
// groups 256 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw32(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(256 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}

// D[tmem] (+)= A * B^T, bf16 operands from shared memory, fp32 accumulator
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (no wait)
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
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct Maps {
    CUtensorMap x, c, e;
};

// Three-input maximum (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

// Fold 32 accumulator columns (global centre indices col0 ..) into the
// running arg-max; only the first `nv` of them are real centres (FULL: all).
// L2: the accumulator is the score; cosine: divided by |c| from `bias`.
template <int METRIC, bool FULL>
__device__ __forceinline__ void fold32(const uint32_t (&r)[32], const float *bias, int col0, int nv,
                                       float &best, int &bidx) {
    float v[32];
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
        if (METRIC == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u) v[k + u] = __uint_as_float(r[k + u]);
        } else {
            const float4 bn = *reinterpret_cast<const float4 *>(bias + k);
            const float bb[4] = {bn.x, bn.y, bn.z, bn.w};   // the term holds |c|
#pragma unroll
            for (int u = 0; u < 4; ++u) v[k + u] = bb[u] > 0.f ? __uint_as_float(r[k + u]) / bb[u] : 0.f;
        }
    }
    if (!FULL) {
#pragma unroll
        for (int k = 0; k < 32; ++k)
            if (k >= nv) v[k] = kNegInf;
    }
    float m11[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) m11[i] = max3f(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    m11[10] = fmaxf(v[30], v[31]);
    const float cm = max3f(max3f(m11[0], m11[1], m11[2]), max3f(m11[3], m11[4], m11[5]),
                           max3f(max3f(m11[6], m11[7], m11[8]), m11[9], m11[10]));
    if (cm > best) {
        int first = 31;
#pragma unroll
        for (int k = 31; k >= 0; --k)
            if (v[k] == cm) first = k;
        best = cm;
        bidx = col0 + first;
    }
}

template <int METRIC>
__global__ void __launch_bounds__(kThreads, 1)
assign_tc_kernel(const __grid_constant__ Maps maps, const float *__restrict__ norms, int N, int K,
                 int32_t *__restrict__ assign, int *err) {
    extern __shared__ unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int p0 = blockIdx.x * kM;
    const int ntiles = (K + kN - 1) / kN;

    if (tid == 0) {
        mbar_init(&sm.a_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.b_full[s], 1);
            mbar_init(&sm.b_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], kEpiWarps);
        }
        for (int s = 0; s < kBias; ++s) {
            mbar_init(&sm.bias_full[s], 32);
            mbar_init(&sm.bias_empty[s], kEpiWarps);
        }
        fence_mbar_init();
    }
    if (METRIC == 0) {
        // the ones of the bias step: columns 0-2 of each 16-byte half of every
        // 32-byte row (both halves alike, so the swizzle leaves them in place);
        // the tensor cores read them through the async proxy
        for (int i = tid; i < kEBytes / 16; i += kThreads) {
            const uint32_t one = 0x3F80u;  // bf16 1.0
            reinterpret_cast<uint4 *>(sm.ae)[i] = make_uint4(one | (one << 16), one, 0u, 0u);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
            mbar_arrive_expect_tx(&sm.a_full, kABytes);
            for (int m = 0; m < 2; ++m)
                for (int kh = 0; kh < 2; ++kh)
                    tma_load_3d(sm.a + (m * 2 + kh) * kSub, &maps.x, kh * 64, p0 + m * kMH, h, &sm.a_full);
        }
        const float *nh = norms + (size_t)h * K;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % kStages, r = t % kBias;
            if (lane == 0) {
                if (t >= kStages) ok &= mbar_wait(&sm.b_empty[s], ((t / kStages) - 1) & 1);
                mbar_arrive_expect_tx(&sm.b_full[s], kBBytes + (METRIC == 0 ? kEBytes : 0));
                tma_load_3d(sm.b[s], &maps.c, 0, t * kN, h, &sm.b_full[s]);
                tma_load_3d(sm.b[s] + kSub, &maps.c, 64, t * kN, h, &sm.b_full[s]);
                if (METRIC == 0) tma_load_3d(sm.be[s], &maps.e, 0, t * kN, h, &sm.b_full[s]);
            }
            if (METRIC == 0) continue;
            if (t >= kBias) ok &= mbar_wait(&sm.bias_empty[r], ((t / kBias) - 1) & 1);
#pragma unroll
            for (int u = 0; u < kN / 32; ++u) {
                const int col = t * kN + u * 32 + lane;
                float nr = col < K ? __ldg(nh + col) : 0.f;
                if (METRIC == 1) nr = sqrtf(nr);
                sm.bias[r][u * 32 + lane] = nr;
            }
            mbar_arrive(&sm.bias_full[r]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer
        if (lane == 0) {
            // kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B,
            // both K-major, N = 128, M = 128
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                                   ((uint32_t)(kMH >> 4) << 24);
            ok &= mbar_wait(&sm.a_full, 0);
            const uint32_t a_base = smem_addr(sm.a);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStages, b = t & 1;
                ok &= mbar_wait(&sm.b_full[s], (t / kStages) & 1);
                if (t >= 2) ok &= mbar_wait(&sm.acc_empty[b], ((t >> 1) - 1) & 1);
                tc_fence_after();
                const uint32_t b_base = smem_addr(sm.b[s]);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
#pragma unroll
                    for (int j = 0; j < kD / 16; ++j) {
                        // k-step j: box j/4, +32 bytes per 16 elements inside the 128-byte row
                        const uint32_t koff = (uint32_t)((j >> 2) * kSub + (j & 3) * 32);
                        const uint64_t ad = sdesc_sw128(a_base + (uint32_t)(m * 2 * kSub) + koff);
                        const uint64_t bd = sdesc_sw128(b_base + koff);
                        umma_bf16(tmem + (uint32_t)((b * 2 + m) * kN), ad, bd, idesc, j > 0 ? 1u : 0u);
                    }
                    if (METRIC == 0)  // + 1 x (-|c|^2 / 2), in three bf16 parts
                        umma_bf16(tmem + (uint32_t)((b * 2 + m) * kN), sdesc_sw32(smem_addr(sm.ae)),
                                  sdesc_sw32(smem_addr(sm.be[s])), idesc, 1u);
                }
                umma_commit(&sm.b_empty[s]);   // the centroid stage is free once these MMAs finish
                umma_commit(&sm.acc_full[b]);  // and the accumulator pair is ready for the epilogue
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue
        const int e = warp - 2;
        const int m = e >> 2;                // M-half
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int row = m * kMH + q * 32 + lane;
        float best = kNegInf;
        int bidx = 0;
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1, r = t % kBias;
            ok &= mbar_wait(&sm.acc_full[b], (t >> 1) & 1);
            if (METRIC == 1) ok &= mbar_wait(&sm.bias_full[r], (t / kBias) & 1);
            tc_fence_after();
            const int nv = min(kN, K - t * kN);
            const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((b * 2 + m) * kN);
#pragma unroll 1
            for (int c0 = 0; c0 < kN; c0 += 64) {
                if (c0 >= nv) break;
                uint32_t r0[32], r1[32];
                tmem_ld32(tb + (uint32_t)c0, r0);
                tmem_ld32(tb + (uint32_t)c0 + 32, r1);
                tmem_wait_ld();
                if (nv == kN) {
                    fold32<METRIC, true>(r0, sm.bias[r] + c0, t * kN + c0, 32, best, bidx);
                    fold32<METRIC, true>(r1, sm.bias[r] + c0 + 32, t * kN + c0 + 32, 32, best, bidx);
                } else {
                    fold32<METRIC, false>(r0, sm.bias[r] + c0, t * kN + c0, nv - c0, best, bidx);
                    fold32<METRIC, false>(r1, sm.bias[r] + c0 + 32, t * kN + c0 + 32, nv - c0 - 32, best, bidx);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.acc_empty[b]);
                if (METRIC == 1) mbar_arrive(&sm.bias_empty[r]);
            }
        }
        if (p0 + row < N) assign[(size_t)h * N + p0 + row] = bidx;
    }
    if (!ok) atomicExch(err, (int)ASM_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace atc

// ============================================= batched seeding, one round ==
//
// One round of batched k-means++ seeding (bf16, d = 128, up to 256 centres
// per round), fused: the nearest of the round's centres for every point (the
// L2 arg-max above, on tcgen05) and D2 = min(D2, |x - that centre|^2), then
// the sum of D2 over each 32-point range.
//
// D2 must stay exact (fp64 from the stored values), but most points do not
// move in a round.  The accumulator gives <x, c> - |c|^2 / 2 in fp32, so
// |x|^2 - 2 * acc approximates |x - c|^2 to within a few 1e-5 of
// |x|^2 + |c|^2 (131 roundings of 2^-23 each, relative to sum |x_i c_i| and
// |c|^2 / 2, plus the fp32 norms).  As |c|^2 <= 2 |x|^2 + 2 |x - c|^2, the
// margin 2^-9 (3 |x|^2 + 2 |estimate|) is, to first order, at least
// 2^-9 (|x|^2 + |c|^2), some 40 times the error, and needs no |c|^2.  A
// point whose estimate exceeds its D2 by more than that keeps D2 unchanged,
// which the exact distance would also do; the others get the exact fp64
// distance, one warp per point (each lane four elements, a butterfly sum),
// from their row re-read in L2 (streamed in moments before) and their centre
// in shared memory.  Points with D2 = 0 cannot move.
//
// Grid (CTAs per head, heads): a CTA owns a contiguous run of one head's
// 128-point tiles and loads that head's centres once.  Warp 0 streams the
// point tiles (four stages, each free again once its MMAs finish), warp 1
// issues the MMAs into 512 TMEM columns (four accumulators of
// up to 128 centres, two of up to 256), warps 2-17 are four groups of four
// (one per TMEM lane quarter), one per accumulator (the last two idle when
// B > 128), that take the tiles in turn: arg-max, screen, exact update, sums.
// Launched as a dependent of the kernel that picks the round's centres: the
// set-up and the first point tiles overlap its end.  A head with no centre
// this round does no more.  Every wait is bounded; after a timeout a role stops
// and the workspace error word is set.
namespace bsr {

constexpr int kTile = 128;                    // points per item (one M = 128 MMA)
constexpr int kMaxTiles = 2;                  // centre tiles of 128: B <= 256
constexpr int kXStages = 4;                   // point stages (five were measured slower)
constexpr int kGroups = 4;                    // epilogue groups of four warps
constexpr int kThreads = (2 + 4 * kGroups) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kXBytes = 2 * atc::kSub;        // [k-half] 128-row boxes
constexpr int kExact = 4;                     // flagged points per batch of exact distances

struct Smem {
    unsigned char ae[atc::kEBytes];             // the ones the bias parts multiply
    unsigned char ce[kMaxTiles][atc::kEBytes];  // bias parts of the centres
    unsigned char c[kMaxTiles][atc::kBBytes];   // centre tiles ([k-half] 128-row boxes)
    unsigned char x[kXStages][kXBytes];         // point stages
    uint64_t x_full[kXStages], x_empty[kXStages], acc_full[4], acc_empty[4], c_full;
    uint32_t tmem_base;
};

struct Args {
    const __nv_bfloat16 *x;  // [H][N][128] the points (exact distances re-read them from L2)
    const float *xn;     // [H][N] |x|^2 (fp32)
    double *d2;          // [H][N]
    double *bs1;         // [H][NR1] D2 sums of 32-point ranges
    const int *st;       // [H][4]; st[4h + 2] = centres kept this round (0: none)
    int *err;
    int N, B, NR1, tiles;  // tiles: 128-point tiles per head
};

__device__ __forceinline__ double bf16_lo(uint32_t w) { return (double)__uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return (double)__uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kThreads, 1)
bseed_round_tc(const __grid_constant__ atc::Maps maps, const Args a) {
    using namespace atc;
    extern __shared__ unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = (int)((long long)blockIdx.x * a.tiles / gridDim.x);
    const int t1 = (int)((long long)(blockIdx.x + 1) * a.tiles / gridDim.x);
    const int nitems = t1 - t0;
    const int B = a.B, N = a.N, ntiles = (B + kN - 1) / kN;
    // accumulators of ntiles x 128 columns, one per epilogue group: a group
    // consumes every phase of its accumulator's barriers (sharing one between
    // two groups would let a group's parity wait pass on the other's phase)
    const int nacc = ntiles == 1 ? 4 : 2;
    constexpr int nst = kXStages;
    unsigned char *const xs0 = sm.x[0];
    auto ctile = [&](int t) -> unsigned char * { return t ? sm.c[1] : sm.c[0]; };  // no local array
    const size_t hN = (size_t)h * N;

    if (tid == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(&sm.x_full[s], 1);
            mbar_init(&sm.x_empty[s], 1);
        }
        for (int b = 0; b < 4; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 4);
        }
        mbar_init(&sm.c_full, 1);
        fence_mbar_init();
    }
    for (int i = tid; i < kEBytes / 16; i += kThreads) {  // the ones of the bias step
        const uint32_t one = 0x3F80u;
        reinterpret_cast<uint4 *>(sm.ae)[i] = make_uint4(one | (one << 16), one, 0u, 0u);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

    // The points do not depend on the preceding kernel (the round's picks):
    // the first stages stream in before waiting for it.
    const int pre = min(nst, nitems);
    auto load_x = [&](int j) {
        const int s = j % nst;
        unsigned char *dst = xs0 + (size_t)s * kXBytes;
        mbar_arrive_expect_tx(&sm.x_full[s], kXBytes);
        const int p0 = (t0 + j) * kTile;
        tma_load_3d(dst, &maps.x, 0, p0, h, &sm.x_full[s]);
        tma_load_3d(dst + kSub, &maps.x, 64, p0, h, &sm.x_full[s]);
    };
    if (warp == 0 && lane == 0)
        for (int j = 0; j < pre; ++j) load_x(j);
    pdl_wait();
    if (a.st[4 * h + 2] == 0) {
        // no centre this round: D2 and the sums stand; the early copies land first
        if (warp == 0 && lane == 0)
            for (int j = 0; j < pre; ++j) ok &= mbar_wait(&sm.x_full[j], 0);
        goto done;
    }

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&sm.c_full, (uint32_t)ntiles * (kBBytes + kEBytes));
            for (int t = 0; t < ntiles; ++t) {
                tma_load_3d(ctile(t), &maps.c, 0, t * kN, h, &sm.c_full);
                tma_load_3d(ctile(t) + kSub, &maps.c, 64, t * kN, h, &sm.c_full);
                tma_load_3d(sm.ce[t], &maps.e, 0, t * kN, h, &sm.c_full);
            }
            for (int j = pre; j < nitems; ++j) {
                const int s = j % nst;
                if (!(ok = mbar_wait(&sm.x_empty[s], ((j / nst) - 1) & 1))) break;
                load_x(j);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                                   ((uint32_t)(kTile >> 4) << 24);
            ok = mbar_wait(&sm.c_full, 0);
            for (int j = 0; j < nitems && ok; ++j) {
                const int s = j % nst, b = j % nacc, u = j / nacc;
                if (!(ok = mbar_wait(&sm.x_full[s], (j / nst) & 1))) break;
                if (u >= 1 && !(ok = mbar_wait(&sm.acc_empty[b], (u - 1) & 1))) break;
                tc_fence_after();
                const uint32_t x_base = smem_addr(xs0 + (size_t)s * kXBytes);
                for (int t = 0; t < ntiles; ++t) {
                    const uint32_t d = tmem + (uint32_t)((b * ntiles + t) * kN);
                    const uint32_t c_base = smem_addr(ctile(t));
#pragma unroll
                    for (int k = 0; k < kD / 16; ++k) {
                        const uint32_t koff = (uint32_t)((k >> 2) * kSub + (k & 3) * 32);
                        umma_bf16(d, sdesc_sw128(x_base + koff), sdesc_sw128(c_base + koff), idesc, k > 0 ? 1u : 0u);
                    }
                    umma_bf16(d, sdesc_sw32(smem_addr(sm.ae)), sdesc_sw32(smem_addr(sm.ce[t])), idesc, 1u);
                }
                umma_commit(&sm.x_empty[s]);   // the point stage is free once these MMAs finish
                umma_commit(&sm.acc_full[b]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- arg-max, screen, exact D2, sums
        const int e = warp - 2, g = e >> 2, q = warp & 3;  // group, TMEM lane quarter
        const int kh = lane >> 4, ch = (lane & 15) >> 1, hb = (lane & 1) << 3;  // this lane's 4 elements
        if (g >= nacc) goto done;                          // two groups when B > 128
        if (!(ok = mbar_wait(&sm.c_full, 0))) goto done;  // centres read below for exact distances
        for (int j = g; j < nitems; j += nacc) {
            const int b = j % nacc;
            const int base = (t0 + j) * kTile + q * 32;  // this warp's 32 points
            const int p = base + lane;
            const bool inb = p < N;
            const double dold = inb ? __ldcg(a.d2 + hN + p) : 0.0;
            const float xnv = inb ? __ldg(a.xn + hN + p) : 0.f;
            if (!(ok = mbar_wait(&sm.acc_full[b], (j / nacc) & 1))) break;
            tc_fence_after();
            float best = kNegInf;
            int bidx = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int nv = min(kN, B - t * kN);
                const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((b * ntiles + t) * kN);
#pragma unroll 1
                for (int c0 = 0; c0 < kN; c0 += 32) {
                    if (c0 >= nv) break;
                    uint32_t r0[32];
                    tmem_ld32(tb + (uint32_t)c0, r0);
                    tmem_wait_ld();
                    if (nv - c0 >= 32) fold32<0, true>(r0, nullptr, t * kN + c0, 32, best, bidx);
                    else fold32<0, false>(r0, nullptr, t * kN + c0, nv - c0, best, bidx);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
            // screen: keep D2 where the estimate is clearly above it
            const float est = xnv - 2.f * best;
            const float margin = (3.f * xnv + 2.f * fabsf(est)) * 0x1p-9f;
            const bool flag = inb && dold > 0.0 && !((double)(est - margin) > dold);
            unsigned fm = __ballot_sync(0xffffffffu, flag);
            double fin = dold;
            const uint2 *xw = reinterpret_cast<const uint2 *>(a.x + (hN + base) * kD) + lane;  // 4 elements per lane
            while (fm) {
                // up to kExact flagged points at a time: their rows from L2 (just
                // streamed), their centres from shared memory
                int src[kExact];
                uint2 xv[kExact], cv[kExact];
#pragma unroll
                for (int k = 0; k < kExact; ++k) {
                    src[k] = fm ? __ffs(fm) - 1 : -1;
                    fm &= fm - 1;
                    const int c = __shfl_sync(0xffffffffu, bidx, max(src[k], 0)), cr = c & (kN - 1);
                    xv[k] = src[k] >= 0 ? __ldcg(xw + src[k] * (kD / 4)) : make_uint2(0u, 0u);
                    cv[k] = *reinterpret_cast<const uint2 *>(
                        ctile(c >> 7) + kh * kSub + cr * 128 + (((ch ^ (cr & 7)) << 4) | hb));
                }
#pragma unroll
                for (int k = 0; k < kExact; ++k) {
                    if (src[k] < 0) break;  // the same for every lane
                    const double u0 = bf16_lo(xv[k].x) - bf16_lo(cv[k].x), u1 = bf16_hi(xv[k].x) - bf16_hi(cv[k].x);
                    const double u2 = bf16_lo(xv[k].y) - bf16_lo(cv[k].y), u3 = bf16_hi(xv[k].y) - bf16_hi(cv[k].y);
                    double acc = fma(u3, u3, fma(u2, u2, fma(u1, u1, u0 * u0)));
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                    if (lane == src[k] && acc < fin) fin = acc;
                }
            }
            if (inb && fin < dold) a.d2[hN + p] = fin;
            // the 32-point range sum (a butterfly: every lane ends with the same value)
            double v = inb ? fin : 0.0;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0 && base < N) a.bs1[(size_t)h * a.NR1 + base / 32] = v;
        }
    }
done:
    if (!ok) atomicExch(a.err, (int)ASM_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace bsr

bool make_map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows);
bool make_map_rows16(CUtensorMap *m, const void *base, uint64_t d1, uint64_t d2, uint32_t rows);

}  // namespace asmk

// bf16, d = 128.  `norms` [H, K] holds |c|^2 of the stored (bf16) centres
// (the cosine term); `bias` [H, K, 16] bf16 the three parts of -|c|^2 / 2
// in columns 0-2 and zeros (the L2 term; unused for cosine).
cudaError_t asm_assign_tc_launch(const void *x, const void *c, const float *norms, const void *bias, int H, int N,
                                 int K, int metric, int32_t *assign, int *err, cudaStream_t st) {
    using namespace asmk;
    atc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!make_map_3d(&maps.x, x, atc::kD, N, H, atc::kMH) || !make_map_3d(&maps.c, c, atc::kD, K, H, atc::kN) ||
        (metric == 0 && !make_map_rows16(&maps.e, bias, K, H, atc::kN)))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(atc::Smem) + 1024;
    auto kern = metric == 0 ? atc::assign_tc_kernel<0> : atc::assign_tc_kernel<1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((N + atc::kM - 1) / atc::kM, H);
    kern<<<grid, atc::kThreads, smem, st>>>(maps, norms, N, K, assign, err);
    return cudaGetLastError();
}

// One fused round of batched seeding (bf16, d = 128, B <= 256 centres per
// head in `c` [H][B][128]); `bias` [H][B][16] as for the assignment, `xn`
// [H][N] |x|^2; D2 and the 32-point sums are updated in place.
cudaError_t asm_bseed_round_tc_launch(const void *x, const void *c, const void *bias,
                                      const float *xn, double *d2, double *bs1, const int *st, int H, int N,
                                      int B, int NR1, int num_sms, int *err, cudaStream_t stream) {
    using namespace asmk;
    if (B < 1 || B > bsr::kMaxTiles * atc::kN) return cudaErrorInvalidValue;
    atc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!make_map_3d(&maps.x, x, atc::kD, N, H, bsr::kTile) || !make_map_3d(&maps.c, c, atc::kD, B, H, atc::kN) ||
        !make_map_rows16(&maps.e, bias, B, H, atc::kN))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(bsr::Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bsr::bseed_round_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bsr::Args a{};
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.xn = xn;
    a.d2 = d2;
    a.bs1 = bs1;
    a.st = st;
    a.err = err;
    a.N = N;
    a.B = B;
    a.NR1 = NR1;
    a.tiles = (N + bsr::kTile - 1) / bsr::kTile;
    // CTAs per head: one wave over the heads (at least one), at most one per tile
    const int per = std::min(std::max(num_sms / H, 1), a.tiles);
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(per, H);
    cfg.blockDim = dim3(bsr::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bsr::bseed_round_tc, maps, a);
}
