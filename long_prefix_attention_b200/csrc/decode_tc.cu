// decode_tc.cu -- bf16 decode step on tensor cores: split units, then merge.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Fase de Inferencia Online": every query head retrieves its nearest memory
// centroid (Recuperacion) and merges that centroid's stored prefix state with
// its attention over the non-prefix tokens by the online-softmax merge
// (Fusion).
//
// Kernel 1 (asm_decode_units) streams the bytes of the step in 32 KB units,
// one unit per CTA: 128 (d=128) or 256 (d=64) centroid rows of one head, or
// 64 / 128 tokens of K and V for one (row b, KV head g).  The unit arrives
// by TMA (128-byte swizzled boxes) while the warps fetch their query
// fragments; four warps then contract it on tensor cores with the streamed
// operand on the 16-row M side ("swapped" tiles, nothing wasted at batch 1):
//   centroids  D[c, b] = C[c, :] q[b, :]   and |c|^2 = diag(C C^T) from the same fragments
//   attention  S^T[t, h] = K[t, :] q[h, :],   O^T[d, h] = V^T[d, t] P^T[t, h]
// and write one partial per unit: the best (score, index) per row b, or the
// unnormalised (m, l, o) per head.  Centroid units come first in the grid;
// with ASM_DECODE_PREFETCH_CENTROIDS they start their loads before the
// programmatic-dependent-launch wait.
//
// Kernel 2 (asm_decode_merge), one CTA per (b, h), reads every partial of the
// pair in one round (arg-max of the scores, log-sum-exp of the attention
// partials), gathers (a_bar, logZ_bar)[idx] in a second round and writes the
// merged state.  Both kernels use programmatic dependent launch, so the merge
// of one call and the centroid loads of the next overlap the tail of the
// previous kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {
namespace tc {

constexpr int kUnit = 32768;     // bytes per unit
constexpr int kWarps = 4;        // compute warps per unit CTA
constexpr int kThreads = kWarps * 32;
constexpr int kScanFmaRows = 2;  // query rows up to which centroid units scan on CUDA cores

template <int D>
struct Geo {
    static constexpr int ROWB = 2 * D;             // bytes per bf16 row
    static constexpr int CS = kUnit / ROWB;        // centroid rows per unit
    static constexpr int TS = kUnit / (2 * ROWB);  // tokens per unit
    static constexpr int HALVES = D / 64;          // 128-byte column halves
    static constexpr int KS = D / 16;              // k-steps over the head dim
    static constexpr int RMT = CS / kWarps / 16;   // 16-row centroid tiles per warp
    static constexpr int TMT = TS / kWarps / 16;   // 16-token tiles per warp
};

struct Args {
    const __nv_bfloat16 *q;       // [B][Hq][D]
    const __nv_bfloat16 *qs;      // [B][Hq][D] queries of the centroid search (q unless given)
    const __nv_bfloat16 *centroids;             // [Hq][K][D]
    const __nv_bfloat16 *k_cache, *v_cache;     // [B][Hkv][Tmax][D]
    const __nv_bfloat16 *k_prefix, *v_prefix;   // [Hkv][Lp][D]
    const __nv_bfloat16 *a_bar;   // [Hq][K][D]
    const float *logz_bar;        // [Hq][K]
    const int *local_len;         // [B]
    __nv_bfloat16 *out;           // [B][Hq][D]
    float *lse_out;               // [B][Hq] or null
    int *idx_out;                 // [B][Hq] or null
    int B, Hq, Hkv, K, Tmax, Lp;
    float qscale;                 // softmax scale * log2(e)
    int metric, mode, flags;
    int nS;                       // centroid units per head (mode 0)
    int nP, nA;                   // prefix / local units per (b, g)
    int ext_prefix;               // the nP prefix partials come from the batched prefix kernel
    // mode 2 (two-level search): centroid units scan the members of the P
    // clusters the select kernel kept for each (b, h), in nsub units each
    int *sel;                     // [B][Hq][P] kept clusters (workspace)
    const int *seg_off;           // [Hq][K1 + 1] member rows of each cluster
    const __nv_bfloat16 *supers;  // [Hq][K1][D] super-centres
    int K1, P, nsub;
    int n_scan;                   // Hq * nS
    float2 *ws_srch;              // [B][Hq][nS]
    float2 *ws_ml;                // [B][Hq][nP+nA]
    float *ws_o;                  // [B][Hq][nP+nA][D]
    int *ws_err;
};

struct Maps {
    CUtensorMap c, k, v, kp, vp;
};

__device__ __forceinline__ void set_error(int *err) { atomicExch(err, (int)ASM_ERR_TIMEOUT); }

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// s += lo^2 + hi^2 of a packed bf16 pair.
__device__ __forceinline__ float sq2(uint32_t x, float s) {
    const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xffff0000u);
    return fmaf(hi, hi, fmaf(lo, lo, s));
}

// Centroid scan on CUDA cores for a few query rows: one centroid row per
// lane, read as 16-byte chunks of the 128-byte-swizzled tile (four
// wavefronts per warp-wide read, the minimum for 512 bytes), the query rows
// in fp32 shared memory (broadcast reads).  |c|^2 and <q_b, c> in fp32; the
// warp's best (score, index) per query row goes to wbw[b].
template <int D>
__device__ __forceinline__ void scan_fma(const unsigned char *tile, const float *sq, int nq, int metric,
                                         int first, int valid, int warp, int lane, float2 *wbw) {
    using Gm = Geo<D>;
    constexpr int RPL = Gm::CS / (kWarps * 32);  // rows per lane
    constexpr int CH = D / 8;                     // 16-byte chunks per row
    float bs[kScanFmaRows];
    int bi[kScanFmaRows];
#pragma unroll
    for (int b = 0; b < kScanFmaRows; ++b) {
        bs[b] = kNegInf;
        bi[b] = 0x7fffffff;
    }
#pragma unroll
    for (int rr = 0; rr < RPL; ++rr) {
        const int r = (warp * RPL + rr) * 32 + lane;
        float nrm = 0.f, dot[kScanFmaRows];
#pragma unroll
        for (int b = 0; b < kScanFmaRows; ++b) dot[b] = 0.f;
#pragma unroll 4
        for (int c = 0; c < CH; ++c) {
            const int half = c >> 3, cc = c & 7;
            const uint4 v = *reinterpret_cast<const uint4 *>(tile + half * (Gm::CS * 128) + r * 128 +
                                                             ((cc ^ (r & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float x[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                x[2 * k] = __uint_as_float(w[k] << 16);
                x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) nrm = fmaf(x[k], x[k], nrm);
#pragma unroll
            for (int b = 0; b < kScanFmaRows; ++b) {
                if (b < nq) {
                    const float4 q0 = *reinterpret_cast<const float4 *>(sq + b * D + c * 8);
                    const float4 q1 = *reinterpret_cast<const float4 *>(sq + b * D + c * 8 + 4);
                    float t = dot[b];
                    t = fmaf(x[0], q0.x, t); t = fmaf(x[1], q0.y, t); t = fmaf(x[2], q0.z, t);
                    t = fmaf(x[3], q0.w, t); t = fmaf(x[4], q1.x, t); t = fmaf(x[5], q1.y, t);
                    t = fmaf(x[6], q1.z, t); t = fmaf(x[7], q1.w, t);
                    dot[b] = t;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kScanFmaRows; ++b) {
            if (b >= nq) break;
            float sc = (metric == 0) ? dot[b] - 0.5f * nrm : (nrm > 0.f ? dot[b] / sqrtf(nrm) : 0.f);
            int ci = first + r;
            if (r >= valid) { sc = kNegInf; ci = 0x7fffffff; }
            if (better(sc, ci, bs[b], bi[b])) { bs[b] = sc; bi[b] = ci; }
        }
    }
#pragma unroll
    for (int b = 0; b < kScanFmaRows; ++b) {
        if (b >= nq) break;
        warp_argmax(bs[b], bi[b]);
        if (lane == 0) wbw[b] = make_float2(bs[b], __int_as_float(bi[b]));
    }
}

// ------------------------------------------------------------ unit kernel --

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 6)  // six CTAs per SM (shared memory allows six)
asm_decode_units(const Args a, const __grid_constant__ Maps maps) {
    using Gm = Geo<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *tile = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(tile + kUnit);  // [2]: the unit's two halves
    // [W][G][D] attention partials of the warps: over the K half of the tile,
    // which every warp has read (barrier) before any writes here
    float *wo = reinterpret_cast<float *>(tile);
    static_assert(kWarps * G * D * sizeof(float) <= kUnit / 2, "partials fit the K half");
    float *wm = reinterpret_cast<float *>(bar + 2);       // [W][G]
    float *wl = wm + kWarps * G;                          // [W][G]
    float2 *wb = reinterpret_cast<float2 *>(wl + kWarps * G);  // [W][B]
    float *sq = reinterpret_cast<float *>(                   // [kScanFmaRows][D], 16-byte aligned
        (reinterpret_cast<uintptr_t>(wb + kWarps * a.B) + 15) & ~(uintptr_t)15);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, quad = lane & 3, i4 = lane >> 3;
    const uint32_t sbuf = smem_addr(tile);

    // ---- which unit
    const int u = blockIdx.x;
    const bool scan = u < a.n_scan;
    int h = 0, b = 0, g = 0, slot, first, valid;
    bool prefix = false;
    int qrow0 = 0, nq = a.B;  // the query rows a centroid unit serves
    if (scan && a.mode == 2) {
        // one (b, h, kept cluster p, sub-range) per unit; its rows are known
        // once the select kernel has finished
        const int sub = u % a.nsub, r1 = u / a.nsub, p = r1 % a.P, r2 = r1 / a.P;
        h = r2 % a.Hq;
        b = r2 / a.Hq;
        slot = p * a.nsub + sub;
        qrow0 = b;
        nq = 1;
        g = h / G;
        first = 0;
        valid = 0;
    } else if (scan) {
        h = u / a.nS;
        slot = u - h * a.nS;
        first = slot * Gm::CS;
        valid = min(Gm::CS, a.K - first);
        g = h / G;
    } else {
        // prefix units (explicit shared prefix) first, ordered (g, slot, b)
        // with b fastest: the B rows that read one prefix tile run together,
        // so the tile comes from HBM once and from L2 for the other rows;
        // then the local units, ordered (b, g, slot)
        const int v = u - a.n_scan, npu = a.ext_prefix ? 0 : a.B * a.Hkv * a.nP;
        if (v < npu) {
            b = v % a.B;
            const int r = v / a.B;
            slot = r % a.nP;
            g = r / a.nP;
            prefix = true;
        } else {
            const int w = v - npu, bg = w / a.nA;
            slot = a.nP + (w - bg * a.nA);
            b = bg / a.Hkv;
            g = bg - b * a.Hkv;
            prefix = false;
        }
        first = (prefix ? slot : slot - a.nP) * Gm::TS;
        valid = prefix ? min(Gm::TS, a.Lp - first) : Gm::TS;  // refined by the row length below
    }

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Two barriers, so that compute starts on the first half of a unit while
    // the second lands: the column halves of a centroid tile (d = 128; at
    // d = 64 the whole tile is the first half), or the K and V of a token tile.
    auto issue = [&](int vrows) {
        if (scan && vrows > 0) {
#pragma unroll
            for (int hf = 0; hf < Gm::HALVES; ++hf) {
                mbar_arrive_expect_tx(bar + hf, Gm::CS * 128);
                tma_load_3d(tile + hf * Gm::CS * 128, &maps.c, 64 * hf, first, h, bar + hf);
            }
            if (Gm::HALVES == 1) mbar_arrive(bar + 1);
        } else if (scan) {
            mbar_arrive(bar);  // a unit past its cluster's members: nothing to load
            mbar_arrive(bar + 1);
        } else if (vrows > 0) {
            const CUtensorMap *mk = prefix ? &maps.kp : &maps.k;
            const CUtensorMap *mv = prefix ? &maps.vp : &maps.v;
            const int c2 = prefix ? g : b * a.Hkv + g;
            mbar_arrive_expect_tx(bar, Gm::TS * Gm::ROWB);
            mbar_arrive_expect_tx(bar + 1, Gm::TS * Gm::ROWB);
#pragma unroll
            for (int hf = 0; hf < Gm::HALVES; ++hf) tma_load_3d(tile + hf * Gm::TS * 128, mk, 64 * hf, first, c2, bar);
#pragma unroll
            for (int hf = 0; hf < Gm::HALVES; ++hf)
                tma_load_3d(tile + kUnit / 2 + hf * Gm::TS * 128, mv, 64 * hf, first, c2, bar + 1);
        } else {
            mbar_arrive(bar);
            mbar_arrive(bar + 1);
        }
    };
    // static centroids may stream before the dependency wait (caller's choice)
    const bool early = scan && (a.flags & 1) && a.mode != 2;
    if (early && tid == 0) issue(valid);
    if (!early && !(scan && a.mode == 2)) {
        // Warm L2 with this unit's rows while the preceding kernel finishes.
        // Always safe: L2 is the coherence point, so a row the preceding
        // kernel still writes is read correctly after the wait below.  The
        // row count of an attention unit comes from a relaxed read of the
        // length, a hint only (a stale value costs bandwidth, not results).
        int rows = valid;
        const __nv_bfloat16 *kr = nullptr, *vr = nullptr;
        if (scan) {
            kr = a.centroids + ((size_t)h * a.K + first) * D;
        } else if (prefix) {
            kr = a.k_prefix + ((size_t)g * a.Lp + first) * D;
            vr = a.v_prefix + ((size_t)g * a.Lp + first) * D;
        } else {
            int len;
            asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(len) : "l"(a.local_len + b));
            rows = min(Gm::TS, min(max(len, 0), a.Tmax) - first);
            kr = a.k_cache + (((size_t)b * a.Hkv + g) * a.Tmax + first) * D;
            vr = a.v_cache + (((size_t)b * a.Hkv + g) * a.Tmax + first) * D;
        }
        constexpr int LPR = Gm::ROWB / 128;  // 128-byte lines per row
        for (int i = tid; i < rows * LPR; i += kThreads) {
            const size_t off = (size_t)i * 64;  // elements: one line
            asm volatile("prefetch.global.L2 [%0];" ::"l"(kr + off));
            if (vr) asm volatile("prefetch.global.L2 [%0];" ::"l"(vr + off));
        }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (!scan && !prefix) valid = min(Gm::TS, min(max(__ldg(a.local_len + b), 0), a.Tmax) - first);
    if (scan && a.mode == 2) {
        const int c = __ldcg(a.sel + ((size_t)b * a.Hq + h) * a.P + slot / a.nsub);
        const int *so = a.seg_off + (size_t)h * (a.K1 + 1);
        first = __ldg(so + c) + (slot % a.nsub) * Gm::CS;
        valid = min(Gm::CS, __ldg(so + c + 1) - first);
    }
    if (!early && tid == 0) issue(valid);

    if (scan && nq <= kScanFmaRows) {
        // ------------------------------- centroid unit, few query rows: CUDA cores
        for (int i = tid; i < nq * (D / 4); i += kThreads) {
            const int bq = i / (D / 4), c4 = i - bq * (D / 4);
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(a.qs + ((size_t)(qrow0 + bq) * a.Hq + h) * D) + c4);
            *reinterpret_cast<float4 *>(sq + bq * D + 4 * c4) =
                make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                            __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
        }
        __syncthreads();
        if (!mbar_wait(bar, 0) || !mbar_wait(bar + 1, 0)) set_error(a.ws_err);
        scan_fma<D>(tile, sq, nq, a.metric, first, valid, warp, lane, wb + warp * a.B);
    } else if (scan) {
        // ------------------------------- centroid unit, more query rows: tensor cores
        constexpr int KS = Gm::KS, RMT = Gm::RMT;
        float nrl[RMT], nrh[RMT];
#pragma unroll 1
        for (int nt = 0; nt * 8 < nq; ++nt) {
            const int bq = 8 * nt + gid;
            const uint32_t *qr = reinterpret_cast<const uint32_t *>(
                a.qs + ((size_t)(qrow0 + min(bq, nq - 1)) * a.Hq + h) * D);
            uint32_t qb0[KS], qb1[KS];
#pragma unroll
            for (int j = 0; j < KS; ++j) {
                qb0[j] = bq < nq ? __ldg(qr + 8 * j + quad) : 0u;
                qb1[j] = bq < nq ? __ldg(qr + 8 * j + 4 + quad) : 0u;
            }
            // the next n-tile's query rows into L1 while this one multiplies
            constexpr int QL = D * 2 / 128;  // 128-byte lines per query row
            if ((nt + 1) * 8 < nq && lane < 8 * QL) {
                const int rn = min(8 * (nt + 1) + lane / QL, nq - 1);
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a.qs + ((size_t)(qrow0 + rn) * a.Hq + h) * D +
                                                               (lane % QL) * 64));
            }
            if (nt == 0 && !mbar_wait(bar, 0)) set_error(a.ws_err);
            float bs[2] = {kNegInf, kNegInf};
            int bi[2] = {0x7fffffff, 0x7fffffff};
#pragma unroll
            for (int mt = 0; mt < RMT; ++mt) {
                const int r0 = (warp * RMT + mt) * 16;
                const int row = r0 + 8 * (i4 & 1) + (lane & 7);
                float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
                float sl = 0.f, sh = 0.f;
#pragma unroll
                for (int j = 0; j < KS; ++j) {
                    if (j == KS / 2 && nt == 0 && mt == 0 && !mbar_wait(bar + 1, 0)) set_error(a.ws_err);
                    const int col = 16 * j + 8 * (i4 >> 1);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(sbuf + (col >> 6) * (Gm::CS * 128) + swz128(row, (col & 63) >> 3), a0, a1, a2, a3);
                    if (j & 1) mma_bf16_16816(d1, a0, a1, a2, a3, qb0[j], qb1[j]);
                    else       mma_bf16_16816(d0, a0, a1, a2, a3, qb0[j], qb1[j]);
                    if (nt == 0) {
                        // |c|^2 of rows gid (a0, a2) and gid + 8 (a1, a3), this lane's columns
                        sl = sq2(a2, sq2(a0, sl));
                        sh = sq2(a3, sq2(a1, sh));
                    }
                }
                if (nt == 0) {
                    sl += __shfl_xor_sync(0xffffffffu, sl, 1);
                    sh += __shfl_xor_sync(0xffffffffu, sh, 1);
                    sl += __shfl_xor_sync(0xffffffffu, sl, 2);
                    sh += __shfl_xor_sync(0xffffffffu, sh, 2);
                    nrl[mt] = sl;
                    nrh[mt] = sh;
                }
                float dd[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) dd[k] = d0[k] + d1[k];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int rloc = r0 + gid + 8 * hr;
                    const float nr = hr ? nrh[mt] : nrl[mt];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float dot = dd[2 * hr + e];
                        float sc = (a.metric == 0) ? dot - 0.5f * nr : (nr > 0.f ? dot / sqrtf(nr) : 0.f);
                        int ci = first + rloc;
                        if (rloc >= valid) { sc = kNegInf; ci = 0x7fffffff; }
                        if (better(sc, ci, bs[e], bi[e])) { bs[e] = sc; bi[e] = ci; }
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
#pragma unroll
                for (int m = 4; m <= 16; m <<= 1) {
                    const float os = __shfl_xor_sync(0xffffffffu, bs[e], m);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi[e], m);
                    if (better(os, oi, bs[e], bi[e])) { bs[e] = os; bi[e] = oi; }
                }
                const int bb = 8 * nt + 2 * quad + e;
                if (gid == 0 && bb < nq) wb[warp * a.B + bb] = make_float2(bs[e], __int_as_float(bi[e]));
            }
        }
    }
    if (scan) {
        __syncthreads();
#pragma unroll 1
        for (int bb = tid; bb < nq; bb += kThreads) {
            float bs = kNegInf;
            int bi = 0x7fffffff;
            for (int w = 0; w < kWarps; ++w) {
                const float2 v = wb[w * a.B + bb];
                if (better(v.x, __float_as_int(v.y), bs, bi)) { bs = v.x; bi = __float_as_int(v.y); }
            }
            a.ws_srch[((size_t)(qrow0 + bb) * a.Hq + h) * a.nS + slot] = make_float2(bs, __int_as_float(bi));
            if (bi != 0x7fffffff) {
                // warm L2 with this unit's candidate state for the merge's gather
                const __nv_bfloat16 *row = a.a_bar + ((size_t)h * a.K + bi) * D;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(row));
                if (D * 2 > 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 64));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.logz_bar + (size_t)h * a.K + bi));
            }
        }
        return;
    }

    // ------------------------------------------------ attention unit
    constexpr int KS = Gm::KS, TMT = Gm::TMT, NMD = D / 16;
    const int nslots = a.nP + a.nA;
    float *so = wo + warp * G * D;
    if (valid <= 0) {
        // nothing to attend in this unit: an empty partial
        for (int i = tid; i < G * D; i += kThreads) {
            const int hh = i / D, dd = i - hh * D;
            const size_t bh = (size_t)b * a.Hq + g * G + hh;
            a.ws_o[(bh * nslots + slot) * D + dd] = 0.f;
            if (dd == 0) a.ws_ml[bh * nslots + slot] = make_float2(kNegInf, 0.f);
        }
        return;
    }
    // B fragments of Q^T: n = head gid of the group (heads >= G are zero)
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(a.q + ((size_t)b * a.Hq + g * G + min(gid, G - 1)) * D);
    uint32_t qb0[KS], qb1[KS];
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        qb0[j] = gid < G ? __ldg(qrow + 8 * j + quad) : 0u;
        qb1[j] = gid < G ? __ldg(qrow + 8 * j + 4 + quad) : 0u;
    }
    if (!mbar_wait(bar, 0)) set_error(a.ws_err);
    const int t0 = warp * TMT * 16;  // first token of this warp
    float sf[TMT][4];
#pragma unroll
    for (int mt = 0; mt < TMT; ++mt) {
        sf[mt][0] = sf[mt][1] = sf[mt][2] = sf[mt][3] = 0.f;
        const int row = t0 + 16 * mt + 8 * (i4 & 1) + (lane & 7);
#pragma unroll
        for (int j = 0; j < KS; ++j) {
            const int col = 16 * j + 8 * (i4 >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(sbuf + (col >> 6) * (Gm::TS * 128) + swz128(row, (col & 63) >> 3), a0, a1, a2, a3);
            mma_bf16_16816(sf[mt], a0, a1, a2, a3, qb0[j], qb1[j]);
        }
    }
    // base-2 softmax statistics per head (2quad + e) over this warp's tokens
    float mx[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int mt = 0; mt < TMT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int tok = t0 + 16 * mt + gid + 8 * (k >> 1);
            const float v = tok < valid ? sf[mt][k] * a.qscale : kNegInf;
            sf[mt][k] = v;
            mx[k & 1] = fmaxf(mx[k & 1], v);
        }
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int m = 4; m <= 16; m <<= 1) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], m));
    float ls[2] = {0.f, 0.f};
#pragma unroll
    for (int mt = 0; mt < TMT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float v = sf[mt][k];
            const float p = (v == kNegInf) ? 0.f : ex2f(v - mx[k & 1]);
            sf[mt][k] = p;
            ls[k & 1] += p;
        }
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int m = 4; m <= 16; m <<= 1) ls[e] += __shfl_xor_sync(0xffffffffu, ls[e], m);
    // P^T as B fragments (movmatrix turns (token, head) pairs into (head, token))
    uint32_t pb0[TMT], pb1[TMT];
#pragma unroll
    for (int kk = 0; kk < TMT; ++kk) {
        pb0[kk] = movm_t(pack_bf16(sf[kk][0], sf[kk][1]));
        pb1[kk] = movm_t(pack_bf16(sf[kk][2], sf[kk][3]));
    }
    // every warp is done with K (its half becomes the partials), and V is here
    __syncthreads();
    if (!mbar_wait(bar + 1, 0)) set_error(a.ws_err);
    const uint32_t vbase = sbuf + kUnit / 2;
#pragma unroll
    for (int md = 0; md < NMD; ++md) {
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        const int col = 16 * md + 8 * (i4 & 1);
#pragma unroll
        for (int kk = 0; kk < TMT; ++kk) {
            const int row = t0 + 16 * kk + 8 * (i4 >> 1) + (lane & 7);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vbase + (col >> 6) * (Gm::TS * 128) + swz128(row, (col & 63) >> 3), a0, a1, a2, a3);
            mma_bf16_16816(o, a0, a1, a2, a3, pb0[kk], pb1[kk]);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int hh = 2 * quad + e;
            if (hh < G) {
                so[hh * D + 16 * md + gid] = o[e];
                so[hh * D + 16 * md + gid + 8] = o[2 + e];
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int hh = 2 * quad + e;
        if (gid == 0 && hh < G) {
            wm[warp * G + hh] = mx[e];
            wl[warp * G + hh] = ls[e];
        }
    }
    __syncthreads();
    // fold the four warps' states into the unit's partial
#pragma unroll 1
    for (int i = tid; i < G * D; i += kThreads) {
        const int hh = i / D, dd = i - hh * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            if (wl[w * G + hh] > 0.f) M = fmaxf(M, wm[w * G + hh]);
        float L = 0.f, o = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                if (!(wl[w * G + hh] > 0.f)) continue;
                const float sc = ex2f(wm[w * G + hh] - M);
                L += wl[w * G + hh] * sc;
                o += wo[(w * G + hh) * D + dd] * sc;
            }
        }
        const size_t bh = (size_t)b * a.Hq + g * G + hh;
        a.ws_o[(bh * nslots + slot) * D + dd] = o;
        if (dd == 0) a.ws_ml[bh * nslots + slot] = make_float2(M, L);
    }
}

// ---------------------------------------------------------- select kernel --
//
// Two-level search, first level: one CTA per (b, h) scores the K1
// super-centres with the retrieval rule and keeps the P best (ties to the
// smaller cluster index) for the centroid units.

constexpr int kSelMaxK1 = 4096;

template <int D>
__global__ void __launch_bounds__(kThreads)
asm_index_select(const Args a) {
    constexpr int EPL = D / 32;
    const int bh = blockIdx.x, h = bh % a.Hq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ float sc[kSelMaxK1];
    pdl_wait();
    pdl_launch_dependents();
    float qv[EPL];
    load_vec<__nv_bfloat16, EPL>(a.qs + (size_t)bh * D + lane * EPL, qv);
    const __nv_bfloat16 *S = a.supers + (size_t)h * a.K1 * D;
    for (int j = warp; j < a.K1; j += kWarps) {
        float sv[EPL];
        load_vec<__nv_bfloat16, EPL>(S + (size_t)j * D + lane * EPL, sv);
        float dt = 0.f, nr = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            dt = fmaf(qv[e], sv[e], dt);
            nr = fmaf(sv[e], sv[e], nr);
        }
        dt = warp_sum(dt);
        nr = warp_sum(nr);
        if (lane == 0) sc[j] = (a.metric == 0) ? dt - 0.5f * nr : (nr > 0.f ? dt / sqrtf(nr) : 0.f);
    }
    __syncthreads();
    if (warp == 0) {
        for (int p = 0; p < a.P; ++p) {
            float bs = kNegInf;
            int bi = 0x7fffffff;
            for (int j = lane; j < a.K1; j += 32)
                if (better(sc[j], j, bs, bi)) { bs = sc[j]; bi = j; }
            warp_argmax(bs, bi);
            if (bi == 0x7fffffff) bi = 0;
            if (lane == 0) {
                a.sel[(size_t)bh * a.P + p] = bi;
                sc[bi] = kNegInf;
            }
            __syncwarp();
        }
    }
}

// ----------------------------------------------------------- merge kernel --
//
// One CTA per (b, h) of SG x D threads: thread (sg, t) owns output dim t of
// the attention partials sg, sg + SG, ...; it keeps SLOTS of them in flight
// per round.  SG grows with the partial count (16 or 32 partials per
// thread, up to SG = 8), so a long local window or prefix does not turn the
// merge into a serial loop.

constexpr int kMergeSlots = 32;  // partial rows a thread keeps in flight per round (at most)
constexpr int kMergeMaxSG = 8;   // slot groups per CTA (up to 8 x D threads)
constexpr int kMergeSml = 2048;  // (m, l) pairs staged in shared memory

template <int D, int SLOTS>
__global__ void __launch_bounds__(kMergeMaxSG * D)
asm_decode_merge(const Args a) {
    static_assert(SLOTS <= kMergeSlots, "slots per round");
    const int bh = blockIdx.x;
    const int b = bh / a.Hq, h = bh - b * a.Hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NT = blockDim.x, SG = NT / D, sg = tid / D, t = tid - sg * D;
    constexpr int MW = kMergeMaxSG * D / 32;
    __shared__ float red_m[MW];
    __shared__ float2 sb[MW];
    __shared__ int sidx;
    __shared__ float sM;
    __shared__ float2 sml[kMergeSml];
    __shared__ float so[kMergeMaxSG][D];
    __shared__ float sl[kMergeMaxSG];
    const int nslots = a.nP + a.nA;
    const bool search = a.mode != 1;  // a memory lookup (flat or two-level) precedes the merge
    pdl_wait();
    // ---- round 1: the centroid scores, the attention maxima, and each
    //      thread's first SLOTS partials
    float2 best = make_float2(kNegInf, __int_as_float(0x7fffffff));
    if (search) {
        for (int s = tid; s < a.nS; s += NT) {
            const float2 v = __ldcg(a.ws_srch + (size_t)bh * a.nS + s);
            if (better(v.x, __float_as_int(v.y), best.x, __float_as_int(best.y))) best = v;
        }
    }
    const float2 *mlp = a.ws_ml + (size_t)bh * nslots;
    const float *op = a.ws_o + (size_t)bh * nslots * D + t;
    float ov[SLOTS];
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const int s = sg + SG * k;
        ov[k] = s < nslots ? __ldcg(op + (size_t)s * D) : 0.f;
    }
    float mloc = kNegInf;
    for (int s = tid; s < nslots; s += NT) {
        const float2 ml = __ldcg(mlp + s);
        if (s < kMergeSml) sml[s] = ml;
        if (ml.y > 0.f) mloc = fmaxf(mloc, ml.x);
    }
    // block reductions: arg-max of the scores, max of the attention partials
    {
        float bs = best.x;
        int bi = __float_as_int(best.y);
        warp_argmax(bs, bi);
        mloc = warp_max(mloc);
        if (lane == 0) {
            sb[warp] = make_float2(bs, __int_as_float(bi));
            red_m[warp] = mloc;
        }
        __syncthreads();
        if (tid == 0) {
            float s0 = kNegInf;
            int i0 = 0x7fffffff;
            float m0 = kNegInf;
            for (int w = 0; w < NT / 32; ++w) {
                if (better(sb[w].x, __float_as_int(sb[w].y), s0, i0)) { s0 = sb[w].x; i0 = __float_as_int(sb[w].y); }
                m0 = fmaxf(m0, red_m[w]);
            }
            sidx = (i0 == 0x7fffffff) ? 0 : i0;
            sM = m0;
        }
        __syncthreads();
    }
    const int idx = sidx;
    const float M = sM;
    // The next kernel may start now: its prefetch stream (the next step's
    // units warm L2 before their dependency wait) then queues behind this
    // kernel's first round of loads instead of ahead of them.
    pdl_launch_dependents();
    // ---- round 2: the retrieved state (issued before the weighted sums)
    float zb2 = kNegInf, ab = 0.f;
    if (search && sg == 0) {
        zb2 = __ldg(a.logz_bar + (size_t)h * a.K + idx) * kLog2e;
        ab = __bfloat162float(a.a_bar[((size_t)h * a.K + idx) * D + t]);
    }
    float L = 0.f, o = 0.f;
    if (M != kNegInf) {
        for (int k0 = 0;; k0 += SLOTS) {
            if (k0 > 0) {
                if (sg + SG * k0 >= nslots) break;
#pragma unroll
                for (int k = 0; k < SLOTS; ++k) {
                    const int s = sg + SG * (k0 + k);
                    ov[k] = s < nslots ? __ldcg(op + (size_t)s * D) : 0.f;
                }
            }
#pragma unroll
            for (int k = 0; k < SLOTS; ++k) {
                const int s = sg + SG * (k0 + k);
                if (s >= nslots) break;
                const float2 ml = s < kMergeSml ? sml[s] : __ldcg(mlp + s);
                if (ml.y > 0.f) {
                    const float w = ex2f(ml.x - M);
                    L += ml.y * w;
                    o = fmaf(w, ov[k], o);
                }
            }
            if (sg + SG * (k0 + SLOTS) >= nslots) break;
        }
    }
    // slot groups meet in shared memory
    if (SG > 1) {
        so[sg][t] = o;
        if (t == 0) sl[sg] = L;
        __syncthreads();
        if (sg != 0) return;
        for (int gg = 1; gg < SG; ++gg) {
            o += so[gg][t];
            L += sl[gg];
        }
    }
    const float zl2 = (L > 0.f) ? M + lg2f(L) : kNegInf;
    const float loc = (L > 0.f) ? o / L : 0.f;
    float res, lse2;
    if (search && !(zb2 == kNegInf && zl2 == kNegInf)) {
        const float m = fmaxf(zb2, zl2);
        const float eb = ex2f(zb2 - m), el = ex2f(zl2 - m);
        lse2 = m + lg2f(eb + el);
        res = (eb * ab + el * loc) / (eb + el);
    } else if (search) {
        lse2 = kNegInf;
        res = 0.f;
    } else {
        lse2 = zl2;
        res = loc;
    }
    a.out[(size_t)bh * D + t] = __float2bfloat16_rn(res);
    if (t == 0) {
        if (a.lse_out) a.lse_out[bh] = lse2 * kLn2;
        if (a.idx_out && search) a.idx_out[bh] = idx;
    }
}

}  // namespace tc

// ------------------------------------------------------------- host side --

bool make_map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows);

namespace {
struct TcWs {
    size_t off_sel, off_srch, off_ml, off_o, total;
};
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
// mode 0: flat search (K centres); 1: explicit prefix (Lp); 2: two-level
// search with P kept clusters of at most max_seg members (K unused).
TcWs tc_ws_layout(int mode, int B, int Hq, int K, int Lp, int Tmax, int d, int P = 0, int max_seg = 0) {
    const int CS = tc::kUnit / (2 * d), TS = tc::kUnit / (4 * d);
    const size_t nS = mode == 0 ? (size_t)(K + CS - 1) / CS
                    : mode == 2 ? (size_t)P * ((max_seg + CS - 1) / CS) : 0;
    const size_t nP = mode == 1 ? (size_t)(Lp + TS - 1) / TS : 0;
    const size_t nA = (size_t)(Tmax + TS - 1) / TS;
    TcWs w;
    w.off_sel = 256;  // word 0: device-side error code
    w.off_srch = al256(w.off_sel + sizeof(int) * (size_t)B * Hq * (mode == 2 ? P : 0));
    w.off_ml = al256(w.off_srch + sizeof(float2) * (size_t)B * Hq * nS);
    w.off_o = al256(w.off_ml + sizeof(float2) * (size_t)B * Hq * (nP + nA));
    w.total = al256(w.off_o + sizeof(float) * (size_t)B * Hq * (nP + nA) * d);
    return w;
}

template <int D, int G>
cudaError_t tc_launch(tc::Args a, const void *centroids, const void *k_prefix, const void *v_prefix,
                      const void *k_cache, const void *v_cache, cudaStream_t st) {
    using Gm = tc::Geo<D>;
    tc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if ((a.mode == 0 || a.mode == 2) && !make_map_3d(&maps.c, centroids, D, a.K, a.Hq, Gm::CS))
        return cudaErrorInvalidValue;
    if (a.Tmax > 0 && (!make_map_3d(&maps.k, k_cache, D, a.Tmax, (uint64_t)a.B * a.Hkv, Gm::TS) ||
                       !make_map_3d(&maps.v, v_cache, D, a.Tmax, (uint64_t)a.B * a.Hkv, Gm::TS)))
        return cudaErrorInvalidValue;
    if (a.mode == 1 && a.Lp > 0 && (!make_map_3d(&maps.kp, k_prefix, D, a.Lp, a.Hkv, Gm::TS) ||
                                    !make_map_3d(&maps.vp, v_prefix, D, a.Lp, a.Hkv, Gm::TS)))
        return cudaErrorInvalidValue;
    const int units = a.n_scan + a.B * a.Hkv * ((a.ext_prefix ? 0 : a.nP) + a.nA);
    const size_t smem = 1024 + tc::kUnit + 16 + sizeof(float) * tc::kWarps * G * 2 +
                        sizeof(float2) * tc::kWarps * a.B + 16 + sizeof(float) * tc::kScanFmaRows * D;
    auto k1 = tc::asm_decode_units<D, G>;
    static size_t k1_smem = 0;
    if (smem > k1_smem) {
        cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k1_smem = smem;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(units);
    c1.blockDim = dim3(tc::kThreads);
    c1.dynamicSmemBytes = smem;
    c1.stream = st;
    c1.attrs = attr;
    c1.numAttrs = 1;
    if (units > 0) {
        cudaError_t e = cudaLaunchKernelEx(&c1, k1, a, maps);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t c2 = {};
    // slot groups of the merge, at most kMergeMaxSG
    const int nslots = a.nP + a.nA;
    int sg = 1;
    // With few (b, h) pairs (at most 128 merge CTAs) and partials that fit
    // one round at 16 per thread, each thread takes 16, so the CTAs grow and
    // each thread's dependent chain of weighted sums is short (LLaMA layer,
    // B = 1: 9.6 against 10.3 us per step); otherwise 32 per round, so that
    // the CTAs stay small or the rounds few.
    const bool short_rounds = a.B * a.Hq <= 128 && nslots <= 16 * tc::kMergeMaxSG;
    const int per = short_rounds ? 16 : tc::kMergeSlots;
    while (sg < tc::kMergeMaxSG && sg * per < nslots) sg *= 2;
    c2.gridDim = dim3(a.B * a.Hq);
    c2.blockDim = dim3(sg * D);
    c2.stream = st;
    c2.attrs = attr;
    c2.numAttrs = 1;
    return short_rounds ? cudaLaunchKernelEx(&c2, tc::asm_decode_merge<D, 16>, a)
                        : cudaLaunchKernelEx(&c2, tc::asm_decode_merge<D, tc::kMergeSlots>, a);
}

template <int D>
cudaError_t tc_launch_g(int G, const tc::Args &a, const void *c, const void *kp, const void *vp, const void *kc,
                        const void *vc, cudaStream_t st) {
    switch (G) {
        case 1: return tc_launch<D, 1>(a, c, kp, vp, kc, vc, st);
        case 2: return tc_launch<D, 2>(a, c, kp, vp, kc, vc, st);
        case 4: return tc_launch<D, 4>(a, c, kp, vp, kc, vc, st);
        case 8: return tc_launch<D, 8>(a, c, kp, vp, kc, vc, st);
        default: return cudaErrorInvalidValue;
    }
}
}  // namespace

}  // namespace asmk

size_t asm_decode_tc_ws_bytes(int mode, int B, int Hq, int K, int Lp, int Tmax, int d) {
    return asmk::tc_ws_layout(mode, B, Hq, K, Lp, Tmax, d).total;
}

cudaError_t asm_decode_tc_launch(int mode, const void *q, const void *centroids, const void *a_bar,
                                 const float *logz_bar, const void *k_prefix, const void *v_prefix, int Lp,
                                 const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                                 int Hq, int Hkv, int K, int Tmax, int d, float scale, int metric, void *out,
                                 float *lse_out, int32_t *idx_out, unsigned flags, void *ws, cudaStream_t st,
                                 const void *q_search) {
    using namespace asmk;
    const TcWs w = tc_ws_layout(mode, B, Hq, K, Lp, Tmax, d);
    tc::Args a{};
    a.q = (const __nv_bfloat16 *)q;
    a.qs = q_search ? (const __nv_bfloat16 *)q_search : a.q;
    a.centroids = (const __nv_bfloat16 *)centroids;
    a.k_cache = (const __nv_bfloat16 *)k_cache;
    a.v_cache = (const __nv_bfloat16 *)v_cache;
    a.k_prefix = (const __nv_bfloat16 *)k_prefix;
    a.v_prefix = (const __nv_bfloat16 *)v_prefix;
    a.a_bar = (const __nv_bfloat16 *)a_bar;
    a.logz_bar = logz_bar;
    a.local_len = local_len;
    a.out = (__nv_bfloat16 *)out;
    a.lse_out = lse_out;
    a.idx_out = idx_out;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.K = K; a.Tmax = Tmax; a.Lp = Lp;
    a.qscale = scale * kLog2e;
    a.metric = metric;
    a.mode = mode;
    a.flags = (int)flags;
    const int CS = tc::kUnit / (2 * d), TS = tc::kUnit / (4 * d);
    a.nS = mode == 0 ? (K + CS - 1) / CS : 0;
    a.nP = mode == 1 ? (Lp + TS - 1) / TS : 0;
    a.nA = (Tmax + TS - 1) / TS;
    a.n_scan = Hq * a.nS;
    char *base = static_cast<char *>(ws);
    a.ws_err = reinterpret_cast<int *>(base);
    a.ws_srch = reinterpret_cast<float2 *>(base + w.off_srch);
    a.ws_ml = reinterpret_cast<float2 *>(base + w.off_ml);
    a.ws_o = reinterpret_cast<float *>(base + w.off_o);
    const int G = Hq / Hkv;
    if (mode == 1 && Lp > 0 && B >= 2 && d == 128) {
        // A shared prefix read by several rows: tensor-core prefix chunks for
        // all B * G query rows of each KV group at once (the prefix streams
        // once per layer), about two waves of CTAs, written as the first
        // partial slots; the units kernel then covers the local tokens only.
        static int sms = 0;
        if (sms == 0 && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0) != cudaSuccess) sms = 148;
        const int row_tiles = (B * G + 255) / 256;
        int nch = (2 * sms + Hkv * row_tiles - 1) / (Hkv * row_tiles);
        int chunk = (Lp + nch - 1) / nch;
        chunk = ((chunk + 127) / 128) * 128;
        nch = (Lp + chunk - 1) / chunk;
        a.nP = nch;
        a.ext_prefix = 1;
        cudaError_t e = asm_prefix_partials_tc_launch(q, k_prefix, v_prefix, B, Hq, Hkv, Lp, chunk, scale, a.ws_ml,
                                                      a.ws_o, a.nP + a.nA, st);
        if (e != cudaSuccess) return e;
    }
    if (d == 128) return tc_launch_g<128>(G, a, centroids, k_prefix, v_prefix, k_cache, v_cache, st);
    return tc_launch_g<64>(G, a, centroids, k_prefix, v_prefix, k_cache, v_cache, st);
}

size_t asm_decode_indexed_tc_ws_bytes(int B, int Hq, int P, int max_seg, int Tmax, int d) {
    return asmk::tc_ws_layout(2, B, Hq, 0, 0, Tmax, d, P, max_seg).total;
}

// Two-level search decode: select kernel (kept clusters), units (members of
// the kept clusters and the local tokens), merge.
cudaError_t asm_decode_indexed_tc_launch(const void *q, const void *supers, const int32_t *seg_off, int K1, int P,
                                         int max_seg, const void *centroids, const void *a_bar, const float *logz_bar,
                                         const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                                         int Hq, int Hkv, int K, int Tmax, int d, float scale, int metric, void *out,
                                         float *lse_out, int32_t *idx_out, void *ws, cudaStream_t st) {
    using namespace asmk;
    const TcWs w = tc_ws_layout(2, B, Hq, K, 0, Tmax, d, P, max_seg);
    tc::Args a{};
    a.q = (const __nv_bfloat16 *)q;
    a.qs = a.q;
    a.centroids = (const __nv_bfloat16 *)centroids;
    a.k_cache = (const __nv_bfloat16 *)k_cache;
    a.v_cache = (const __nv_bfloat16 *)v_cache;
    a.a_bar = (const __nv_bfloat16 *)a_bar;
    a.logz_bar = logz_bar;
    a.local_len = local_len;
    a.out = (__nv_bfloat16 *)out;
    a.lse_out = lse_out;
    a.idx_out = idx_out;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.K = K; a.Tmax = Tmax; a.Lp = 0;
    a.qscale = scale * kLog2e;
    a.metric = metric;
    a.mode = 2;
    a.flags = 0;
    const int CS = tc::kUnit / (2 * d), TS = tc::kUnit / (4 * d);
    a.K1 = K1;
    a.P = P;
    a.nsub = (max_seg + CS - 1) / CS;
    a.nS = P * a.nsub;
    a.nP = 0;
    a.nA = (Tmax + TS - 1) / TS;
    a.n_scan = B * Hq * a.nS;
    a.seg_off = seg_off;
    a.supers = (const __nv_bfloat16 *)supers;
    char *base = static_cast<char *>(ws);
    a.ws_err = reinterpret_cast<int *>(base);
    a.sel = reinterpret_cast<int *>(base + w.off_sel);
    a.ws_srch = reinterpret_cast<float2 *>(base + w.off_srch);
    a.ws_ml = reinterpret_cast<float2 *>(base + w.off_ml);
    a.ws_o = reinterpret_cast<float *>(base + w.off_o);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c0 = {};
    c0.gridDim = dim3(B * Hq);
    c0.blockDim = dim3(tc::kThreads);
    c0.stream = st;
    c0.attrs = attr;
    c0.numAttrs = 1;
    cudaError_t e = (d == 128) ? cudaLaunchKernelEx(&c0, tc::asm_index_select<128>, a)
                               : cudaLaunchKernelEx(&c0, tc::asm_index_select<64>, a);
    if (e != cudaSuccess) return e;
    const int G = Hq / Hkv;
    if (d == 128) return tc_launch_g<128>(G, a, centroids, nullptr, nullptr, k_cache, v_cache, st);
    return tc_launch_g<64>(G, a, centroids, nullptr, nullptr, k_cache, v_cache, st);
}
