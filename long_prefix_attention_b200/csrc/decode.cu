// decode.cu -- fp32 ASM decode step and full-attention flash-decode.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Fase de Inferencia Online": each query head retrieves the nearest memory
// centroid (Recuperacion) and merges that centroid's precomputed prefix state
// (a_bar, Z_bar) with its attention over the non-prefix tokens through the
// online-softmax merge (Fusion).
//
// One launch does the whole step.  The bytes that must stream from HBM are
// cut into 16 KB work units laid out KV group by KV group (g = KV head):
//     [centroid rows of the G query heads of g] [local K/V of (b=0,g)] ...
// (flash-decode mode instead has, per (b,g), [prefix K/V units][local units]).
// CTA i owns the contiguous unit range [i*upc, (i+1)*upc), one CTA per SM.
// A producer warp streams the units through a ring of shared-memory stages
// with 1-D bulk copies, completing on mbarrier transaction counts; four
// consumer warps process each unit on CUDA cores in fp32 (the bf16 storage
// type runs in decode_tc.cu).  Consecutive units of one key (a head for centroid scans, a
// (b,g) pair for attention) are reduced in registers and written as ONE
// partial per CTA run, into the slot of the run's first unit.  Each CTA then
// adds the run length to the (b,g) arrival counter; the CTA that completes a
// counter merges the partials of that (b,g) -- arg-max of the centroid
// scores, log-sum-exp of the attention partials, the gather of
// (a_bar, logZ_bar)[idx] and the final state merge -- writes the outputs and
// resets the counter for the next call.  No CTA ever waits for another.
//
// Launched with programmatic dependent launch: every thread waits for the
// preceding grid before reading inputs.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace asmk {

constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kUnitBytes = 16384;
constexpr int kDecodeStages = 8;

template <typename T, int D, int G>
struct DCfg {
    static constexpr int EPL = D / 32;                         // dims per lane
    static constexpr int ROWB = D * (int)sizeof(T);            // bytes per row
    static constexpr int CS = kUnitBytes / ROWB;               // centroid rows / unit
    static constexpr int TS = kUnitBytes / (2 * ROWB);         // tokens / unit
    static constexpr int TSW = (32 / G) < TS ? (32 / G) : TS;  // tokens / warp step
    static constexpr int NV = G * TSW;                         // values reduced / step
    static constexpr int R = 32 / NV;                          // lanes per value
    static constexpr int NTG = TS / TSW;                       // token groups / unit
    static constexpr int CSW = CS / kDecodeConsumerWarps;      // centroid rows / warp
    static_assert(NV <= 32 && (NV & (NV - 1)) == 0, "NV");
    static_assert(CSW >= 1 && CSW <= 32 && (CSW & (CSW - 1)) == 0, "CSW");
};

struct DecodeArgs {
    const void *q;
    const void *qs;  // the queries of the centroid search (q unless given)
    const void *centroids;
    const void *a_bar;
    const float *logz_bar;
    const void *k_prefix;
    const void *v_prefix;
    const void *k_cache;
    const void *v_cache;
    const int *local_len;
    void *out;
    float *lse_out;
    int *idx_out;
    int B, Hq, Hkv, K, Tmax, Lp;
    float scale;   // softmax scale
    float qscale;  // scale * log2(e): attention logits are kept in base 2
    int metric;
    int mode;      // 0: memory lookup + local; 1: explicit prefix + local
    int flags;
    int nS;        // centroid units per head (mode 0)
    int nP;        // prefix units per (b,g) (mode 1)
    int nA;        // local units per (b,g)
    int UG;        // units per KV group
    int U;         // total units
    int upc;       // units per CTA
    int ccap;      // (b, g) pairs one CTA may have to merge
    float inv_UG, inv_nS, inv_perb;  // reciprocals for the unit-index divisions
    float2 *ws_srch;  // [B][Hq][nS]   (score, idx bits)
    float2 *ws_ml;    // [B][Hq][nP+nA] (m, l), base-2 logits
    float *ws_o;      // [B][Hq][nP+nA][D] unnormalised outputs
    int *ws_cnt;      // [B][Hkv] arrival counters (self-resetting)
    int *ws_err;
};

// n / d for 0 <= n < 2^31 and d >= 1, from a float reciprocal and an exact fix-up.
__device__ __forceinline__ int fdiv(int n, int d, float inv) {
    int q = __float2int_rz((float)n * inv);
    int r = n - q * d;
    while (r < 0) { --q; r += d; }
    while (r >= d) { ++q; r -= d; }
    return q;
}

// Decoded work unit.
struct Unit {
    int kind;   // 0 = centroid scan, 1 = attention
    int h;      // query head (scan)
    int b, g;   // row and KV head (attention); g also for scans
    int slot;   // slot within the key's partial array
    int first;  // first row (scan) / first token (attention) within its source
    int valid;  // valid rows / tokens in this unit (may be <= 0)
    int prefix; // attention unit over the explicit prefix (mode 1)
    int key;    // run key
};

template <typename T, int D, int G>
__device__ __noinline__ Unit decode_unit(const DecodeArgs &a, int u, const int *lens) {
    using C = DCfg<T, D, G>;
    Unit x;
    x.g = fdiv(u, a.UG, a.inv_UG);
    int r = u - x.g * a.UG;
    x.prefix = 0;
    if (a.mode == 0 && r < G * a.nS) {
        x.kind = 0;
        const int hh = fdiv(r, a.nS, a.inv_nS);
        x.h = x.g * G + hh;
        x.slot = r - hh * a.nS;
        x.b = 0;
        x.first = x.slot * C::CS;
        x.valid = min(C::CS, a.K - x.first);
        x.key = x.h;  // centroid keys: 0 .. Hq-1
        return x;
    }
    x.kind = 1;
    x.h = 0;
    const int per_b = a.nP + a.nA;
    const int r2 = (a.mode == 0) ? r - G * a.nS : r;
    x.b = fdiv(r2, per_b, a.inv_perb);
    x.slot = r2 - x.b * per_b;
    x.key = a.Hq + x.b * a.Hkv + x.g;  // attention keys follow the centroid keys
    if (x.slot < a.nP) {
        x.prefix = 1;
        x.first = x.slot * C::TS;
        x.valid = min(C::TS, a.Lp - x.first);
    } else {
        x.first = (x.slot - a.nP) * C::TS;
        x.valid = lens ? min(C::TS, min(max(__ldg(lens + x.b), 0), a.Tmax) - x.first) : C::TS;
    }
    return x;
}

__device__ __forceinline__ void set_error(int *err) { atomicExch(err, (int)ASM_ERR_TIMEOUT); }

// Runs recorded per CTA before their arrivals are published together.
constexpr int kMaxRuns = 32;

// Publish one run immediately (used only when a CTA has more than kMaxRuns
// runs): fence, count, and queue the (b, g) pairs it completes.
__device__ void publish_run(const DecodeArgs &a, int kind, int g, int b, int len, int G,
                            int *combine_list) {
    __threadfence();
    const int target = (a.mode == 0 ? G * a.nS : a.nP) + a.nA;
    for (int bb = 0; bb < a.B; ++bb) {
        if (kind == 1 && bb != b) continue;
        const int old = atomicAdd(&a.ws_cnt[bb * a.Hkv + g], len);
        if (old + len == target) {
            const int slot = combine_list[0]++;
            if (slot < a.ccap) {
                combine_list[1 + 2 * slot] = bb;
                combine_list[2 + 2 * slot] = g;
            } else {
                set_error(a.ws_err);
            }
        }
    }
}

// Consumer-only barrier (named barrier 1, the four consumer warps).
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecodeConsumerWarps * 32) : "memory");
}

// Slots of a key holding partials: slot 0 and every slot whose unit starts a
// CTA range.  operator()(j) is the j-th such slot (j < count).
struct SlotSeq {
    int first, step, count;
    __device__ SlotSeq(int base, int nslots, int upc) {
        step = upc;
        const int f = (upc - base % upc) % upc;
        if (nslots <= 0) {
            first = 0;
            count = 0;
        } else if (f == 0) {
            first = 0;
            count = (nslots + upc - 1) / upc;
        } else {
            first = f;
            count = 1 + (f < nslots ? (nslots - f + upc - 1) / upc : 0);
        }
    }
    __device__ int operator()(int j) const {
        return first == 0 ? j * step : (j == 0 ? 0 : first + (j - 1) * step);
    }
};

// Merge all partials of (b, g) and write the outputs (consumer warps).  The
// partial rows of a head are read in batches of 8 issued together, then the
// retrieved state is gathered; all weights are computed in base 2.
constexpr int kCombineBatch = 8;

template <typename T, int D, int G, int NW = kDecodeConsumerWarps>
__device__ __noinline__ void combine(const DecodeArgs &a, int b, int g, int warp, int lane) {
    using C = DCfg<T, D, G>;
    const int nslots = a.nP + a.nA;
#pragma unroll 1
    for (int hh = warp; hh < G; hh += NW) {
        const int h = g * G + hh;
        const size_t bh = (size_t)b * a.Hq + h;
        const SlotSeq as(g * a.UG + (a.mode == 0 ? G * a.nS : 0) + b * nslots, nslots, a.upc);
        // retrieval: arg-max over the scan partials of head h
        int idx = 0;
        if (a.mode == 0) {
            const SlotSeq ss(g * a.UG + hh * a.nS, a.nS, a.upc);
            float bs = kNegInf;
            int bi = 0x7fffffff;
#pragma unroll 1
            for (int j = lane; j < ss.count; j += 32) {
                const float2 v = __ldcg(a.ws_srch + bh * a.nS + ss(j));
                const int vi = __float_as_int(v.y);
                if (better(v.x, vi, bs, bi)) { bs = v.x; bi = vi; }
            }
            warp_argmax(bs, bi);
            idx = (bi == 0x7fffffff) ? 0 : bi;
        }
        float ab[C::EPL];
        float zb2 = kNegInf;  // retrieved log Z in base 2
        if (a.mode == 0) {
            zb2 = __ldg(a.logz_bar + (size_t)h * a.K + idx) * kLog2e;
            load_vec<T, C::EPL>((const T *)a.a_bar + ((size_t)h * a.K + idx) * D + lane * C::EPL, ab);
        }
        // log-sum-exp of the attention partials (base 2)
        float M = kNegInf;
#pragma unroll 1
        for (int j = lane; j < as.count; j += 32) {
            const float2 ml = __ldcg(a.ws_ml + bh * nslots + as(j));
            if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        M = warp_max(M);
        float L = 0.f;
        float o[C::EPL];
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) o[e] = 0.f;
        if (M != kNegInf) {
#pragma unroll 1
            for (int j0 = 0; j0 < as.count; j0 += kCombineBatch) {
                // lanes 0..7 hold the batch's weights, every lane its dims of each row
                float w = 0.f;
                if (lane < kCombineBatch && j0 + lane < as.count) {
                    const float2 ml = __ldcg(a.ws_ml + bh * nslots + as(j0 + lane));
                    if (ml.y > 0.f) {
                        w = ex2f(ml.x - M);
                        L += ml.y * w;
                    }
                }
                float v[kCombineBatch][C::EPL];
#pragma unroll
                for (int k = 0; k < kCombineBatch; ++k) {
                    const bool use = j0 + k < as.count;
                    const float *os = a.ws_o + (bh * nslots + as(use ? j0 + k : 0)) * D + lane * C::EPL;
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) v[k][e] = use ? __ldcg(os + e) : 0.f;
                }
#pragma unroll
                for (int k = 0; k < kCombineBatch; ++k) {
                    const float wk = __shfl_sync(0xffffffffu, w, k);
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) o[e] = fmaf(wk, v[k][e], o[e]);
                }
            }
            L = warp_sum(L);
        }
        const float zl2 = (L > 0.f) ? M + lg2f(L) : kNegInf;
        const float invL = (L > 0.f) ? 1.f / L : 0.f;
        float res[C::EPL];
        float lse2;
        if (a.mode == 0 && !(zb2 == kNegInf && zl2 == kNegInf)) {
            const float m = fmaxf(zb2, zl2);
            const float eb = ex2f(zb2 - m), el = ex2f(zl2 - m);
            lse2 = m + lg2f(eb + el);
            const float inv = 1.f / (eb + el);
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) res[e] = (eb * ab[e] + el * (o[e] * invL)) * inv;
        } else if (a.mode == 0) {
            lse2 = kNegInf;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) res[e] = 0.f;
        } else {
            lse2 = zl2;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) res[e] = o[e] * invL;
        }
        store_vec<T, C::EPL>((T *)a.out + bh * D + lane * C::EPL, res);
        if (lane == 0) {
            if (a.lse_out) a.lse_out[bh] = lse2 * kLn2;
            if (a.idx_out && a.mode == 0) a.idx_out[bh] = idx;
        }
    }
}

// ---------------------------------------------------------------- kernel --

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 1)
decode_kernel(const DecodeArgs a) {
    using C = DCfg<T, D, G>;
    constexpr int S = kDecodeStages;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled TMA tiles
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *stage_buf = smem;                                   // S * kUnitBytes
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * kUnitBytes);
    uint64_t *empty = full + S;
    float *flush_o = reinterpret_cast<float *>(empty + S);             // [W][G][D]
    float *flush_m = flush_o + kDecodeConsumerWarps * G * D;           // [W][G]
    float *flush_l = flush_m + kDecodeConsumerWarps * G;               // [W][G]
    float2 *best = reinterpret_cast<float2 *>(flush_l + kDecodeConsumerWarps * G);  // [W][B]
    int *combine_list = reinterpret_cast<int *>(best + kDecodeConsumerWarps * a.B);  // [1 + 2*ccap]
    int4 *runs = reinterpret_cast<int4 *>(combine_list + ((2 * a.ccap + 4) & ~3));  // (kind, g, b, len)
    int *n_runs = reinterpret_cast<int *>(runs + kMaxRuns);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u_begin = blockIdx.x * a.upc;
    const int u_end = min(a.U, u_begin + a.upc);
    const int n_units = u_end - u_begin;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecodeConsumerWarps);
        }
        fence_mbar_init();
        *n_runs = 0;
        combine_list[0] = 0;
    }
    __syncthreads();

    pdl_wait();
    pdl_launch_dependents();
    const int *lens = a.local_len;

    if (warp == kDecodeConsumerWarps) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            // start fetching the row lengths the local units of this range need
            asm volatile("prefetch.global.L1 [%0];" ::"l"(lens));
            asm volatile("prefetch.global.L1 [%0];" ::"l"(lens + (a.B - 1)));
            for (int i = 0; i < n_units; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) set_error(a.ws_err);
                const Unit x = decode_unit<T, D, G>(a, u_begin + i, lens);
                unsigned char *dst = stage_buf + (size_t)s * kUnitBytes;
                if (x.valid <= 0) {
                    mbar_arrive(&full[s]);
                    continue;
                }
                const uint32_t rb = (uint32_t)x.valid * C::ROWB;
                if (x.kind == 0) {
                    const char *src = (const char *)a.centroids + ((size_t)x.h * a.K + x.first) * C::ROWB;
                    mbar_arrive_expect_tx(&full[s], rb);
                    bulk_g2s(dst, src, rb, &full[s]);
                } else {
                    size_t off;
                    const char *kb, *vb;
                    if (x.prefix) {
                        off = ((size_t)x.g * a.Lp + x.first) * C::ROWB;
                        kb = (const char *)a.k_prefix;
                        vb = (const char *)a.v_prefix;
                    } else {
                        off = (((size_t)x.b * a.Hkv + x.g) * a.Tmax + x.first) * C::ROWB;
                        kb = (const char *)a.k_cache;
                        vb = (const char *)a.v_cache;
                    }
                    mbar_arrive_expect_tx(&full[s], 2 * rb);
                    bulk_g2s(dst, kb + off, rb, &full[s]);
                    bulk_g2s(dst + kUnitBytes / 2, vb + off, rb, &full[s]);
                }
            }
            // Drain: every issued copy has landed before the CTA may exit.
            for (int i = max(0, n_units - S); i < n_units; ++i)
                if (!mbar_wait(&full[i % S], (i / S) & 1)) set_error(a.ws_err);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    int cur_key = -1;
    Unit run{};
    int run_len = 0;
    // attention state: (m, l, o) per head of the group, lanes = dims
    float m_run[G], l_run[G], o_run[G][C::EPL];
    float qreg[G][C::EPL];

    auto flush = [&](const Unit &rx, int len) {
        // Publish this CTA's partial of the run's key, then count arrivals.
        if (rx.kind == 0) {
            consumer_sync();
            for (int b = tid; b < a.B; b += kDecodeConsumerWarps * 32) {
                float bs = kNegInf;
                int bi = 0x7fffffff;
                for (int w = 0; w < kDecodeConsumerWarps; ++w) {
                    const float2 v = best[w * a.B + b];
                    const int vi = __float_as_int(v.y);
                    if (better(v.x, vi, bs, bi)) { bs = v.x; bi = vi; }
                }
                a.ws_srch[((size_t)b * a.Hq + rx.h) * a.nS + rx.slot] = make_float2(bs, __int_as_float(bi));
            }
        } else {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if (lane == 0) {
                    flush_m[warp * G + h] = m_run[h];
                    flush_l[warp * G + h] = l_run[h];
                }
#pragma unroll
                for (int e = 0; e < C::EPL; ++e)
                    flush_o[(warp * G + h) * D + lane * C::EPL + e] = o_run[h][e];
            }
            consumer_sync();
            const int nslots = a.nP + a.nA;
            for (int i = tid; i < G * D; i += kDecodeConsumerWarps * 32) {
                const int h = i / D, dd = i % D;
                float M = kNegInf;
                for (int w = 0; w < kDecodeConsumerWarps; ++w)
                    if (flush_l[w * G + h] > 0.f) M = fmaxf(M, flush_m[w * G + h]);
                float L = 0.f, o = 0.f;
                if (M != kNegInf) {
                    for (int w = 0; w < kDecodeConsumerWarps; ++w) {
                        if (!(flush_l[w * G + h] > 0.f)) continue;
                        const float sc = exp2f(flush_m[w * G + h] - M);
                        L += flush_l[w * G + h] * sc;
                        o += flush_o[(w * G + h) * D + dd] * sc;
                    }
                }
                const size_t bh = (size_t)rx.b * a.Hq + rx.g * G + h;
                a.ws_o[(bh * nslots + rx.slot) * D + dd] = o;
                if (dd == 0) a.ws_ml[bh * nslots + rx.slot] = make_float2(M, L);
            }
        }
        // record the run; its arrival is published once, at the end of the CTA
        consumer_sync();
        if (*n_runs >= kMaxRuns) __threadfence();  // overflow: published right away below
        consumer_sync();
        if (tid == 0) {
            const int r = *n_runs;
            if (r < kMaxRuns) {
                runs[r] = make_int4(rx.kind, rx.g, rx.b, len);
                *n_runs = r + 1;
            } else {
                publish_run(a, rx.kind, rx.g, rx.b, len, G, combine_list);  // overflow: at once
            }
        }
        consumer_sync();
    };

    for (int i = 0; i < n_units; ++i) {
        const int s = i % S;
        const Unit x = decode_unit<T, D, G>(a, u_begin + i, lens);
        if (x.key != cur_key) {
            if (cur_key >= 0) flush(run, run_len);
            cur_key = x.key;
            run = x;
            run_len = 0;
            if (x.kind == 0) {
                for (int b = lane; b < a.B; b += 32)
                    best[warp * a.B + b] = make_float2(kNegInf, __int_as_float(0x7fffffff));
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    m_run[h] = kNegInf;
                    l_run[h] = 0.f;
                    float qv[C::EPL];
                    load_vec<T, C::EPL>((const T *)a.q + ((size_t)x.b * a.Hq + x.g * G + h) * D + lane * C::EPL, qv);
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) {
                        o_run[h][e] = 0.f;
                        qreg[h][e] = qv[e] * a.qscale;
                    }
                }
            }
            __syncwarp();
        }
        ++run_len;
        if (!mbar_wait(&full[s], (i / S) & 1)) set_error(a.ws_err);
        const unsigned char *buf = stage_buf + (size_t)s * kUnitBytes;

        if (x.kind == 0) {
            // ---------------- centroid scan (CUDA cores): CSW rows per warp
            const int r0 = warp * C::CSW;
            float nrm[C::CSW];
            float cf[C::CSW][C::EPL];
#pragma unroll
            for (int r = 0; r < C::CSW; ++r) {
                if (r0 + r < x.valid) {
                    load_vec<T, C::EPL>(reinterpret_cast<const T *>(buf + (size_t)(r0 + r) * C::ROWB) + lane * C::EPL, cf[r]);
                } else {
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) cf[r][e] = 0.f;
                }
                float t = 0.f;
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) t = fmaf(cf[r][e], cf[r][e], t);
                nrm[r] = t;
            }
            const float nr = transpose_reduce<C::CSW>(nrm, lane);
            const int my_row = lane / (32 / C::CSW);
            const int my_c = x.first + r0 + my_row;
            const bool my_valid = (r0 + my_row) < x.valid;
            for (int b = 0; b < a.B; ++b) {
                float qv[C::EPL];
                load_vec<T, C::EPL>((const T *)a.qs + ((size_t)b * a.Hq + x.h) * D + lane * C::EPL, qv);
                float dp[C::CSW];
#pragma unroll
                for (int r = 0; r < C::CSW; ++r) {
                    float t = 0.f;
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) t = fmaf(qv[e], cf[r][e], t);
                    dp[r] = t;
                }
                const float dot = transpose_reduce<C::CSW>(dp, lane);
                float sc = (a.metric == 0) ? dot - 0.5f * nr : (nr > 0.f ? dot / sqrtf(nr) : 0.f);
                int ci = my_c;
                if (!my_valid) { sc = kNegInf; ci = 0x7fffffff; }
                warp_argmax(sc, ci);
                if (lane == 0) {
                    const float2 cur = best[warp * a.B + b];
                    if (better(sc, ci, cur.x, __float_as_int(cur.y)))
                        best[warp * a.B + b] = make_float2(sc, __int_as_float(ci));
                }
            }
        } else {
            // ---------------- attention (CUDA cores): warps take token groups
            const unsigned char *kb = buf;
            const unsigned char *vb = buf + kUnitBytes / 2;
            for (int tg = warp; tg < C::NTG; tg += kDecodeConsumerWarps) {
                const int t0 = tg * C::TSW;
                if (t0 >= x.valid) break;
                float part[C::NV];
#pragma unroll
                for (int t = 0; t < C::TSW; ++t) {
                    float kf[C::EPL];
                    if (t0 + t < x.valid) {
                        load_vec<T, C::EPL>(reinterpret_cast<const T *>(kb + (size_t)(t0 + t) * C::ROWB) + lane * C::EPL, kf);
                    } else {
#pragma unroll
                        for (int e = 0; e < C::EPL; ++e) kf[e] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < C::EPL; ++e) acc = fmaf(qreg[h][e], kf[e], acc);
                        part[h * C::TSW + t] = acc;
                    }
                }
                float sv = transpose_reduce<C::NV>(part, lane);
                const int vidx = lane / C::R;
                const int my_t = vidx % C::TSW;
                if (t0 + my_t >= x.valid) sv = kNegInf;
                float mx = sv;
#pragma unroll
                for (int m = 16 / G; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
                float mnew[G], alpha[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float mh = __shfl_sync(0xffffffffu, mx, h * (32 / G));
                    mnew[h] = fmaxf(m_run[h], mh);
                    alpha[h] = (mnew[h] == kNegInf) ? 1.f : exp2f(m_run[h] - mnew[h]);
                }
                const int my_h = vidx / C::TSW;
                float mh_l = mnew[0];
#pragma unroll
                for (int h = 1; h < G; ++h) if (my_h == h) mh_l = mnew[h];
                const float p = (sv == kNegInf) ? 0.f : exp2f(sv - mh_l);
                float ps = p;
#pragma unroll
                for (int m = 16 / G; m >= C::R; m >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float sh = __shfl_sync(0xffffffffu, ps, h * (32 / G));
                    l_run[h] = l_run[h] * alpha[h] + sh;
                    m_run[h] = mnew[h];
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) o_run[h][e] *= alpha[h];
                }
#pragma unroll
                for (int t = 0; t < C::TSW; ++t) {
                    if (t0 + t >= x.valid) break;
                    float vf[C::EPL];
                    load_vec<T, C::EPL>(reinterpret_cast<const T *>(vb + (size_t)(t0 + t) * C::ROWB) + lane * C::EPL, vf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float ph = __shfl_sync(0xffffffffu, p, (h * C::TSW + t) * C::R);
#pragma unroll
                        for (int e = 0; e < C::EPL; ++e) o_run[h][e] = fmaf(ph, vf[e], o_run[h][e]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (cur_key >= 0) flush(run, run_len);

    // Publish: make this CTA's partials visible, then add every run's length
    // to its arrival counters in parallel; a counter that reaches its target
    // marks (b, g) for merging by this CTA.
    __threadfence();
    consumer_sync();
    const int nr = *n_runs;
    for (int t = tid; t < nr * a.B; t += kDecodeConsumerWarps * 32) {
        const int4 rr = runs[t / a.B];
        const int b = t % a.B;
        if (rr.x == 1 && b != rr.z) continue;  // attention runs count for their own row only
        const int target = (a.mode == 0 ? G * a.nS : a.nP) + a.nA;
        const int old = atomicAdd(&a.ws_cnt[b * a.Hkv + rr.y], rr.w);
        if (old + rr.w == target) {
            const int slot = atomicAdd(&combine_list[0], 1);
            if (slot < a.ccap) {
                combine_list[1 + 2 * slot] = b;
                combine_list[2 + 2 * slot] = rr.y;
            } else {
                set_error(a.ws_err);  // cannot happen: ccap bounds the pairs of one CTA
            }
        }
    }
    __threadfence();
    consumer_sync();
    const int nc = min(combine_list[0], a.ccap);
    for (int j = 0; j < nc; ++j) combine<T, D, G>(a, combine_list[1 + 2 * j], combine_list[2 + 2 * j], warp, lane);
    consumer_sync();
    for (int j = tid; j < nc; j += kDecodeConsumerWarps * 32)
        atomicExch(&a.ws_cnt[combine_list[1 + 2 * j] * a.Hkv + combine_list[2 + 2 * j]], 0);
}

// ------------------------------------------------------------- host side --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D bf16 map over decode queries q[B][Hq][d] seen as [B][Hkv][G][d]: a box
// of 64 columns x G heads x 1 group x 128/G rows holds the 128 (row, head)
// pairs of one KV group, row-major by (row, head).
bool make_map_qgroups(CUtensorMap *m, const void *q, int B, int Hkv, int G, int d) {
    auto fn = encode_fn();
    if (!fn || q == nullptr || B < 1 || G < 1 || 128 % G != 0) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)G, (cuuint64_t)Hkv, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)G * d * 2, (cuuint64_t)Hkv * G * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)(128 / G)};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map [d2][d1][d0] with a box of 64 columns x `rows` rows x 1.
bool make_map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows) {
    auto fn = encode_fn();
    if (!fn || base == nullptr || d1 == 0 || d2 == 0) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {64, rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map [d2][d1][16]: a box of the 16 columns (one 32-byte row,
// 32-byte swizzle) x `rows` rows x 1.
bool make_map_rows16(CUtensorMap *m, const void *base, uint64_t d1, uint64_t d2, uint32_t rows) {
    auto fn = encode_fn();
    if (!fn || base == nullptr || d1 == 0 || d2 == 0) return false;
    cuuint64_t dims[3] = {16, d1, d2};
    cuuint64_t strides[2] = {32, 32 * d1};
    cuuint32_t box[3] = {16, rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int G>
static void decode_geometry(DecodeArgs &a, int workers) {
    using C = DCfg<T, D, G>;
    a.nS = (a.mode == 0) ? (a.K + C::CS - 1) / C::CS : 0;
    a.nP = (a.mode == 1) ? (a.Lp + C::TS - 1) / C::TS : 0;
    a.nA = (a.Tmax + C::TS - 1) / C::TS;
    a.UG = (a.mode == 0 ? G * a.nS : 0) + a.B * (a.nP + a.nA);
    a.U = a.Hkv * a.UG;
    a.upc = (a.U + workers - 1) / workers;
    if (a.upc < 1) a.upc = 1;
    // KV groups one CTA range can touch, times the rows of each
    const int groups = min(a.Hkv, (a.upc + a.UG - 1) / a.UG + 1);
    a.ccap = a.B * groups;
    a.inv_UG = 1.f / (float)a.UG;
    a.inv_nS = a.nS > 0 ? 1.f / (float)a.nS : 0.f;
    a.inv_perb = (a.nP + a.nA) > 0 ? 1.f / (float)(a.nP + a.nA) : 0.f;
}

template <typename T, int D, int G>
static cudaError_t decode_launch_t(DecodeArgs a, int num_sms, cudaStream_t st) {
    using C = DCfg<T, D, G>;
    decode_geometry<T, D, G>(a, num_sms);
    const int grid = (a.U + a.upc - 1) / a.upc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
    const size_t smem = 1024 + (size_t)kDecodeStages * kUnitBytes + 2 * kDecodeStages * sizeof(uint64_t) +
                        sizeof(float) * kDecodeConsumerWarps * G * (D + 2) +
                        sizeof(float2) * kDecodeConsumerWarps * a.B + sizeof(int) * ((2 * a.ccap + 4) & ~3) +
                        sizeof(int4) * (kMaxRuns + 1);
    auto kern = decode_kernel<T, D, G>;
    static size_t attr_smem = 0;  // largest dynamic smem opted in so far (per instantiation)
    if (smem > attr_smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_smem = smem;
    }
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, kern, a);
    }
}

template <typename T, int D>
static cudaError_t decode_launch_g(const DecodeArgs &a, int G, int num_sms, cudaStream_t st) {
    switch (G) {
        case 1: return decode_launch_t<T, D, 1>(a, num_sms, st);
        case 2: return decode_launch_t<T, D, 2>(a, num_sms, st);
        case 4: return decode_launch_t<T, D, 4>(a, num_sms, st);
        case 8: return decode_launch_t<T, D, 8>(a, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace asmk

// Workspace layout shared by the size functions and the launcher.
namespace {
struct DecodeWs {
    size_t off_cnt, off_srch, off_ml, off_o, total;
};
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeWs decode_ws_layout(int mode, int B, int Hq, int Hkv, int K, int Lp, int Tmax, int d, asm_dtype dt) {
    const int rowb = d * (dt == ASM_BF16 ? 2 : 4);
    const int CS = asmk::kUnitBytes / rowb, TS = asmk::kUnitBytes / (2 * rowb);
    const size_t nS = mode == 0 ? (size_t)(K + CS - 1) / CS : 0;
    const size_t nP = mode == 1 ? (size_t)(Lp + TS - 1) / TS : 0;
    const size_t nA = (size_t)(Tmax + TS - 1) / TS;
    DecodeWs w;
    w.off_cnt = 256;
    w.off_srch = align256(w.off_cnt + sizeof(int) * (size_t)B * Hkv);
    w.off_ml = align256(w.off_srch + sizeof(float2) * (size_t)B * Hq * nS);
    w.off_o = align256(w.off_ml + sizeof(float2) * (size_t)B * Hq * (nP + nA));
    w.total = align256(w.off_o + sizeof(float) * (size_t)B * Hq * (nP + nA) * d);
    return w;
}
}  // namespace

size_t asm_decode_ws_bytes(int mode, int B, int Hq, int Hkv, int K, int Lp, int Tmax, int d, asm_dtype dt) {
    if (dt == ASM_BF16) return asm_decode_tc_ws_bytes(mode, B, Hq, K, Lp, Tmax, d);
    return decode_ws_layout(mode, B, Hq, Hkv, K, Lp, Tmax, d, dt).total;
}

cudaError_t asm_decode_launch(int mode, const void *q, const void *centroids, const void *a_bar,
                              const float *logz_bar, const void *k_prefix, const void *v_prefix, int Lp,
                              const void *k_cache, const void *v_cache, const int32_t *local_len, int B,
                              int Hq, int Hkv, int K, int Tmax, int d, float scale, int metric, asm_dtype dt,
                              void *out, float *lse_out, int32_t *idx_out, unsigned flags, void *ws,
                              int num_sms, cudaStream_t st, const void *q_search) {
    using namespace asmk;
    DecodeWs w = decode_ws_layout(mode, B, Hq, Hkv, K, Lp, Tmax, d, dt);
    DecodeArgs a{};
    a.q = q; a.qs = q_search ? q_search : q; a.centroids = centroids; a.a_bar = a_bar; a.logz_bar = logz_bar;
    a.k_prefix = k_prefix; a.v_prefix = v_prefix; a.k_cache = k_cache; a.v_cache = v_cache;
    a.local_len = local_len; a.out = out; a.lse_out = lse_out; a.idx_out = idx_out;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.K = K; a.Tmax = Tmax; a.Lp = Lp;
    a.scale = scale; a.qscale = scale * kLog2e; a.metric = metric; a.mode = mode; a.flags = (int)flags;
    char *base = static_cast<char *>(ws);
    a.ws_err = reinterpret_cast<int *>(base);
    a.ws_cnt = reinterpret_cast<int *>(base + w.off_cnt);
    a.ws_srch = reinterpret_cast<float2 *>(base + w.off_srch);
    a.ws_ml = reinterpret_cast<float2 *>(base + w.off_ml);
    a.ws_o = reinterpret_cast<float *>(base + w.off_o);
    const int G = Hq / Hkv;
    if (dt == ASM_BF16)
        return asm_decode_tc_launch(mode, q, centroids, a_bar, logz_bar, k_prefix, v_prefix, Lp, k_cache, v_cache,
                                    local_len, B, Hq, Hkv, K, Tmax, d, scale, metric, out, lse_out, idx_out, flags,
                                    ws, st, q_search);
    if (d == 128) return decode_launch_g<float, 128>(a, G, num_sms, st);
    return decode_launch_g<float, 64>(a, G, num_sms, st);
}

size_t asm_decode_ws_header_bytes(int B, int Hkv, asm_dtype dt) {
    if (dt == ASM_BF16) return 256;  // the bf16 kernels keep no counters: only the error word
    return align256(256 + sizeof(int) * (size_t)B * Hkv);
}
