// decode.cu -- fused ASM decode step and the full-attention flash-decode.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Fase de Inferencia Online": each query head retrieves the nearest memory
// centroid (Recuperacion) and merges that centroid's precomputed prefix state
// (a_bar, Z_bar) with its attention over the non-prefix tokens through the
// online-softmax merge (Fusion).
//
// One launch does the whole step.  The bytes that must stream from HBM are
// cut into 16 KB work units laid out group by group (g = KV head):
//     [centroid rows of the G query heads of g] [local K/V of (b=0,g)] ...
// (flash-decode mode instead has, per (b,g), [prefix K/V units][local units]).
// CTA i owns the contiguous unit range [i*upc, (i+1)*upc).  A producer warp
// streams the units through a ring of shared-memory stages with 1-D bulk
// copies (cp.async.bulk + mbarrier transaction counts); four consumer warps
// process each unit.  Consecutive units of one key (a head for centroid
// scans, a (b,g) pair for attention) are reduced in registers and written as
// ONE partial per CTA run, into the slot of the run's first unit.  Each CTA
// then adds the run length to the (b,g) arrival counter; the CTA that
// completes a counter merges all partials of that (b,g) -- argmax of the
// centroid scores, log-sum-exp of the attention partials, the gather of
// (a_bar, logZ_bar)[idx] and the final state merge -- writes the outputs and
// resets the counter for the next call.  No CTA ever waits for another.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kUnitBytes = 16384;

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
    float qscale;  // scale * log2(e): attention logits are kept in base 2
    int metric;
    int mode;      // 0: memory lookup + local; 1: explicit prefix + local
    int nS;        // centroid units per head (mode 0)
    int nP;        // prefix units per (b,g) (mode 1)
    int nA;        // local units per (b,g)
    int UG;        // units per KV group
    int U;         // total units
    int upc;       // units per CTA
    int stages;
    float2 *ws_srch;  // [B][Hq][nS]   (score, idx bits)
    float2 *ws_ml;    // [B][Hq][nP+nA] (m, l), base-2 logits
    float *ws_o;      // [B][Hq][nP+nA][D] unnormalised outputs
    int *ws_cnt;      // [B][Hkv] arrival counters (self-resetting)
    int *ws_err;
};

// Decoded work unit.
struct Unit {
    int kind;   // 0 = centroid scan, 1 = attention
    int h;      // query head (scan)
    int b, g;   // row and KV head (attention); g also for scans
    int slot;   // slot within the key's partial array
    int first;  // first row (scan) / first token (attention) within its source
    int valid;  // valid rows / tokens in this unit (may be <= 0)
    const char *src_k;  // first byte to copy (scan: centroid rows; attn: K rows)
    const char *src_v;  // attention: V rows
    int key;    // run key
};

template <typename T, int D, int G>
__device__ __forceinline__ Unit decode_unit(const DecodeArgs &a, int u, const int *lens) {
    using C = DCfg<T, D, G>;
    Unit x;
    x.g = u / a.UG;
    int r = u - x.g * a.UG;
    x.src_v = nullptr;
    if (a.mode == 0 && r < G * a.nS) {
        x.kind = 0;
        x.h = x.g * G + r / a.nS;
        x.slot = r % a.nS;
        x.b = 0;
        x.first = x.slot * C::CS;
        x.valid = min(C::CS, a.K - x.first);
        x.src_k = (const char *)a.centroids + ((size_t)x.h * a.K + x.first) * C::ROWB;
        x.key = x.h;  // centroid keys: 0 .. Hq-1
        return x;
    }
    x.kind = 1;
    x.h = 0;
    int per_b = a.nP + a.nA;
    int r2 = (a.mode == 0) ? r - G * a.nS : r;
    x.b = r2 / per_b;
    x.slot = r2 % per_b;
    x.key = a.Hq + x.b * a.Hkv + x.g;  // attention keys follow the centroid keys
    if (x.slot < a.nP) {
        x.first = x.slot * C::TS;
        x.valid = min(C::TS, a.Lp - x.first);
        size_t off = ((size_t)x.g * a.Lp + x.first) * C::ROWB;
        x.src_k = (const char *)a.k_prefix + off;
        x.src_v = (const char *)a.v_prefix + off;
    } else {
        x.first = (x.slot - a.nP) * C::TS;
        x.valid = min(C::TS, lens[x.b] - x.first);
        size_t off = (((size_t)x.b * a.Hkv + x.g) * a.Tmax + x.first) * C::ROWB;
        x.src_k = (const char *)a.k_cache + off;
        x.src_v = (const char *)a.v_cache + off;
    }
    return x;
}

__device__ __forceinline__ void set_error(int *err) { atomicExch(err, (int)ASM_ERR_TIMEOUT); }

// Consumer-only barrier (named barrier 1, the four consumer warps).
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecodeConsumerWarps * 32) : "memory");
}

// Merge all partials of (b, g) and write the outputs (consumer warps).
template <typename T, int D, int G>
__device__ void combine(const DecodeArgs &a, int b, int g, int warp, int lane) {
    using C = DCfg<T, D, G>;
    const int nslots = a.nP + a.nA;
    for (int hh = warp; hh < G; hh += kDecodeConsumerWarps) {
        const int h = g * G + hh;
        const size_t bh = (size_t)b * a.Hq + h;
        // ---- retrieval: arg-max over the scan partials of head h
        int idx = 0;
        if (a.mode == 0) {
            float bs = kNegInf;
            int bi = 0x7fffffff;
            const int ubase = g * a.UG + hh * a.nS;
            for (int s = lane; s < a.nS; s += 32) {
                if (s == 0 || (ubase + s) % a.upc == 0) {
                    float2 v = __ldcg(a.ws_srch + bh * a.nS + s);
                    int vi = __float_as_int(v.y);
                    if (better(v.x, vi, bs, bi)) { bs = v.x; bi = vi; }
                }
            }
            warp_argmax(bs, bi);
            idx = (bi == 0x7fffffff) ? 0 : bi;
        }
        // ---- local (and prefix) attention: log-sum-exp of the partials
        const int abase = g * a.UG + (a.mode == 0 ? G * a.nS : 0) + b * nslots;
        float M = kNegInf;
        for (int s = lane; s < nslots; s += 32) {
            if (s == 0 || (abase + s) % a.upc == 0) {
                float2 ml = __ldcg(a.ws_ml + bh * nslots + s);
                if (ml.y > 0.f) M = fmaxf(M, ml.x);
            }
        }
        M = warp_max(M);
        float L = 0.f;
        float o[C::EPL];
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) o[e] = 0.f;
        if (M != kNegInf) {
            for (int s = 0; s < nslots; ++s) {
                if (!(s == 0 || (abase + s) % a.upc == 0)) continue;
                float2 ml = __ldcg(a.ws_ml + bh * nslots + s);
                if (!(ml.y > 0.f)) continue;
                float w = exp2f(ml.x - M);
                L += ml.y * w;
                const float *os = a.ws_o + (bh * nslots + s) * D + lane * C::EPL;
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[e] += w * __ldcg(os + e);
            }
        }
        float zl = (L > 0.f) ? (M + log2f(L)) * kLn2 : kNegInf;  // natural log
        float res[C::EPL];
        float lse;
        if (a.mode == 0) {
            const float zb = a.logz_bar[(size_t)h * a.K + idx];
            float ab[C::EPL];
            load_vec<T, C::EPL>((const T *)a.a_bar + ((size_t)h * a.K + idx) * D + lane * C::EPL, ab);
            if (zb == kNegInf && zl == kNegInf) {
                lse = kNegInf;
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) res[e] = 0.f;
            } else {
                const float m = fmaxf(zb, zl);
                const float eb = expf(zb - m), el = expf(zl - m);
                lse = m + logf(eb + el);
                const float wb = eb / (eb + el), wl = el / (eb + el);
                const float invL = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) res[e] = wb * ab[e] + wl * (o[e] * invL);
            }
        } else {
            lse = zl;
            const float invL = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) res[e] = o[e] * invL;
        }
        store_vec<T, C::EPL>((T *)a.out + bh * D + lane * C::EPL, res);
        if (lane == 0) {
            if (a.lse_out) a.lse_out[bh] = lse;
            if (a.idx_out && a.mode == 0) a.idx_out[bh] = idx;
        }
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 3)
decode_kernel(const DecodeArgs a) {
    using C = DCfg<T, D, G>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int S = a.stages;
    unsigned char *stage_buf = smem;                                   // S * kUnitBytes
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * kUnitBytes);
    uint64_t *empty = full + S;
    float *flush_o = reinterpret_cast<float *>(empty + S);             // [W][G][D]
    float *flush_m = flush_o + kDecodeConsumerWarps * G * D;           // [W][G]
    float *flush_l = flush_m + kDecodeConsumerWarps * G;               // [W][G]
    float2 *best = reinterpret_cast<float2 *>(flush_l + kDecodeConsumerWarps * G);  // [W][B]
    int *lens = reinterpret_cast<int *>(best + kDecodeConsumerWarps * a.B);         // [B]
    int *combine_list = lens + a.B;                                    // [B+1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u_begin = blockIdx.x * a.upc;
    const int u_end = min(a.U, u_begin + a.upc);
    const int n_units = u_end - u_begin;

    for (int i = tid; i < a.B; i += blockDim.x) lens[i] = min(max(a.local_len[i], 0), a.Tmax);
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecodeConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kDecodeConsumerWarps) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            for (int i = 0; i < n_units; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) set_error(a.ws_err);
                Unit x = decode_unit<T, D, G>(a, u_begin + i, lens);
                unsigned char *dst = stage_buf + (size_t)s * kUnitBytes;
                if (x.valid > 0) {
                    const uint32_t rb = (uint32_t)x.valid * C::ROWB;
                    if (x.kind == 0) {
                        mbar_arrive_expect_tx(&full[s], rb);
                        bulk_g2s(dst, x.src_k, rb, &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], 2 * rb);
                        bulk_g2s(dst, x.src_k, rb, &full[s]);
                        bulk_g2s(dst + C::TS * C::ROWB, x.src_v, rb, &full[s]);
                    }
                } else {
                    mbar_arrive(&full[s]);
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
    // attention running state (one (m, l, o) per head of the group, per warp)
    float m_run[G], l_run[G], o_run[G][C::EPL];
    float qreg[G][C::EPL];

    auto flush = [&](const Unit &rx, int len) {
        // Publish this CTA's partial of the run's key, then count arrivals.
        if (rx.kind == 0) {
            consumer_sync();
            // merge the per-warp bests for every row b
            for (int b = tid; b < a.B; b += kDecodeConsumerWarps * 32) {
                float bs = kNegInf;
                int bi = 0x7fffffff;
                for (int w = 0; w < kDecodeConsumerWarps; ++w) {
                    float2 v = best[w * a.B + b];
                    int vi = __float_as_int(v.y);
                    if (better(v.x, vi, bs, bi)) { bs = v.x; bi = vi; }
                }
                a.ws_srch[((size_t)b * a.Hq + rx.h) * a.nS + rx.slot] =
                    make_float2(bs, __int_as_float(bi));
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
                        float sc = exp2f(flush_m[w * G + h] - M);
                        L += flush_l[w * G + h] * sc;
                        o += flush_o[(w * G + h) * D + dd] * sc;
                    }
                }
                const size_t bh = (size_t)rx.b * a.Hq + rx.g * G + h;
                a.ws_o[(bh * nslots + rx.slot) * D + dd] = o;
                if (dd == 0) a.ws_ml[bh * nslots + rx.slot] = make_float2(M, L);
            }
        }
        // make the partial visible, then count this run's units
        __threadfence();
        consumer_sync();
        if (tid == 0) {
            int n = 0;
            const int target = (a.mode == 0 ? G * a.nS : a.nP) + a.nA;
            if (rx.kind == 0) {
                for (int b = 0; b < a.B; ++b) {
                    int old = atomicAdd(&a.ws_cnt[b * a.Hkv + rx.g], len);
                    if (old + len == target) combine_list[1 + n++] = b;
                }
            } else {
                int old = atomicAdd(&a.ws_cnt[rx.b * a.Hkv + rx.g], len);
                if (old + len == target) combine_list[1 + n++] = rx.b;
            }
            combine_list[0] = n;
            __threadfence();
        }
        consumer_sync();
        const int n = combine_list[0];
        for (int j = 0; j < n; ++j) {
            const int b = combine_list[1 + j];
            combine<T, D, G>(a, b, rx.g, warp, lane);
        }
        consumer_sync();
        if (tid == 0)
            for (int j = 0; j < n; ++j) atomicExch(&a.ws_cnt[combine_list[1 + j] * a.Hkv + rx.g], 0);
    };

    for (int i = 0; i < n_units; ++i) {
        const int s = i % S;
        const Unit x = decode_unit<T, D, G>(a, u_begin + i, lens);
        if (x.key != cur_key) {
            if (cur_key >= 0) flush(run, run_len);
            cur_key = x.key;
            run = x;
            run_len = 0;
            // start a new run
            if (x.kind == 0) {
                for (int b = lane; b < a.B; b += 32)
                    best[warp * a.B + b] = make_float2(kNegInf, __int_as_float(0x7fffffff));
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    m_run[h] = kNegInf;
                    l_run[h] = 0.f;
                    float qv[C::EPL];
                    load_vec<T, C::EPL>((const T *)a.q + ((size_t)x.b * a.Hq + x.g * G + h) * D +
                                            lane * C::EPL, qv);
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
            // ---------------- centroid scan: CSW rows per warp, all rows b
            const int r0 = warp * C::CSW;
            float nrm[C::CSW];
            float cf[C::CSW][C::EPL];
#pragma unroll
            for (int r = 0; r < C::CSW; ++r) {
                if (r0 + r < x.valid) {
                    load_vec<T, C::EPL>(reinterpret_cast<const T *>(buf + (size_t)(r0 + r) * C::ROWB) +
                                            lane * C::EPL, cf[r]);
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
                load_vec<T, C::EPL>((const T *)a.q + ((size_t)b * a.Hq + x.h) * D + lane * C::EPL, qv);
                float dp[C::CSW];
#pragma unroll
                for (int r = 0; r < C::CSW; ++r) {
                    float t = 0.f;
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) t = fmaf(qv[e], cf[r][e], t);
                    dp[r] = t;
                }
                const float dot = transpose_reduce<C::CSW>(dp, lane);
                float sc;
                if (a.metric == 0) sc = dot - 0.5f * nr;
                else sc = nr > 0.f ? dot / sqrtf(nr) : 0.f;
                int ci = my_c;
                if (!my_valid) { sc = kNegInf; ci = 0x7fffffff; }
                warp_argmax(sc, ci);
                if (lane == 0) {
                    float2 cur = best[warp * a.B + b];
                    if (better(sc, ci, cur.x, __float_as_int(cur.y)))
                        best[warp * a.B + b] = make_float2(sc, __int_as_float(ci));
                }
            }
        } else {
            // ---------------- attention over TS tokens: warp takes token groups
            const unsigned char *kb = buf;
            const unsigned char *vb = buf + C::TS * C::ROWB;
            for (int tg = warp; tg < C::NTG; tg += kDecodeConsumerWarps) {
                const int t0 = tg * C::TSW;
                if (t0 >= x.valid) break;
                float part[C::NV];
#pragma unroll
                for (int t = 0; t < C::TSW; ++t) {
                    float kf[C::EPL];
                    if (t0 + t < x.valid) {
                        load_vec<T, C::EPL>(reinterpret_cast<const T *>(kb + (size_t)(t0 + t) * C::ROWB) +
                                                lane * C::EPL, kf);
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
                // per-head max over this step's tokens (lanes of a head are contiguous)
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
                    load_vec<T, C::EPL>(reinterpret_cast<const T *>(vb + (size_t)(t0 + t) * C::ROWB) +
                                            lane * C::EPL, vf);
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
}

// ------------------------------------------------------------- host side --

template <typename T, int D, int G>
static void decode_geometry(DecodeArgs &a, int num_sms, int ctas_per_sm) {
    using C = DCfg<T, D, G>;
    a.nS = (a.mode == 0) ? (a.K + C::CS - 1) / C::CS : 0;
    a.nP = (a.mode == 1) ? (a.Lp + C::TS - 1) / C::TS : 0;
    a.nA = (a.Tmax + C::TS - 1) / C::TS;
    a.UG = (a.mode == 0 ? G * a.nS : 0) + a.B * (a.nP + a.nA);
    a.U = a.Hkv * a.UG;
    const int workers = num_sms * ctas_per_sm;
    a.upc = (a.U + workers - 1) / workers;
    if (a.upc < 1) a.upc = 1;
}

template <typename T, int D, int G>
static cudaError_t decode_launch_t(DecodeArgs a, int num_sms, cudaStream_t st) {
    const int ctas_per_sm = 3;
    a.stages = 4;
    decode_geometry<T, D, G>(a, num_sms, ctas_per_sm);
    const int grid = (a.U + a.upc - 1) / a.upc;
    const size_t smem = (size_t)a.stages * kUnitBytes + 2 * a.stages * sizeof(uint64_t) +
                        sizeof(float) * kDecodeConsumerWarps * G * (D + 2) +
                        sizeof(float2) * kDecodeConsumerWarps * a.B + sizeof(int) * (2 * a.B + 1);
    auto kern = decode_kernel<T, D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kDecodeThreads, smem, st>>>(a);
    return cudaGetLastError();
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

DecodeWs decode_ws_layout(int mode, int B, int Hq, int Hkv, int K, int Lp, int Tmax, int d,
                          asm_dtype dt) {
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

size_t asm_decode_ws_bytes(int mode, int B, int Hq, int Hkv, int K, int Lp, int Tmax, int d,
                           asm_dtype dt) {
    return decode_ws_layout(mode, B, Hq, Hkv, K, Lp, Tmax, d, dt).total;
}

cudaError_t asm_decode_launch(int mode, const void *q, const void *centroids, const void *a_bar,
                              const float *logz_bar, const void *k_prefix, const void *v_prefix,
                              int Lp, const void *k_cache, const void *v_cache,
                              const int32_t *local_len, int B, int Hq, int Hkv, int K, int Tmax,
                              int d, float scale, int metric, asm_dtype dt, void *out,
                              float *lse_out, int32_t *idx_out, void *ws, int num_sms,
                              cudaStream_t st) {
    using namespace asmk;
    DecodeWs w = decode_ws_layout(mode, B, Hq, Hkv, K, Lp, Tmax, d, dt);
    DecodeArgs a{};
    a.q = q; a.centroids = centroids; a.a_bar = a_bar; a.logz_bar = logz_bar;
    a.k_prefix = k_prefix; a.v_prefix = v_prefix; a.k_cache = k_cache; a.v_cache = v_cache;
    a.local_len = local_len; a.out = out; a.lse_out = lse_out; a.idx_out = idx_out;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.K = K; a.Tmax = Tmax; a.Lp = Lp;
    a.qscale = scale * kLog2e; a.metric = metric; a.mode = mode;
    char *base = static_cast<char *>(ws);
    a.ws_err = reinterpret_cast<int *>(base);
    a.ws_cnt = reinterpret_cast<int *>(base + w.off_cnt);
    a.ws_srch = reinterpret_cast<float2 *>(base + w.off_srch);
    a.ws_ml = reinterpret_cast<float2 *>(base + w.off_ml);
    a.ws_o = reinterpret_cast<float *>(base + w.off_o);
    const int G = Hq / Hkv;
    if (dt == ASM_BF16) {
        if (d == 128) return decode_launch_g<__nv_bfloat16, 128>(a, G, num_sms, st);
        return decode_launch_g<__nv_bfloat16, 64>(a, G, num_sms, st);
    }
    if (d == 128) return decode_launch_g<float, 128>(a, G, num_sms, st);
    return decode_launch_g<float, 64>(a, G, num_sms, st);
}
