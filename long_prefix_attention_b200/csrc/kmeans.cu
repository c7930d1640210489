// kmeans.cu -- clustering of the calibration queries into K centroids.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Agrupamiento" (the query vectors are clustered, e.g. by k-means, into K
// centroids) and "Agregacion" (a centroid's query vector is the mean of its
// cluster's queries).  Seeding is k-means++ (D^2 sampling) with the uniform
// draws supplied by the caller.
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <vector>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

namespace {
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
}

// ============================================================ k-means++ ===
//
// One launch per round r.  The centre chosen in round r - 1 lowers D2_i =
// min(D2_i, |x_i - c|^2) (fp64, exact for bf16 inputs and for the products of
// fp32 inputs); the last block of each head to arrive (an arrival counter, no
// waiting) brings the partial sums of D2 up to date, finds where the running
// sum first exceeds u * sum(D2) and records the pick.  The partial sums form
// two levels, each summed in index order: S1 over 32 points and S2 over 32
// consecutive S1.
//
// Exact pruning.  From a regrouping round on, the points are grouped by the
// chosen centre nearest to them (regrouped on a schedule as centres are
// added).  Group g has anchor a_g (its centre) and radius R_g = max |x - a_g|
// over its members; a piece (the part of a group inside one block's range of
// positions) also keeps M >= max sqrt(D2) over its members.  By the triangle
// inequality every member has |x - c| >= |c - a_g| - R_g, so when a lower
// bound of |c - a_g| exceeds R_g + M no member's D2 can fall and the piece is
// skipped.  The lower bound comes from int8 copies of c and a_g with
// power-of-two scales: |c - a| >= |c' - a'| - |c - c'| - |a - a'|, where
// |c' - a'|^2 is formed from an exact integer dot product and the two
// quantisation errors are computed exactly and rounded up.  R_g and M are
// stored rounded up and the margins cover the fp64 rounding, so the D2
// values, and therefore the picks, are those of the unpruned update.
//
// Rounds are chained by programmatic dependent launch: a round's blocks read
// the grouping (static between regroupings) while the previous round ends.

constexpr int kSeedThreads = 256;
constexpr int kSeedWarps = kSeedThreads / 32;
constexpr int kSeedChMin = 2048;     // positions per block: chosen at launch so
constexpr int kSeedChMax = 8192;     // that the grid is one wave
constexpr int kSeedS = 32;           // points per S1 sum, S1 sums per S2 sum
constexpr int kSeedMaxN = 1 << 24;   // S2 dirty bits fit the block's 2 KB bitmap
constexpr double kSeedMargin = 1e-12;
constexpr int kSeedScreen = 128;      // first round of the fp32 screen
// Record of the centre a round picked, for the next round: its row (up to
// 512 bytes), its int8 codes (up to 128 bytes, at 512) and scale, |codes|^2
// and quantisation error (at 640).
constexpr int kSeedCenBytes = 1024;
constexpr int kSeedCenCodes = 512, kSeedCenScal = 640;

struct SeedWs {
    size_t off_d2, off_bs1, off_bs2, off_r2, off_gs, off_ge, off_gr, off_gn, off_near, off_perm, off_gcnt, off_seg,
        off_cur, off_pg, off_pm, off_plo, off_phi, off_pcnt, off_gq, off_dirty, off_taken, off_cnt, off_ctr, off_cen,
        off_skey, off_anc, off_aws, total;
    int nr1, nr2, dstride, nbmax, anchors;
    size_t cap;
};
// Anchors of the static groups that prune the rounds before the first
// grouping by chosen centres (0: none).  Every (N / A)-th point is an anchor;
// each point joins its nearest anchor (tensor-core assignment), so the
// groups need the bf16 d = 128 assignment kernel and enough rounds before
// the first regrouping to pay for themselves.  At the build shape 4096
// anchors gave 228.8 ms of seeding, 3072 235.6 and 6144 228.9 (earlier, with
// the first regrouping at round 1024: 4096 239.7, 2048 and 8192 246.8).
int seed_static_anchors(int N, int d, int K) {
    if (d != 128 || K < 512 || N < 8192) return 0;
    return std::min(4096, std::min(K / 2, N / 16));
}

SeedWs seed_ws(int H, int N, int d, int K) {
    const size_t h = (size_t)H, n = (size_t)N, k = (size_t)K;
    SeedWs w;
    w.nr1 = (N + kSeedS - 1) / kSeedS;
    w.nr2 = (w.nr1 + kSeedS - 1) / kSeedS;
    w.dstride = (w.nr1 + 7) & ~7;  // dirty flags are read 8 at a time
    w.nbmax = (N + kSeedChMin - 1) / kSeedChMin + 1;
    // piece records of block b start at b * (ch + 1): at most N + N / ch + ch + 1
    w.cap = n + (size_t)w.nbmax + kSeedChMax + 1;
    w.off_d2 = 0;
    w.off_bs1 = al256(w.off_d2 + sizeof(double) * h * n);
    w.off_bs2 = al256(w.off_bs1 + sizeof(double) * h * w.nr1);
    w.off_r2 = al256(w.off_bs2 + sizeof(double) * h * w.nr2);
    w.off_gs = al256(w.off_r2 + sizeof(double) * h * k);
    w.off_ge = al256(w.off_gs + sizeof(float) * h * k);
    w.off_gr = al256(w.off_ge + sizeof(float) * h * k);
    w.off_gn = al256(w.off_gr + sizeof(float) * h * k);
    w.off_near = al256(w.off_gn + sizeof(int) * h * k);
    w.off_perm = al256(w.off_near + sizeof(int) * h * n);
    w.off_gcnt = al256(w.off_perm + sizeof(int) * h * n);
    w.off_seg = al256(w.off_gcnt + sizeof(int) * h * k);
    w.off_cur = al256(w.off_seg + sizeof(int) * h * (k + 1));
    w.off_pg = al256(w.off_cur + sizeof(int) * h * k);
    w.off_pm = al256(w.off_pg + sizeof(int) * h * w.cap);
    w.off_plo = al256(w.off_pm + sizeof(float) * h * w.cap);
    w.off_phi = al256(w.off_plo + sizeof(uint16_t) * h * w.cap);
    w.off_pcnt = al256(w.off_phi + sizeof(uint16_t) * h * w.cap);
    w.off_gq = al256(w.off_pcnt + sizeof(int) * h * (size_t)w.nbmax);
    w.off_dirty = al256(w.off_gq + h * k * (size_t)d);
    w.off_taken = al256(w.off_dirty + h * (size_t)w.dstride);
    w.off_cnt = al256(w.off_taken + h * n);
    w.off_ctr = al256(w.off_cnt + sizeof(int) * h);
    w.off_cen = al256(w.off_ctr + sizeof(int) * (size_t)K);
    // the static anchor groups of the early rounds (bf16, d = 128 only)
    w.anchors = seed_static_anchors(N, d, K);
    const size_t a = (size_t)w.anchors;
    w.off_skey = al256(w.off_cen + kSeedCenBytes * h);
    w.off_anc = al256(w.off_skey + (a ? sizeof(int) * h * n : 0));
    w.off_aws = al256(w.off_anc + 2 * h * a * (size_t)d);
    w.total = al256(w.off_aws + (a ? asm_kmeans_ws_bytes(H, N, d, w.anchors) : 0));
    return w;
}

struct SeedArgs {
    const double *u;
    int32_t *idx;           // [H][K] picks
    double *d2;             // [H][N] D2 by point
    double *bs1, *bs2;      // [H][NR1], [H][NR2] partial sums of D2
    double *r2;             // [H][G] group R^2 (regrouping scratch)
    float *gs, *ge, *gr;    // [H][G] anchor scale, anchor quantisation error, R (rounded up)
    int32_t *gn;            // [H][G] |int8 anchor|^2
    int8_t *gq;             // [H][G][D] int8 anchor
    int32_t *near;          // [H][N] round of the nearest chosen centre
    int32_t *perm;          // [H][N] point at each position (grouped order)
    int32_t *gcnt, *seg, *cur;  // regrouping scratch: [H][G], [H][G+1], [H][G]
    int32_t *pg;            // [H][CAP] piece records: group,
    float *pm;              //   bound M (rounded up),
    uint16_t *plo, *phi;    //   first and end offset in the block
    int32_t *pcnt;          // [H][NBMAX] pieces of each block
    unsigned char *dirty;   // [H][DSTRIDE] S1 range touched this round
    unsigned char *taken;   // [H][N] point already chosen
    int *cnt;               // [H] arrival counters
    int *ctr;               // [K] work counters of the rounds with dynamic chunks
    unsigned char *cen;     // [H][kSeedCenBytes] the last chosen centre (see seed_write_centre)
    int32_t *skey;          // [H][N] nearest static anchor of each point
    void *anc;              // [H][A][D] the static anchors' rows
    void *aws;              // workspace of the assignment to the anchors
    int A;                  // static anchors (0: none)
    int N, K, NR1, NR2, DSTRIDE, NBMAX;
    size_t CAP;
};

// Inclusive prefix sum over the block (fp64); every thread gets its value.
__device__ __forceinline__ double block_scan_d(double v, double *sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, v, m);
        if (lane >= m) v += y;
    }
    __syncthreads();
    if (lane == 31) sh[warp] = v;
    __syncthreads();
    double off = 0.0;
    for (int w = 0; w < warp; ++w) off += sh[w];
    return v + off;
}

// Inclusive prefix sum over the warp (fp64, fixed order).
__device__ __forceinline__ double warp_scan_d(double v, int lane) {
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, v, m);
        if (lane >= m) v += y;
    }
    return v;
}

// D2 geometry: a point is LPP lanes x 16 bytes; one 16-byte load per lane
// covers PPL = 32 / LPP points, so a warp reads 32 points with LPP
// independent loads, all issued before any arithmetic.
template <typename T, int D>
struct SeedGeo {
    static constexpr int E16 = 16 / (int)sizeof(T);   // elements per 16-byte load
    static constexpr int LPP = D / E16;                // lanes per point
    static constexpr int PPL = 32 / LPP;               // points per load
};

// Widen the E16 elements of a 16-byte chunk to fp64.
template <typename T>
__device__ __forceinline__ void widen16(const uint4 &u, double *out) {
    if constexpr (sizeof(T) == 4) {
        out[0] = (double)__uint_as_float(u.x);
        out[1] = (double)__uint_as_float(u.y);
        out[2] = (double)__uint_as_float(u.z);
        out[3] = (double)__uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            out[2 * e] = (double)__uint_as_float(w[e] << 16);
            out[2 * e + 1] = (double)__uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
}

// 32 rows at once: lane j names row `row`; rows whose bit in `mask` is clear
// are not read.  Lane l loads 16-byte chunk l % LPP of rows i * PPL + l / LPP.
template <typename T, int D, bool STREAM>
__device__ __forceinline__ void load32(const T *__restrict__ xh, int row, unsigned mask, int lane,
                                       uint4 (&buf)[SeedGeo<T, D>::LPP]) {
    using G = SeedGeo<T, D>;
    const int sub = lane % G::LPP, grp = lane / G::LPP;
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        const int q = i * G::PPL + grp;
        const int src = __shfl_sync(0xffffffffu, row, q);
        const uint4 *pp = reinterpret_cast<const uint4 *>(xh + (size_t)src * D + sub * G::E16);
        buf[i] = ((mask >> q) & 1u) ? (STREAM ? __ldcs(pp) : __ldg(pp)) : make_uint4(0, 0, 0, 0);
    }
}

// |row - c|^2 (fp64) of the rows load32 read: a transpose-reduction over the
// LPP lanes of a row leaves in lane l the distance of row
// (l % LPP) * PPL + l / LPP (the row index seed_row gives).
template <typename T, int D>
__device__ __forceinline__ double dist32(const uint4 (&buf)[SeedGeo<T, D>::LPP], const double *cv, int lane) {
    using G = SeedGeo<T, D>;
    double part[G::LPP];
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        double xv[G::E16];
        widen16<T>(buf[i], xv);
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < G::E16; ++e) {
            const double t = xv[e] - cv[e];
            acc = fma(t, t, acc);
        }
        part[i] = acc;
    }
#pragma unroll
    for (int n = G::LPP; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const double send = up ? part[k] : part[k + half];
            const double keep = up ? part[k + half] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return part[0];
}
// |row|^2 in fp32 of the rows load32 read (same lane layout as dist32); for
// the screen of the fused batched rounds, which allows far more than its error.
template <typename T, int D>
__device__ __forceinline__ float sumsq32(const uint4 (&buf)[SeedGeo<T, D>::LPP], int lane) {
    using G = SeedGeo<T, D>;
    float part[G::LPP];
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        const uint32_t w[4] = {buf[i].x, buf[i].y, buf[i].z, buf[i].w};
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if constexpr (sizeof(T) == 4) {
                const float v = __uint_as_float(w[e]);
                acc = fmaf(v, v, acc);
            } else {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
                acc = fmaf(hi, hi, fmaf(lo, lo, acc));
            }
        }
        part[i] = acc;
    }
#pragma unroll
    for (int n = G::LPP; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = up ? part[k] : part[k + half];
            const float keep = up ? part[k + half] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return part[0];
}
template <typename T, int D>
__device__ __forceinline__ int seed_row(int lane) {
    using G = SeedGeo<T, D>;
    return (lane % G::LPP) * G::PPL + lane / G::LPP;
}


// Widen the E16 elements of a 16-byte chunk to fp32 (exact).
template <typename T>
__device__ __forceinline__ void widen16f(const uint4 &u, float *out) {
    if constexpr (sizeof(T) == 4) {
        out[0] = __uint_as_float(u.x);
        out[1] = __uint_as_float(u.y);
        out[2] = __uint_as_float(u.z);
        out[3] = __uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            out[2 * e] = __uint_as_float(w[e] << 16);
            out[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
}


// dist32 in fp32 (same lane layout): each of the D terms and partial sums is
// rounded once, so the result is within (D + 2) 2^-24 < 1e-5 (D <= 128)
// relative of the exact squared distance.
template <typename T, int D>
__device__ __forceinline__ float dist32f(const uint4 (&buf)[SeedGeo<T, D>::LPP], const float *cv, int lane) {
    using G = SeedGeo<T, D>;
    float part[G::LPP];
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        float xv[G::E16];
        widen16f<T>(buf[i], xv);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < G::E16; ++e) {
            const float t = xv[e] - cv[e];
            acc = fmaf(t, t, acc);
        }
        part[i] = acc;
    }
#pragma unroll
    for (int n = G::LPP; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = up ? part[k] : part[k + half];
            const float keep = up ? part[k + half] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return part[0];
}

// A point's D2 can fall only if its fp32 distance, lowered by its rounding
// bound, is not above D2 (with the fp64 margin): otherwise the exact update
// would leave D2 as it is.
__device__ __forceinline__ bool seed_may_fall(float d32, double old) {
    return !((double)d32 * (1.0 - 1e-5) > old * (1.0 + kSeedMargin));
}

// ---- int8 copies for the anchor test
//
// A row of D int8 is D / 16 lanes x 16 bytes; a warp covers 32 rows with
// D / 16 loads per lane (the layout of load32 with 16-byte chunks of int8).
template <int D>
struct Q8 {
    static constexpr int L8 = D / 16;  // lanes per row
    static constexpr int R8 = 32 / L8;  // rows per load
};
template <int D>
__device__ __forceinline__ int q8_row(int lane) {
    return (lane % Q8<D>::L8) * Q8<D>::R8 + lane / Q8<D>::L8;
}
template <int D>
__device__ __forceinline__ int q8_lane(int row) {
    return (row % Q8<D>::R8) * Q8<D>::L8 + row / Q8<D>::R8;
}

// Power-of-two scale s with max|v| <= 127 s (1 for a zero vector).
__device__ __forceinline__ float q8_scale(float amax) {
    if (!(amax > 0.f)) return 1.f;
    int e;
    frexpf(amax * (1.0f / 127.0f) * (1.0f + 1e-6f), &e);
    return ldexpf(1.0f, e);
}
__device__ __forceinline__ int q8_code(float v, float s) {
    return max(-127, min(127, __float2int_rn(v / s)));
}

// Exact integer dot products of 32 int8 rows (loaded as by load32) with this
// lane's 16-byte chunk of an int8 vector; the transpose-reduction leaves in
// lane l the dot product of row q8_row(l).
template <int D>
__device__ __forceinline__ int dot32q(const uint4 (&buf)[Q8<D>::L8], const uint4 &qc, int lane) {
    constexpr int L8 = Q8<D>::L8;
    int part[L8];
#pragma unroll
    for (int i = 0; i < L8; ++i) {
        int acc = __dp4a((int)buf[i].x, (int)qc.x, 0);
        acc = __dp4a((int)buf[i].y, (int)qc.y, acc);
        acc = __dp4a((int)buf[i].z, (int)qc.z, acc);
        part[i] = __dp4a((int)buf[i].w, (int)qc.w, acc);
    }
#pragma unroll
    for (int n = L8; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const int send = up ? part[k] : part[k + half];
            const int keep = up ? part[k + half] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return part[0];
}

// The int8 copy of a vector held by the warp, 16 elements per lane (lane l:
// elements (l % L8) * 16 ..): its scale, this lane's codes, |codes|^2 and the
// quantisation error |v - s codes| (fp64, rounded up to float).
template <typename T, int D>
__device__ __forceinline__ void q8_vector(const T *__restrict__ v, int lane, float &s, uint4 &codes, int &n2,
                                          float &err) {
    constexpr int L8 = Q8<D>::L8;
    const int c0 = (lane % L8) * 16;
    float f[16];
    if constexpr (sizeof(T) == 2) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(v + c0));
        const uint4 b = __ldg(reinterpret_cast<const uint4 *>(v + c0 + 8));
        widen16f<T>(a, f);
        widen16f<T>(b, f + 8);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) widen16f<T>(__ldg(reinterpret_cast<const uint4 *>(v + c0 + 4 * k)), f + 4 * k);
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    s = q8_scale(amax);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    int nn = 0;
    double ee = 0.0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const int q = q8_code(f[e], s);
        w[e >> 2] |= ((uint32_t)(q & 0xff)) << (8 * (e & 3));
        nn += q * q;
        const double dlt = (double)f[e] - (double)q * (double)s;
        ee = fma(dlt, dlt, ee);
    }
    codes = make_uint4(w[0], w[1], w[2], w[3]);
    // each chunk is held by R8 lanes: count lanes 0 .. L8 - 1 only
    if (lane >= L8) {
        nn = 0;
        ee = 0.0;
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        nn += __shfl_xor_sync(0xffffffffu, nn, m);
        ee += __shfl_xor_sync(0xffffffffu, ee, m);
    }
    n2 = nn;
    err = __double2float_ru(sqrt(ee) * (1.0 + kSeedMargin));
}

// Warp-wide: write the record of centre pk of a head (its row, then the int8
// copy the anchor test uses) for the next round, which then reads one record
// instead of the centre's index and then its row.  Out of line, like the
// refresh below, so that the round kernels' own code stays as it was.
template <typename T, int D>
__device__ __noinline__ void seed_write_centre(const T *__restrict__ xh, int pk, unsigned char *rec, int lane) {
    constexpr int L8 = Q8<D>::L8, U = 16 * (int)sizeof(T) / 16;  // uint4 per lane's 16 elements
    float sc, ec;
    uint4 qc;
    int n2;
    q8_vector<T, D>(xh + (size_t)pk * D, lane, sc, qc, n2, ec);
    if (lane < L8) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xh + (size_t)pk * D + lane * 16);
        uint4 *dst = reinterpret_cast<uint4 *>(rec) + lane * U;
#pragma unroll
        for (int k = 0; k < U; ++k) dst[k] = __ldg(src + k);
        reinterpret_cast<uint4 *>(rec + kSeedCenCodes)[lane] = qc;
    }
    if (lane == 0) {
        reinterpret_cast<float *>(rec + kSeedCenScal)[0] = sc;
        reinterpret_cast<int *>(rec + kSeedCenScal)[1] = n2;
        reinterpret_cast<float *>(rec + kSeedCenScal)[2] = ec;
    }
}

// The refresh with every S1 and S2 sum of the head cached in shared memory
// (s1c [NR1], s2c [NR2]): one round of loads brings the flags and all sums,
// the flagged S1 sums are recomputed from D2 and the S2 sums above them from
// the cache.  Out of line: inlined into the round kernel, it changed the code
// of the update loop before it and slowed that by more than it saves.
__device__ __noinline__ void seed_refresh_cached(double *b1, double *b2, unsigned char *dh, const double *d2h, int N,
                                                 int NR1, int NR2, int *dl, uint32_t *sd2, double *s1c, double *s2c,
                                                 int *nlist) {
    const int tid = threadIdx.x;
    // one round of loads: the flags, every S1 sum and every S2 sum
    uint2 f[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int kb = (i * kSeedThreads + tid) * 8;
        f[i] = kb < NR1 ? __ldcg(reinterpret_cast<const uint2 *>(dh + kb)) : make_uint2(0u, 0u);
    }
    // (every load issued before the first store: the stores go through a
    // generic pointer that could alias them)
    constexpr int kS1PerThread = 16;  // NR1 <= 2 * 8 * kSeedThreads
    double t1[kS1PerThread];
#pragma unroll
    for (int i = 0; i < kS1PerThread; ++i) {
        const int k = i * kSeedThreads + tid;
        t1[i] = k < NR1 ? __ldcg(b1 + k) : 0.0;
    }
    const double t2 = tid < NR2 ? __ldcg(b2 + tid) : 0.0;
#pragma unroll
    for (int i = 0; i < kS1PerThread; ++i) {
        const int k = i * kSeedThreads + tid;
        if (k < NR1) s1c[k] = t1[i];
    }
    if (tid < NR2) s2c[tid] = t2;
    for (int i = tid; i < (NR2 + 31) / 32; i += kSeedThreads) sd2[i] = 0u;
    if (tid == 0) *nlist = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int kb = (i * kSeedThreads + tid) * 8;
        const unsigned long long bits = (unsigned long long)f[i].x | ((unsigned long long)f[i].y << 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (((bits >> (8 * e)) & 0xffull) && kb + e < NR1) {
                const int k = kb + e;
                dl[atomicAdd(nlist, 1)] = k;
                atomicOr(&sd2[k >> 10], 1u << ((k >> 5) & 31));
            }
    }
    __syncthreads();
    const int nd = *nlist;
    for (int j = tid; j < nd; j += kSeedThreads) {
        const int k = dl[j];
        const int q0 = k * kSeedS, q1 = min(N, q0 + kSeedS);
        double v = 0.0;
        if (q1 - q0 == kSeedS) {
            double t[kSeedS];
#pragma unroll
            for (int e = 0; e < kSeedS; ++e) t[e] = __ldcg(d2h + q0 + e);
#pragma unroll
            for (int e = 0; e < kSeedS; ++e) v += t[e];
        } else {
            for (int i = q0; i < q1; ++i) v += __ldcg(d2h + i);
        }
        b1[k] = v;
        s1c[k] = v;
        dh[k] = 0;
    }
    __syncthreads();
    if (tid < NR2 && ((sd2[tid >> 5] >> (tid & 31)) & 1u)) {
        const int k0 = tid * kSeedS, k1 = min(NR1, k0 + kSeedS);
        double v = 0.0;
        for (int k = k0; k < k1; ++k) v += s1c[k];
        b2[tid] = v;
        s2c[tid] = v;
    }
}

// ---- arrival and pick (the last of the `arrivals` arrivals of head h in round r)
//
// REFRESH: bring the S1 sums of the ranges flagged this round and the S2
// sums above them up to date first.  dl (>= 2048 ints) and sd2 (>= 2048
// bytes) are shared memory the block no longer needs.  With a shared-memory
// cache of `cache_n` doubles that holds every S1 and S2 sum of the head, the
// sums are loaded once, together with the flags, and the refresh and the
// scans read them from there (the same values in the same order, so the same
// pick, with fewer dependent trips to L2).
template <bool REFRESH, typename T, int D>
__device__ __forceinline__ void seed_arrive_pick(const T *__restrict__ x, const SeedArgs &s, int h, int r,
                                                 int arrivals, int *dl, uint32_t *sd2, double *cache = nullptr,
                                                 int cache_n = 0) {
    __shared__ double sh[kSeedWarps];
    __shared__ int nlist, last, pick_blk;
    __shared__ double sh_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = s.N, K = s.K;
    const size_t hN = (size_t)h * N;
    double *d2h = s.d2 + hN;
    unsigned char *tk = s.taken + hN;
    unsigned char *dh = s.dirty + (size_t)h * s.DSTRIDE;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int old = atomicAdd(&s.cnt[h], 1);
        last = (old == arrivals - 1);
        __threadfence();
    }
    __syncthreads();
    if (!last) return;

    const double ur = s.u[(size_t)h * K + r];
    const T *xh = x + hN * D;
    unsigned char *rec = s.cen + (size_t)h * kSeedCenBytes;
    if (r == 0) {
        if (warp == 0) {
            int pk = (int)floor(ur * (double)N);
            pk = min(max(pk, 0), N - 1);
            if (lane == 0) {
                s.idx[(size_t)h * K] = pk;
                tk[pk] = 1;
                s.cnt[h] = 0;
            }
            seed_write_centre<T, D>(xh, pk, rec, lane);
        }
        return;
    }
    const int NR1 = s.NR1, NR2 = s.NR2;
    double *b1 = s.bs1 + (size_t)h * NR1;
    double *b2 = s.bs2 + (size_t)h * NR2;
    // cached: every S1 and S2 sum in shared memory (at most two flag words of
    // 8 ranges per thread, one scan chunk of S2 sums)
    const bool cached = REFRESH && cache != nullptr && NR1 + NR2 <= cache_n && NR1 <= 2 * 8 * kSeedThreads &&
                        NR2 <= kSeedThreads;
    double *s1c = cache, *s2c = cached ? cache + NR1 : nullptr;
    if (cached) {
        seed_refresh_cached(b1, b2, dh, d2h, N, NR1, NR2, dl, sd2, s1c, s2c, &nlist);
    } else if constexpr (REFRESH) {
        // S1 sums of the ranges touched this round (each in index order),
        // then the S2 sums over them
        for (int i = tid; i < (NR2 + 31) / 32; i += kSeedThreads) sd2[i] = 0u;
        for (int k0 = 0; k0 < NR1; k0 += kSeedThreads * 8) {
            if (tid == 0) nlist = 0;
            __syncthreads();
            const int kb = k0 + tid * 8;
            if (kb < NR1) {
                const uint2 f = __ldcg(reinterpret_cast<const uint2 *>(dh + kb));
                const unsigned long long bits = (unsigned long long)f.x | ((unsigned long long)f.y << 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (((bits >> (8 * e)) & 0xffull) && kb + e < NR1) {
                        const int k = kb + e;
                        dl[atomicAdd(&nlist, 1)] = k;
                        atomicOr(&sd2[k >> 10], 1u << ((k >> 5) & 31));
                    }
            }
            __syncthreads();
            const int nd = nlist;
            for (int j = tid; j < nd; j += kSeedThreads) {
                const int k = dl[j];
                const int q0 = k * kSeedS, q1 = min(N, q0 + kSeedS);
                double v = 0.0;
                if (q1 - q0 == kSeedS) {
                    double t[kSeedS];
#pragma unroll
                    for (int e = 0; e < kSeedS; ++e) t[e] = __ldcg(d2h + q0 + e);
#pragma unroll
                    for (int e = 0; e < kSeedS; ++e) v += t[e];
                } else {
                    for (int i = q0; i < q1; ++i) v += __ldcg(d2h + i);
                }
                b1[k] = v;
                dh[k] = 0;
            }
            __syncthreads();
        }
        for (int k2 = tid; k2 < NR2; k2 += kSeedThreads) {
            if ((sd2[k2 >> 5] >> (k2 & 31)) & 1u) {
                const int k0 = k2 * kSeedS, k1 = min(NR1, k0 + kSeedS);
                double v = 0.0;
                for (int k = k0; k < k1; ++k) v += __ldcg(b1 + k);
                b2[k2] = v;
            }
        }
    }
    __syncthreads();
    auto get1 = [&](int k) { return cached ? s1c[k] : __ldcg(b1 + k); };
    auto get2 = [&](int k) { return cached ? s2c[k] : __ldcg(b2 + k); };
    double total = 0.0;
    {
        double v = 0.0;
        for (int k = tid; k < NR2; k += kSeedThreads) v += get2(k);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
        __syncthreads();
        if (lane == 0) sh[warp] = v;
        __syncthreads();
        for (int w = 0; w < kSeedWarps; ++w) total += sh[w];
    }
    if (total > 0.0) {
        const double thr = ur * total;
        if (tid == 0) pick_blk = 0x7fffffff;
        // the first S2 range whose running sum exceeds thr
        double carry = 0.0;
        for (int c0 = 0; c0 < NR2; c0 += kSeedThreads) {
            const int kk = c0 + tid;
            const double v = kk < NR2 ? get2(kk) : 0.0;
            const double inc = block_scan_d(v, sh) + carry;
            __syncthreads();
            if (kk < NR2 && inc > thr) atomicMin(&pick_blk, kk);
            if (tid == kSeedThreads - 1) sh[0] = inc;  // carry into the next chunk
            __syncthreads();
            carry = sh[0];
            if (kk == pick_blk) sh_base = inc - v;  // exclusive running sum
            __syncthreads();
        }
        const int k2 = pick_blk;
        const double base2 = sh_base;
        __syncthreads();
        if (warp == 0) {
            // then the S1 range, then the point; at either level, when
            // rounding keeps the running sum at or below thr inside the
            // chosen range, its last element with positive mass is taken
            int pk = -1;
            if (k2 != 0x7fffffff) {
                const int k = k2 * kSeedS + lane;
                const double v1 = k < NR1 ? get1(k) : 0.0;
                const double inc1 = warp_scan_d(v1, lane);
                const unsigned cr1 = __ballot_sync(0xffffffffu, k < NR1 && base2 + inc1 > thr);
                const unsigned pos1 = __ballot_sync(0xffffffffu, v1 > 0.0);
                const int l1 = cr1 ? __ffs(cr1) - 1 : (pos1 ? 31 - __clz(pos1) : -1);
                if (l1 >= 0) {
                    const double b1x = base2 + __shfl_sync(0xffffffffu, inc1 - v1, l1);
                    const bool exact1 = cr1 != 0u;
                    const int i = (k2 * kSeedS + l1) * kSeedS + lane;
                    const double v0 = i < N ? __ldcg(d2h + i) : 0.0;
                    if (i < N) {
                        // the candidates' rows into L1, for the centre record
#pragma unroll
                        for (int ln = 0; ln < D * (int)sizeof(T) / 128; ++ln)
                            asm volatile("prefetch.global.L1 [%0];" ::"l"(xh + (size_t)i * D + ln * (128 / sizeof(T))));
                    }
                    const double inc0 = warp_scan_d(v0, lane);
                    const unsigned cr0 = exact1 ? __ballot_sync(0xffffffffu, i < N && b1x + inc0 > thr) : 0u;
                    const unsigned pos0 = __ballot_sync(0xffffffffu, v0 > 0.0);
                    const int l0 = cr0 ? __ffs(cr0) - 1 : (pos0 ? 31 - __clz(pos0) : -1);
                    if (l0 >= 0) pk = (k2 * kSeedS + l1) * kSeedS + l0;
                }
            }
            if (lane == 0) pick_blk = pk;
        }
        __syncthreads();
        if (pick_blk < 0) {
            // no range crossed thr (rounding with u near 1): the last point
            // with D2 > 0
            __syncthreads();
            if (tid == 0) pick_blk = -1;
            __syncthreads();
            for (int i = N - 1 - tid; i >= 0; i -= kSeedThreads) {
                if (__ldcg(d2h + i) > 0.0) {
                    atomicMax(&pick_blk, i);
                    break;
                }
            }
            __syncthreads();
            if (tid == 0 && pick_blk < 0) pick_blk = 0;
            __syncthreads();
        }
    } else {
        // every remaining point coincides with a centre: the smallest unchosen index
        if (tid == 0) pick_blk = 0x7fffffff;
        __syncthreads();
        for (int i = tid; i < N; i += kSeedThreads)
            if (!__ldcg(tk + i)) {
                atomicMin(&pick_blk, i);
                break;
            }
        __syncthreads();
        if (tid == 0 && pick_blk == 0x7fffffff) pick_blk = 0;
        __syncthreads();
    }
    if (warp == 0) {
        const int pk = pick_blk;
        if (lane == 0) {
            s.idx[(size_t)h * K + r] = pk;
            tk[pk] = 1;
            s.cnt[h] = 0;
        }
        seed_write_centre<T, D>(xh, pk, rec, lane);
    }
}

// ---- rounds before the first grouping: every point is updated, and each
// range of positions [p0, p1) (a multiple of the S2 range, or the tail) gets
// its S1 and S2 sums written by the block that updated it.
// SCREEN: test each point first with the fp32 distance (worth it once few
// points change per round; without it the kernel needs fewer registers).
template <typename T, int D, bool SCREEN>
__device__ __forceinline__ void seed_full_range(const T *__restrict__ x, const SeedArgs &s, int h, int r, int p0,
                                                int p1, double *s1own) {
    using Gm = SeedGeo<T, D>;
    const int N = s.N, K = s.K;
    const size_t hN = (size_t)h * N;
    const T *xh = x + hN * D;
    double *d2h = s.d2 + hN;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the previous round's centre, from its record
    const uint4 craw = __ldcg(reinterpret_cast<const uint4 *>(s.cen + (size_t)h * kSeedCenBytes) + lane % Gm::LPP);
    double cv[Gm::E16];
    float cvf[Gm::E16];
    widen16<T>(craw, cv);
    widen16f<T>(craw, cvf);
    (void)cvf;
    const int q = seed_row<T, D>(lane);
    double *b1 = s.bs1 + (size_t)h * s.NR1;
    (void)K;
    const int k0 = p0 / kSeedS, k1 = (p1 + kSeedS - 1) / kSeedS;
    for (int base = p0 + warp * 32; base < p1; base += kSeedWarps * 32) {
        const int qp = base + lane;
        const unsigned m = __ballot_sync(0xffffffffu, qp < p1);
        uint4 buf[Gm::LPP];
        load32<T, D, true>(xh, qp, m, lane, buf);
        const int i = base + q;
        const bool mine = (m >> q) & 1u;
        const double old = mine ? d2h[i] : 0.0;
        double fin = old;  // the point's D2 after this round (0 past p1)
        // fp32 screen, then the exact distance where D2 may fall (the
        // rows are read again, from cache, for the rare warps that need it)
        if constexpr (SCREEN) {
            const float d32 = dist32f<T, D>(buf, cvf, lane);  // every lane: it shuffles
            const bool cand = mine && seed_may_fall(d32, old);
            if (__any_sync(0xffffffffu, cand)) {
                uint4 buf2[Gm::LPP];
                load32<T, D, false>(xh, qp, m, lane, buf2);
                const double dist = dist32<T, D>(buf2, cv, lane);
                if (cand && dist < old) {
                    d2h[i] = dist;
                    s.near[hN + i] = r - 1;
                    fin = dist;
                }
            }
        } else {
            const double dist = dist32<T, D>(buf, cv, lane);
            if (mine && dist < old) {
                d2h[i] = dist;
                s.near[hN + i] = r - 1;
                fin = dist;
            }
        }
        // the S1 sum of these 32 points (base is a multiple of 32), in index
        // order from the registers: point j is in lane (j % PPL) LPP + j / PPL
        double v = 0.0;
#pragma unroll
        for (int j = 0; j < kSeedS; ++j)
            v += __shfl_sync(0xffffffffu, fin, (j % Gm::PPL) * Gm::LPP + j / Gm::PPL);
        if (lane == 0) {
            b1[base / kSeedS] = v;
            s1own[base / kSeedS - k0] = v;
        }
    }
    __syncthreads();
    const int m0 = k0 / kSeedS, m1 = (k1 + kSeedS - 1) / kSeedS;
    for (int k2 = m0 + tid; k2 < m1; k2 += kSeedThreads) {
        const int a0 = k2 * kSeedS, a1 = min(s.NR1, a0 + kSeedS);
        double v = 0.0;
        for (int k = a0; k < a1; ++k) v += s1own[k - k0];
        s.bs2[(size_t)h * s.NR2 + k2] = v;
    }
}

// One block per range of ch positions of head blockIdx.y (round 0 clears
// the state).
template <typename T, int D, bool SCREEN>
__global__ void __launch_bounds__(kSeedThreads)
kmeanspp_round_full(const T *__restrict__ x, const SeedArgs s, int r, int ch) {
    const int h = blockIdx.y, N = s.N;
    const size_t hN = (size_t)h * N;
    double *d2h = s.d2 + hN;
    __shared__ double s1own[kSeedChMax / kSeedS];
    const int tid = threadIdx.x;
    const int p0 = blockIdx.x * ch;
    const int p1 = min(N, p0 + ch);
    pdl_wait();
    pdl_launch_dependents();
    if (r == 0) {
        // round 0: clear the state; the last block records floor(u * N)
        unsigned char *dh = s.dirty + (size_t)h * s.DSTRIDE;
        for (int i = p0 + tid; i < p1; i += kSeedThreads) {
            d2h[i] = __longlong_as_double(0x7ff0000000000000LL);  // +inf
            s.taken[hN + i] = 0;
            s.near[hN + i] = 0;
        }
        for (int k = p0 / kSeedS + tid; k < (p1 + kSeedS - 1) / kSeedS; k += kSeedThreads) dh[k] = 0;
    } else {
        seed_full_range<T, D, SCREEN>(x, s, h, r, p0, p1, s1own);
    }
    seed_arrive_pick<false, T, D>(x, s, h, r, gridDim.x, nullptr, nullptr);
}

// The same rounds (r >= 1) with the work handed out dynamically: the grid is
// the blocks that fit the GPU at once, and each block takes the next S2 range
// of positions (1024; head-major order) from the round's counter until none
// is left.  A static split left blocks idle while others still worked (the
// blocks of one round ended 76-136 us after its start; their fp64 rechecks
// and their SM's share differ), and each head now waits only for its last
// range.  The block that completes a head's last range picks for it.
template <typename T, int D, bool SCREEN>
__global__ void __launch_bounds__(kSeedThreads)
kmeanspp_round_full_dyn(const T *__restrict__ x, const SeedArgs s, int r, int H) {
    constexpr int kChunk = kSeedS * kSeedS;
    __shared__ double s1own[kSeedS];
    __shared__ int next_item;
    const int N = s.N, nch = (N + kChunk - 1) / kChunk, total = nch * H;
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) next_item = atomicAdd(&s.ctr[r], 1);
    __syncthreads();
    int it = next_item;
    while (it < total) {
        __syncthreads();  // every thread has read next_item
        // the following range, in flight while this one is updated
        if (threadIdx.x == 0) next_item = atomicAdd(&s.ctr[r], 1);
        const int h = it / nch, p0 = (it - h * nch) * kChunk;
        seed_full_range<T, D, SCREEN>(x, s, h, r, p0, min(N, p0 + kChunk), s1own);
        seed_arrive_pick<false, T, D>(x, s, h, r, nch, nullptr, nullptr);
        __syncthreads();
        it = next_item;
    }
}

// ---- grouped rounds (pruned update)
//
// pre = the grouping may be read before the dependency wait (it was not just
// rebuilt).  Dynamic shared memory, ch positions: point at each position
// (then the dirty S1 ranges), the active positions (piece << 16 | offset),
// the piece bounds (float bits), the piece flags (then the S2 dirty bitmap).
constexpr size_t seed_grouped_smem(int ch) { return (size_t)13 * ch + 16; }

template <typename T, int D>
__global__ void __launch_bounds__(kSeedThreads)
kmeanspp_round_grouped(const T *__restrict__ x, const SeedArgs s, int r, int G, int pre, int ch) {
    using Gm = SeedGeo<T, D>;
    constexpr int L8 = Q8<D>::L8, R8 = Q8<D>::R8;
    const int h = blockIdx.y, b = blockIdx.x, N = s.N, K = s.K;
    const size_t hN = (size_t)h * N, hK = (size_t)h * K;
    const T *xh = x + hN * D;
    double *d2h = s.d2 + hN;
    unsigned char *dh = s.dirty + (size_t)h * s.DSTRIDE;
    extern __shared__ __align__(16) unsigned char seed_smem[];
    int *pperm = reinterpret_cast<int *>(seed_smem);
    uint32_t *alist = reinterpret_cast<uint32_t *>(pperm + ch);
    uint32_t *pmax = alist + ch;
    unsigned char *act = reinterpret_cast<unsigned char *>(pmax + ch + 1);
    __shared__ int npc, na;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p0 = b * ch;
    const int p1 = min(N, p0 + ch);
    const size_t rec = (size_t)h * s.CAP + (size_t)b * (ch + 1);
    (void)G;

    // ---- the block's pieces and the first 256 of them (static data)
    int P = 0, gl = 0, lol = 0, hil = 0, nv = 0;
    float Rv = 0.f, sv = 1.f, ev = 0.f;
    uint4 abuf[L8];
    auto fetch = [&](int pass) {
        const int jl = pass * kSeedThreads + warp * 32 + lane;
        const bool have = jl < P;
        gl = have ? s.pg[rec + jl] : 0;
        lol = have ? s.plo[rec + jl] : 0;
        hil = have ? s.phi[rec + jl] : 0;
        Rv = have ? s.gr[hK + gl] : 0.f;
        sv = have ? s.gs[hK + gl] : 1.f;
        ev = have ? s.ge[hK + gl] : 0.f;
        nv = have ? s.gn[hK + gl] : 0;
        const unsigned am = __ballot_sync(0xffffffffu, have);
#pragma unroll
        for (int i = 0; i < L8; ++i) {
            const int row = i * R8 + lane / L8;
            const int gi = __shfl_sync(0xffffffffu, gl, row);
            abuf[i] = ((am >> row) & 1u)
                          ? __ldg(reinterpret_cast<const uint4 *>(s.gq + (hK + gi) * D + (lane % L8) * 16))
                          : make_uint4(0, 0, 0, 0);
        }
    };
    auto stage = [&]() {
        if (tid == 0) npc = s.pcnt[(size_t)h * s.NBMAX + b];
        for (int o = tid; o < p1 - p0; o += kSeedThreads) pperm[o] = s.perm[hN + p0 + o];
        __syncthreads();
        P = npc;
        fetch(0);
    };
    if (pre) stage();
    pdl_wait();
    pdl_launch_dependents();
    if (!pre) stage();
    if (tid == 0) na = 0;

    // the previous round's centre and its int8 copy, from its record
    const unsigned char *cenr = s.cen + (size_t)h * kSeedCenBytes;
    const uint4 craw = __ldcg(reinterpret_cast<const uint4 *>(cenr) + lane % Gm::LPP);
    double cv[Gm::E16];
    float cvf[Gm::E16];
    widen16<T>(craw, cv);
    widen16f<T>(craw, cvf);
    const uint4 qc = __ldcg(reinterpret_cast<const uint4 *>(cenr + kSeedCenCodes) + lane % L8);
    const float sc = __ldcg(reinterpret_cast<const float *>(cenr + kSeedCenScal));
    const int nqc = __ldcg(reinterpret_cast<const int *>(cenr + kSeedCenScal) + 1);
    const float ec = __ldcg(reinterpret_cast<const float *>(cenr + kSeedCenScal) + 2);
    __syncthreads();  // na cleared

    // triangle test of each piece, then its positions into the active list
    for (int pass = 0; pass * kSeedThreads < P; ++pass) {
        if (pass > 0) fetch(pass);
        const int jl = pass * kSeedThreads + warp * 32 + lane;
        const bool have = jl < P;
        const float Mv = have ? s.pm[rec + jl] : 0.f;
        const int dq = dot32q<D>(abuf, qc, lane);
        const int dot = __shfl_sync(0xffffffffu, dq, q8_lane<D>(lane));  // this lane's piece
        bool upd = false;
        if (have) {
            const double sa = sv, scd = sc;
            const double dc2 = scd * scd * (double)nqc + sa * sa * (double)nv - 2.0 * scd * sa * (double)dot;
            const double lb = sqrt(fmax(dc2, 0.0)) - (double)ec - (double)ev;
            const double slack = 1e-7 * (scd * sqrt((double)nqc) + sa * sqrt((double)nv));
            upd = !(lb > ((double)Rv + (double)Mv) * (1.0 + kSeedMargin) + slack);
            act[jl] = upd ? 1 : 0;
            if (upd) pmax[jl] = 0u;
        }
        unsigned bal = __ballot_sync(0xffffffffu, upd);
        while (bal) {
            const int src = __ffs(bal) - 1;
            bal &= bal - 1;
            const int lo = __shfl_sync(0xffffffffu, lol, src);
            const int len = __shfl_sync(0xffffffffu, hil, src) - lo;
            const uint32_t jj = (uint32_t)(pass * kSeedThreads + warp * 32 + src);
            int start = 0;
            if (lane == 0) start = atomicAdd(&na, len);
            start = __shfl_sync(0xffffffffu, start, 0);
            for (int t = lane; t < len; t += 32) alist[start + t] = (jj << 16) | (uint32_t)(lo + t);
        }
    }
    __syncthreads();

    // D2 update of the active positions, 32 at a time per warp
    const int nact = na;
    const int q = seed_row<T, D>(lane);
    for (int base = warp * 32; base < nact; base += kSeedThreads) {
        const int k = base + lane;
        const bool al = k < nact;
        const uint32_t e = al ? alist[k] : 0u;
        const unsigned m = __ballot_sync(0xffffffffu, al);
        const int pt = al ? pperm[e & 0xffffu] : 0;
        uint4 buf[Gm::LPP];
        load32<T, D, true>(xh, pt, m, lane, buf);
        const int i = __shfl_sync(0xffffffffu, pt, q);
        const uint32_t eq = __shfl_sync(0xffffffffu, e, q);
        const bool mine = (m >> q) & 1u;
        const double old = mine ? d2h[i] : 0.0;
        // fp32 screen, then the exact distance where D2 may fall
        const float d32 = dist32f<T, D>(buf, cvf, lane);  // every lane: it shuffles
        const bool cand = mine && seed_may_fall(d32, old);
        double nd = old;
        if (__any_sync(0xffffffffu, cand)) {
            uint4 buf2[Gm::LPP];
            load32<T, D, false>(xh, pt, m, lane, buf2);
            const double dist = dist32<T, D>(buf2, cv, lane);
            if (cand && dist < old) {
                nd = dist;
                d2h[i] = nd;
                s.near[hN + i] = r - 1;
                dh[i / kSeedS] = 1;
            }
        }
        if (mine) atomicMax(&pmax[eq >> 16], __float_as_uint(__double2float_ru(sqrt(nd))));
    }
    __syncthreads();
    for (int j = tid; j < P; j += kSeedThreads)
        if (act[j]) s.pm[rec + j] = __uint_as_float(pmax[j]);
    // the piece lists (alist, pmax: 8 ch bytes) hold the S1 and S2 sums in the pick
    seed_arrive_pick<true, T, D>(x, s, h, r, gridDim.x, pperm, reinterpret_cast<uint32_t *>(act),
                           reinterpret_cast<double *>(alist), ch);
}

// ---- regrouping (before round r, with G = r - 1 chosen centres applied)
//
// Group g holds the points whose nearest applied centre is centre g; its
// radius is the largest of their D2 (D2 is exactly the distance to that
// centre).  Counting sort (histogram and radius, exclusive scan, scatter),
// the int8 copy of every anchor, then each block's piece records.

__global__ void seed_group_hist(const SeedArgs s, int G) {
    const int h = blockIdx.y, i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= s.N) return;
    const size_t hi = (size_t)h * s.N + i;
    const int g = s.near[hi];
    atomicAdd(&s.gcnt[(size_t)h * G + g], 1);
    atomicMax(reinterpret_cast<unsigned long long *>(s.r2 + (size_t)h * G + g),
              (unsigned long long)__double_as_longlong(s.d2[hi]));
}

// key: the group of each point ([H][N]: the nearest chosen centre, or the
// nearest static anchor)
__global__ void seed_group_scatter(const SeedArgs s, int G, const int32_t *__restrict__ key) {
    const int h = blockIdx.y, i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= s.N) return;
    const size_t hN = (size_t)h * s.N;
    const int g = key[hN + i];
    const int pos = atomicAdd(&s.cur[(size_t)h * G + g], 1);
    s.perm[hN + pos] = i;
}

// Static groups: the anchors' rows (point j N / A of each head), gathered
// for the assignment.
template <typename T, int D>
__global__ void seed_gather_anchors(const T *__restrict__ x, const SeedArgs s) {
    const int h = blockIdx.y, j = blockIdx.x, A = s.A;
    const int ai = (int)((long long)j * s.N / A);
    const T *src = x + ((size_t)h * s.N + ai) * D;
    T *dst = static_cast<T *>(s.anc) + ((size_t)h * A + j) * D;
    for (int e = threadIdx.x; e < D; e += blockDim.x) dst[e] = src[e];
}

// |row - its anchor|^2 (fp64) of the 32 rows load32 read into buf, whose
// anchors' rows (loaded the same way) are in abuf: lane l ends with row
// seed_row(l).
template <typename T, int D>
__device__ __forceinline__ double dist32_pair(const uint4 (&buf)[SeedGeo<T, D>::LPP],
                                              const uint4 (&abuf)[SeedGeo<T, D>::LPP], int lane) {
    using G = SeedGeo<T, D>;
    double part[G::LPP];
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        double xv[G::E16], av[G::E16];
        widen16<T>(buf[i], xv);
        widen16<T>(abuf[i], av);
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < G::E16; ++e) {
            const double t = xv[e] - av[e];
            acc = fma(t, t, acc);
        }
        part[i] = acc;
    }
#pragma unroll
    for (int n = G::LPP; n > 1; n >>= 1) {
        const int half = n >> 1;
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const double send = up ? part[k] : part[k + half];
            const double keep = up ? part[k + half] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return part[0];
}

// Static groups: member counts and R^2 = the largest |x - anchor|^2 (fp64)
// of each group, 32 points per warp.
template <typename T, int D>
__global__ void seed_group_hist_static(const T *__restrict__ x, const SeedArgs s) {
    const int h = blockIdx.y, N = s.N, A = s.A, lane = threadIdx.x & 31;
    const int base = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
    if (base >= N) return;
    const size_t hN = (size_t)h * N;
    const T *xh = x + hN * D;
    const int i = base + lane;
    const unsigned m = __ballot_sync(0xffffffffu, i < N);
    const int g = i < N ? s.skey[hN + i] : 0;
    const int ai = (int)((long long)g * N / A);
    uint4 buf[SeedGeo<T, D>::LPP], abuf[SeedGeo<T, D>::LPP];
    load32<T, D, true>(xh, i, m, lane, buf);
    load32<T, D, false>(xh, ai, m, lane, abuf);
    const double d2 = dist32_pair<T, D>(buf, abuf, lane);
    const int q = seed_row<T, D>(lane);
    const int gq = __shfl_sync(0xffffffffu, g, q);  // this lane's distance is point base + q's
    if ((m >> q) & 1u) {
        atomicAdd(&s.gcnt[(size_t)h * A + gq], 1);
        atomicMax(reinterpret_cast<unsigned long long *>(s.r2 + (size_t)h * A + gq),
                  (unsigned long long)__double_as_longlong(d2));
    }
}

// One warp per group: int8 anchor, scale, |codes|^2, error and R.  The
// anchor is chosen centre g, or with static groups the point g N / G.
template <typename T, int D>
__global__ void seed_group_anchor(const T *__restrict__ x, const SeedArgs s, int G, int is_static) {
    const int h = blockIdx.y, lane = threadIdx.x & 31;
    const int g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (g >= G) return;
    const size_t hK = (size_t)h * s.K;
    const int ai = is_static ? (int)((long long)g * s.N / G) : s.idx[hK + g];
    float sc, err;
    uint4 codes;
    int n2;
    q8_vector<T, D>(x + ((size_t)h * s.N + ai) * D, lane, sc, codes, n2, err);
    if (lane < Q8<D>::L8) *reinterpret_cast<uint4 *>(s.gq + (hK + g) * D + lane * 16) = codes;
    if (lane == 0) {
        s.gs[hK + g] = sc;
        s.ge[hK + g] = err;
        s.gn[hK + g] = n2;
        s.gr[hK + g] = __double2float_ru(sqrt(s.r2[(size_t)h * G + g]) * (1.0 + kSeedMargin));
    }
}

// One block per range of ch positions: the non-empty parts of the groups
// overlapping it, in group order, with M = R to start (centre groups: R is
// the largest sqrt(D2) of the group), or M = +inf (static groups, whose
// radius says nothing of D2: the first round over them visits every piece
// and records its M).
__global__ void seed_group_pieces(const SeedArgs s, int G, int ch, int is_static) {
    const int h = blockIdx.y, b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p0 = b * ch, p1 = min(s.N, p0 + ch);
    const int *seg = s.seg + (size_t)h * (G + 1);
    const size_t hK = (size_t)h * s.K;
    const size_t rec = (size_t)h * s.CAP + (size_t)b * (ch + 1);
    __shared__ int glo, ghi, base, wsum[kSeedWarps];
    if (tid == 0) {
        // last group starting at or before p0, and at or before p1 - 1
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seg[mid] <= p0) lo = mid; else hi = mid - 1;
        }
        glo = lo;
        lo = 0;
        hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seg[mid] <= p1 - 1) lo = mid; else hi = mid - 1;
        }
        ghi = lo;
        base = 0;
    }
    __syncthreads();
    for (int g0 = glo; g0 <= ghi; g0 += kSeedThreads) {
        const int g = g0 + tid;
        int lo = 0, hi = 0;
        if (g <= ghi) {
            lo = max(seg[g], p0);
            hi = min(seg[g + 1], p1);
        }
        const bool v = g <= ghi && lo < hi;
        const unsigned bl = __ballot_sync(0xffffffffu, v);
        if (lane == 0) wsum[warp] = __popc(bl);
        __syncthreads();
        int off = base;
        for (int w = 0; w < warp; ++w) off += wsum[w];
        off += __popc(bl & ((1u << lane) - 1u));
        if (v) {
            s.pg[rec + off] = g;
            s.plo[rec + off] = (uint16_t)(lo - p0);
            s.phi[rec + off] = (uint16_t)(hi - p0);
            s.pm[rec + off] = is_static ? __int_as_float(0x7f800000) : s.gr[hK + g];
        }
        __syncthreads();
        if (tid == 0) {
            int t = 0;
            for (int w = 0; w < kSeedWarps; ++w) t += wsum[w];
            base += t;
        }
        __syncthreads();
    }
    if (tid == 0) s.pcnt[(size_t)h * s.NBMAX + b] = base;
}

// ================================================ batched k-means++ seeding ==
//
// Up to b draws per round from one D2 distribution, repeats within a round
// dropped, then one D2 update with all the round's centres (the batched
// seeding of k-means||, Bahmani et al. 2012, without its reclustering): about
// K / b rounds instead of K.  A round starts with the pick (one CTA per head:
// the S2 sums of the S1 sums and their prefix, the draws' inverse-CDF
// searches over S2 / S1 / point, the kept centres gathered).  For bf16 with
// d = 128 one fused kernel then does the rest (bseed_round_tc in
// assign_tc.cu: tensor-core nearest centre, screened exact D2 update, S1
// sums); otherwise the assignment kernel finds each point's nearest centre
// of the round and bseed_update sets D2 = min(D2, exact fp64 distance to it)
// and the S1 sums (32 points each, index order).  Heads that have all K
// centres skip their work.

struct BSeedArgs {
    const double *u;        // [H][U] draws
    int32_t *idx;           // [H][K] picks
    double *d2;             // [H][N]
    double *bs1;            // [H][NR1] sums of D2 over 32-point ranges (index order)
    float *xn;              // [H][N] |x|^2 (fp32), or null where no round uses it
    unsigned char *taken;   // [H][N]
    int *st;                // [H][4]: centres chosen, draws used, kept this round
    int32_t *key;           // [H][N] nearest centre of the round
    void *cb;               // [H][B][D] the round's centres (storage type)
    __nv_bfloat16 *cbias;   // [H][B][16] bf16 parts of -|c|^2 / 2 (fused rounds), or null
    int *err;
    int N, K, B, U, NR1, NR2;
};

// Round 0: the point floor(u * N) of each head, and D2 to it.
template <typename T, int D>
__global__ void __launch_bounds__(kSeedThreads)
bseed_first(const T *__restrict__ x, const BSeedArgs a) {
    using Gm = SeedGeo<T, D>;
    const int h = blockIdx.y, N = a.N, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t hN = (size_t)h * N;
    const T *xh = x + hN * D;
    int first = (int)floor(a.u[(size_t)h * a.U] * (double)N);
    first = min(max(first, 0), N - 1);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        a.idx[(size_t)h * a.K] = first;
        a.taken[hN + first] = 1;
        a.st[4 * h] = 1;
        a.st[4 * h + 1] = 1;
        a.st[4 * h + 2] = 0;
    }
    const uint4 craw = __ldg(reinterpret_cast<const uint4 *>(xh + (size_t)first * D + (lane % Gm::LPP) * Gm::E16));
    double cv[Gm::E16];
    widen16<T>(craw, cv);
    const int q = seed_row<T, D>(lane);
    const int base = (blockIdx.x * kSeedWarps + warp) * 32;
    if (base >= N) return;
    const int i = base + lane;
    const unsigned m = __ballot_sync(0xffffffffu, i < N);
    uint4 buf[Gm::LPP];
    load32<T, D, true>(xh, i, m, lane, buf);
    const double dist = dist32<T, D>(buf, cv, lane);
    if ((m >> q) & 1u) a.d2[hN + base + q] = dist;
    if (a.xn != nullptr) {
        const float nrm = sumsq32<T, D>(buf, lane);
        if ((m >> q) & 1u) a.xn[hN + base + q] = nrm;
    }
}

// S1 sums (32 points) of every head, index order.
__global__ void __launch_bounds__(kSeedThreads)
bseed_sums(const BSeedArgs a) {
    const int h = blockIdx.y, N = a.N;
    const double *d2h = a.d2 + (size_t)h * N;
    const int k = blockIdx.x * kSeedThreads + threadIdx.x;  // S1 range
    if (k < a.NR1) {
        double v = 0.0;
        const int q0 = k * kSeedS, q1 = min(N, q0 + kSeedS);
        for (int i = q0; i < q1; ++i) v += __ldcg(d2h + i);
        a.bs1[(size_t)h * a.NR1 + k] = v;
    }
}

constexpr int kBSeedMaxB = kSeedThreads;        // draws per round (one per thread)
constexpr int kBSeedMaxNR2 = 2048;              // S2 prefix in shared memory (N <= 2^21)

// Inverse CDF of one draw (threshold thr in (0, total)): the S2 range whose
// prefix first exceeds thr, then the S1 range, then the point, each a running
// sum in index order from the range's base; where rounding keeps a range's
// running sum at or below thr, its last element with positive mass is taken.
__device__ int bseed_search(const BSeedArgs &a, int h, const double *S2, const double *P2, double thr) {
    const int NR1 = a.NR1, NR2 = a.NR2, N = a.N;
    const double *b1 = a.bs1 + (size_t)h * NR1;
    const double *d2h = a.d2 + (size_t)h * N;
    int lo = 0, hi = NR2;  // first k2 with P2[k2] > thr (NR2 if none)
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (P2[mid] > thr) hi = mid; else lo = mid + 1;
    }
    int k2 = lo;
    bool exact = k2 < NR2;
    if (!exact) {  // the last S2 range with positive mass
        k2 = NR2 - 1;
        while (k2 > 0 && !(S2[k2] > 0.0)) --k2;
    }
    double run = k2 > 0 ? P2[k2 - 1] : 0.0;
    const int s0 = k2 * kSeedS, s1 = min(NR1, s0 + kSeedS);
    double t[kSeedS];
#pragma unroll
    for (int e = 0; e < kSeedS; ++e) t[e] = s0 + e < s1 ? __ldcg(b1 + s0 + e) : 0.0;
    int k1 = -1, lastpos = -1;
#pragma unroll
    for (int e = 0; e < kSeedS; ++e) {
        if (k1 < 0 && s0 + e < s1) {
            if (t[e] > 0.0) lastpos = e;
            if (exact && run + t[e] > thr) k1 = e; else run += t[e];
        }
    }
    if (k1 < 0) {
        exact = false;
        k1 = lastpos < 0 ? 0 : lastpos;
    }
    const int q0 = (s0 + k1) * kSeedS, q1 = min(N, q0 + kSeedS);
#pragma unroll
    for (int e = 0; e < kSeedS; ++e) t[e] = q0 + e < q1 ? __ldcg(d2h + q0 + e) : 0.0;
    int pick = -1;
    lastpos = -1;
#pragma unroll
    for (int e = 0; e < kSeedS; ++e) {
        if (pick < 0 && q0 + e < q1) {
            if (t[e] > 0.0) lastpos = e;
            if (exact && run + t[e] > thr) pick = e; else run += t[e];
        }
    }
    if (pick < 0) pick = lastpos < 0 ? 0 : lastpos;
    return q0 + pick;
}

// One CTA per head: the round's draws, repeats dropped, the kept centres
// appended to the picks and gathered for the assignment (the unused slots
// repeat the first kept centre, which changes no minimum).
template <typename T, int D>
__global__ void __launch_bounds__(kSeedThreads)
bseed_pick(const T *__restrict__ x, const BSeedArgs a) {
    const int h = blockIdx.x, N = a.N, K = a.K, B = a.B, tid = threadIdx.x;
    const size_t hN = (size_t)h * N;
    pdl_launch_dependents();  // the round kernel may set up meanwhile
    __shared__ double S2[kBSeedMaxNR2], P2[kBSeedMaxNR2];
    __shared__ int picks[kBSeedMaxB], keep[kBSeedMaxB], pos[kBSeedMaxB], slotpick[kBSeedMaxB], nkept;
    __shared__ double total_s;
    int *st = a.st + 4 * h;
    const int m = st[0], p = st[1];
    if (m >= K) {
        if (tid == 0) st[2] = 0;
        return;
    }
    const int nb = min(B, K - m);
    // S2 sums (32 S1 sums each, index order) and their prefix
    const double *b1 = a.bs1 + (size_t)h * a.NR1;
    for (int k = tid; k < a.NR2; k += kSeedThreads) {
        const int k0 = k * kSeedS, k1 = min(a.NR1, k0 + kSeedS);
        double w = 0.0;
        for (int kk = k0; kk < k1; ++kk) w += __ldcg(b1 + kk);
        S2[k] = w;
        P2[k] = w;
    }
    __syncthreads();
    if (tid == 0) {
        double r = 0.0;
        for (int k = 0; k < a.NR2; ++k) {
            r += P2[k];
            P2[k] = r;
        }
        total_s = r;
    }
    __syncthreads();
    const double total = total_s;
    for (int j = tid; j < nb; j += kSeedThreads) {
        const double uj = a.u[(size_t)h * a.U + (p + j) % a.U];
        int pick;
        if (total > 0.0) {
            pick = bseed_search(a, h, S2, P2, uj * total);
        } else {
            // every remaining point coincides with a centre: the j-th
            // smallest index not yet chosen
            pick = 0;
            int seen = 0;
            for (int i = 0; i < N; ++i)
                if (!a.taken[hN + i]) {
                    if (seen == j) {
                        pick = i;
                        break;
                    }
                    ++seen;
                }
        }
        picks[j] = pick;
    }
    __syncthreads();
    for (int j = tid; j < nb; j += kSeedThreads) {
        int k = 1;
        for (int j2 = 0; j2 < j; ++j2)
            if (picks[j2] == picks[j]) k = 0;
        keep[j] = k;
    }
    __syncthreads();
    {
        // positions of the kept draws: a ballot per warp, the warps' counts in order
        // (nb <= kSeedThreads: one draw per thread)
        __shared__ int wcnt[kSeedWarps];
        const int lane = tid & 31, warp = tid >> 5;
        const unsigned bal = __ballot_sync(0xffffffffu, tid < nb && keep[tid]);
        if (lane == 0) wcnt[warp] = __popc(bal);
        __syncthreads();
        int off = 0, c = 0;
        for (int w = 0; w < kSeedWarps; ++w) {
            off += w < warp ? wcnt[w] : 0;
            c += wcnt[w];
        }
        if (tid < nb) pos[tid] = off + __popc(bal & ((1u << lane) - 1u));
        if (tid == 0) {
            nkept = c;
            st[0] = m + c;
            st[1] = p + nb;
            st[2] = c;
        }
    }
    __syncthreads();
    for (int j = tid; j < nb; j += kSeedThreads)
        if (keep[j]) {
            a.idx[(size_t)h * K + m + pos[j]] = picks[j];
            a.taken[hN + picks[j]] = 1;
            slotpick[pos[j]] = picks[j];
        }
    __syncthreads();
    // the round's centres, then copies of the first one
    const int kept = nkept;
    if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
        // one warp per centre, with the three bf16 parts of -|c|^2 / 2 that the
        // fused round adds on the tensor cores (the sums of centroid_norms)
        const int warp = tid >> 5, lane = tid & 31;
        constexpr int kRows = 8;  // rows in flight per warp
        for (int s0 = warp; s0 < B; s0 += kSeedWarps * kRows) {
            uint2 v[kRows];
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                const int slot = s0 + k * kSeedWarps;
                const int src = slot < kept ? slotpick[slot] : picks[0];
                v[k] = slot < B ? __ldg(reinterpret_cast<const uint2 *>(x + (hN + src) * D) + lane) : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                const int slot = s0 + k * kSeedWarps;
                if (slot >= B) break;  // the same for every lane
                reinterpret_cast<uint2 *>(static_cast<T *>(a.cb) + ((size_t)h * B + slot) * D)[lane] = v[k];
                const float f0 = __uint_as_float(v[k].x << 16), f1 = __uint_as_float(v[k].x & 0xFFFF0000u);
                const float f2 = __uint_as_float(v[k].y << 16), f3 = __uint_as_float(v[k].y & 0xFFFF0000u);
                const float sq = warp_sum(fmaf(f3, f3, fmaf(f2, f2, fmaf(f1, f1, f0 * f0))));
                if (lane < 2) {
                    uint4 row = make_uint4(0u, 0u, 0u, 0u);
                    if (lane == 0) {
                        const float bb = -0.5f * sq;
                        const __nv_bfloat16 hi = __float2bfloat16_rn(bb);
                        const float r1 = bb - __bfloat162float(hi);
                        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
                        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
                        row.x = (uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(mid) << 16);
                        row.y = (uint32_t)__bfloat16_as_ushort(lo);
                    }
                    reinterpret_cast<uint4 *>(a.cbias + ((size_t)h * B + slot) * 16)[lane] = row;
                }
            }
        }
    } else {
        constexpr int C16 = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
        uint4 *cbh = reinterpret_cast<uint4 *>(static_cast<T *>(a.cb) + (size_t)h * B * D);
        for (int w = tid; w < B * C16; w += kSeedThreads) {
            const int slot = w / C16, c = w - slot * C16;
            const int src = slot < kept ? slotpick[slot] : picks[0];
            cbh[w] = __ldg(reinterpret_cast<const uint4 *>(x + (hN + src) * D) + c);
        }
    }
}

// D2 = min(D2, |x - the assigned centre of the round|^2) (exact fp64), then
// the S1 sums of this 1024-position range from the registers.
template <typename T, int D>
__global__ void __launch_bounds__(kSeedThreads)
bseed_update(const T *__restrict__ x, const BSeedArgs a) {
    using Gm = SeedGeo<T, D>;
    const int h = blockIdx.y, N = a.N, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (a.st[4 * h + 2] == 0) return;  // no centre this round: D2 and sums stand
    const size_t hN = (size_t)h * N;
    const T *xh = x + hN * D;
    const T *cbh = static_cast<const T *>(a.cb) + (size_t)h * a.B * D;
    double *d2h = a.d2 + hN;
    const int p0 = blockIdx.x * kSeedS * kSeedS, p1 = min(N, p0 + kSeedS * kSeedS);
    const int q = seed_row<T, D>(lane);
    for (int base = p0 + warp * 32; base < p1; base += kSeedWarps * 32) {
        const int i = base + lane;
        const unsigned m = __ballot_sync(0xffffffffu, i < p1);
        const int c = i < p1 ? min(max(a.key[hN + i], 0), a.B - 1) : 0;  // in range even after a give-up
        uint4 buf[Gm::LPP], abuf[Gm::LPP];
        load32<T, D, true>(xh, i, m, lane, buf);
        load32<T, D, false>(cbh, c, m, lane, abuf);
        const double dist = dist32_pair<T, D>(buf, abuf, lane);
        const bool mine = (m >> q) & 1u;
        double fin = mine ? d2h[base + q] : 0.0;
        if (mine && dist < fin) {
            fin = dist;
            d2h[base + q] = dist;
        }
        double v = 0.0;
#pragma unroll
        for (int j = 0; j < kSeedS; ++j)
            v += __shfl_sync(0xffffffffu, fin, (j % Gm::PPL) * Gm::LPP + j / Gm::PPL);
        if (lane == 0) a.bs1[(size_t)h * a.NR1 + base / kSeedS] = v;
    }
}

// After the last round: heads still short of K take the smallest indices not
// yet chosen.
__global__ void bseed_fill(const BSeedArgs a) {
    const int h = blockIdx.x;
    if (threadIdx.x != 0) return;
    int m = a.st[4 * h];
    const size_t hN = (size_t)h * a.N;
    for (int i = 0; m < a.K && i < a.N; ++i)
        if (!a.taken[hN + i]) {
            a.idx[(size_t)h * a.K + m++] = i;
            a.taken[hN + i] = 1;
        }
    a.st[4 * h] = m;
}

}  // namespace asmk

// ============================================================ init / norms ==
namespace asmk {

template <typename T, int D>
__global__ void kmeans_init(const T *__restrict__ x, int N, int K, const int32_t *__restrict__ init_idx,
                            float *centroids, T *centroids_dt) {
    const int h = blockIdx.y;
    const int c = blockIdx.x * (blockDim.x / D) + threadIdx.x / D;
    const int e = threadIdx.x % D;
    if (c >= K) return;
    const int src = init_idx[(size_t)h * K + c];
    const T v = x[((size_t)h * N + src) * D + e];
    centroids[((size_t)h * K + c) * D + e] = Elem<T>::to_f(v);
    centroids_dt[((size_t)h * K + c) * D + e] = v;
}

// |c|^2 of every storage-dtype centre (fp32), one warp per centre; with
// `bias`, also the row [hi, mid, lo, 0 x 13] (bf16) whose first three parts
// sum to -|c|^2 / 2: each part rounds what the earlier ones leave (the
// differences are exact in fp32), so the sum is within 2^-24 of the value.
template <typename T, int D>
__global__ void centroid_norms(const T *__restrict__ c, int HK, float *norms, __nv_bfloat16 *bias) {
    constexpr int EPL = D / 32;
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (w >= HK) return;
    float f[EPL];
    load_vec<T, EPL>(c + (size_t)w * D + lane * EPL, f);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s = fmaf(f[e], f[e], s);
    s = warp_sum(s);
    if (lane == 0) norms[w] = s;
    if (bias != nullptr && lane < 2) {
        uint4 row = make_uint4(0u, 0u, 0u, 0u);
        if (lane == 0) {
            const float b = -0.5f * s;
            const __nv_bfloat16 hi = __float2bfloat16_rn(b);
            const float r1 = b - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            row.x = (uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(mid) << 16);
            row.y = (uint32_t)__bfloat16_as_ushort(lo);
        }
        reinterpret_cast<uint4 *>(bias + (size_t)w * 16)[lane] = row;
    }
}

// ================================================================ assign ===
//
// Portable CUDA-core assignment: a 64-point x 64-centre register-tiled
// fp32 contraction per step, with the arg-max of <x,c> - |c|^2/2 (or
// <x,c>/|c|) carried across all centre tiles; ties go to the smaller index.

constexpr int kAsP = 64, kAsC = 64, kAsDK = 32;

template <typename T, int D>
__global__ void __launch_bounds__(256)
assign_simple(const T *__restrict__ x, const T *__restrict__ c, const float *__restrict__ norms,
              int N, int K, int metric, int32_t *assign) {
    __shared__ float xs[kAsDK][kAsP + 4];
    __shared__ float cs[kAsDK][kAsC + 4];
    __shared__ float bs_s[16][kAsP];
    __shared__ int bi_s[16][kAsP];
    const int h = blockIdx.y;
    const int p0 = blockIdx.x * kAsP;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // ty: points, tx: centres
    const T *xh = x + (size_t)h * N * D;
    const T *ch = c + (size_t)h * K * D;
    float best[4];
    int bidx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { best[i] = kNegInf; bidx[i] = 0x7fffffff; }

    for (int c0 = 0; c0 < K; c0 += kAsC) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int k0 = 0; k0 < D; k0 += kAsDK) {
            __syncthreads();
            for (int i = threadIdx.x; i < kAsP * kAsDK; i += 256) {
                const int row = i / kAsDK, col = i % kAsDK;
                const int p = p0 + row, cc = c0 + row;
                xs[col][row] = p < N ? Elem<T>::to_f(xh[(size_t)p * D + k0 + col]) : 0.f;
                cs[col][row] = cc < K ? Elem<T>::to_f(ch[(size_t)cc * D + k0 + col]) : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < kAsDK; ++kk) {
                float xv[4], cv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) cv[j] = cs[kk][tx + 16 * j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], cv[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cc = c0 + tx + 16 * j;
            if (cc >= K) continue;
            const float nr = norms[(size_t)h * K + cc];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float s;
                if (metric == 0) s = acc[i][j] - 0.5f * nr;
                else s = nr > 0.f ? acc[i][j] / sqrtf(nr) : 0.f;
                if (better(s, cc, best[i], bidx[i])) { best[i] = s; bidx[i] = cc; }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        bs_s[tx][ty * 4 + i] = best[i];
        bi_s[tx][ty * 4 + i] = bidx[i];
    }
    __syncthreads();
    if (threadIdx.x < kAsP) {
        const int p = p0 + threadIdx.x;
        float bs = kNegInf;
        int bi = 0x7fffffff;
        for (int t = 0; t < 16; ++t)
            if (better(bs_s[t][threadIdx.x], bi_s[t][threadIdx.x], bs, bi)) {
                bs = bs_s[t][threadIdx.x];
                bi = bi_s[t][threadIdx.x];
            }
        if (p < N) assign[(size_t)h * N + p] = (bi == 0x7fffffff) ? 0 : bi;
    }
}

// ================================================================ update ===
//
// Counting sort of the points by cluster (histogram, exclusive scan, scatter,
// then each cluster's member list put in ascending index order), followed
// by the fp32 mean of each cluster's members in that order.

__global__ void hist_kernel(const int32_t *__restrict__ assign, int H, int N, int K, int32_t *counts) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)H * N) return;
    const int h = (int)(i / N);
    atomicAdd(&counts[(size_t)h * K + assign[i]], 1);
}

// Exclusive scan of counts[h, 0:K) into seg_off[h, 0:K] (one block per head)
// and a copy of the offsets into the scatter cursors.
__global__ void scan_kernel(const int32_t *__restrict__ counts, int K, int32_t *seg_off, int32_t *cursor) {
    const int h = blockIdx.x;
    __shared__ int warp_tot[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < K; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < K ? counts[(size_t)h * K + i] : 0;
        int x = v;
        for (int m = 1; m < 32; m <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, m);
            if (lane >= m) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            for (int m = 1; m < 32; m <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, t, m);
                if (lane >= m) t += y;
            }
            warp_tot[lane] = t;  // inclusive prefix of warp totals
        }
        __syncthreads();
        const int excl = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
        if (i < K) {
            seg_off[(size_t)h * (K + 1) + i] = excl;
            cursor[(size_t)h * K + i] = excl;
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) seg_off[(size_t)h * (K + 1) + K] = carry;
}

__global__ void scatter_kernel(const int32_t *__restrict__ assign, int H, int N, int K, int32_t *cursor,
                               int32_t *perm) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)H * N) return;
    const int h = (int)(i / N), p = (int)(i % N);
    const int pos = atomicAdd(&cursor[(size_t)h * K + assign[i]], 1);
    perm[(size_t)h * N + pos] = p;
}

// Put every cluster's member list in ascending order (insertion sort; the
// lists are short, about N / K entries).
__global__ void segsort_kernel(const int32_t *__restrict__ seg_off, int H, int N, int K, int32_t *perm) {
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (size_t)H * K) return;
    const int h = (int)(t / K), c = (int)(t % K);
    int32_t *p = perm + (size_t)h * N;
    const int lo = seg_off[(size_t)h * (K + 1) + c], hi = seg_off[(size_t)h * (K + 1) + c + 1];
    for (int i = lo + 1; i < hi; ++i) {
        const int v = p[i];
        int j = i - 1;
        while (j >= lo && p[j] > v) { p[j + 1] = p[j]; --j; }
        p[j + 1] = v;
    }
}

// One warp per cluster: fp32 mean of its members (member order), or the
// previous centre if empty; writes the fp32 master and its storage copy.
template <typename T, int D>
__global__ void means_kernel(const T *__restrict__ x, const int32_t *__restrict__ perm,
                             const int32_t *__restrict__ seg_off, int H, int N, int K,
                             float *centroids, T *centroids_dt) {
    constexpr int EPL = D / 32;
    const size_t w = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (size_t)H * K) return;
    const int h = (int)(w / K), c = (int)(w % K);
    const int lo = seg_off[(size_t)h * (K + 1) + c], hi = seg_off[(size_t)h * (K + 1) + c + 1];
    float acc[EPL];
    float *cm = centroids + w * D + lane * EPL;
    if (hi > lo) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        for (int i = lo; i < hi; ++i) {
            const int p = perm[(size_t)h * N + i];
            float f[EPL];
            load_vec<T, EPL>(x + ((size_t)h * N + p) * D + lane * EPL, f);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] += f[e];
        }
        const float inv = 1.f / (float)(hi - lo);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] *= inv;
    } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = cm[e];
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) cm[e] = acc[e];
    store_vec<T, EPL>(centroids_dt + w * D + lane * EPL, acc);
}

// Lloyd workspace: a 256-byte header whose first int is the error word
// (5 = a tensor-core wait timed out), the |c|^2 of every centre, and the
// scatter cursors.
struct KmWs {
    size_t off_norm, off_cursor, off_bias, total;
};
KmWs km_ws(int H, int N, int K) {
    (void)N;
    KmWs w;
    w.off_norm = 256;
    w.off_cursor = al256(w.off_norm + sizeof(float) * (size_t)H * K);
    w.off_bias = al256(w.off_cursor + sizeof(int) * (size_t)H * K);   // [H][K][16] bf16
    w.total = al256(w.off_bias + 32 * (size_t)H * K);
    return w;
}

}  // namespace asmk

// ============================================================== host side ==
using namespace asmk;

size_t asm_kmeanspp_ws_bytes(int H, int N, int d, int K) {
    return seed_ws(H, N, d, K).total;
}

namespace {
// Positions per block: the smallest multiple of `step` (at least kSeedChMin)
// for which every head's blocks fit the GPU in one wave, else kSeedChMax.
template <typename KERN>
int seed_block_positions(KERN k, bool grouped, int step, int H, int N, cudaError_t *err) {
    const size_t smax = grouped ? seed_grouped_smem(kSeedChMax) : 0;
    *err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smax);
    if (*err != cudaSuccess) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    for (int ch = kSeedChMin; ch <= kSeedChMax; ch += step) {
        int occ = 0;
        const size_t sm = grouped ? seed_grouped_smem(ch) : 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kSeedThreads, sm) != cudaSuccess) break;
        if ((long)H * ((N + ch - 1) / ch) <= (long)occ * sms) return ch;
    }
    (void)cudaGetLastError();
    return kSeedChMax;
}

// Blocks of kernel k (kSeedThreads, no dynamic shared memory) resident on the GPU at once.
template <typename KERN>
int seed_resident(KERN k, cudaError_t *err) {
    int occ = 0, dev = 0, sms = 0;
    if ((*err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kSeedThreads, 0)) != cudaSuccess ||
        (*err = cudaGetDevice(&dev)) != cudaSuccess ||
        (*err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return 0;
    return std::max(1, occ * sms);
}

template <typename KERN, typename... Args>
cudaError_t seed_launch(KERN k, dim3 grid, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kSeedThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

template <typename T, int D>
cudaError_t seed_all(const T *x, SeedArgs &s, int H, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    const int chf = seed_block_positions(kmeanspp_round_full<T, D, false>, false, kSeedS * kSeedS, H, s.N, &e);
    if (e != cudaSuccess) return e;
    // rounds 1 .. the first grouping: as many blocks as fit the GPU at once,
    // taking S2 ranges of positions dynamically
    const int items = H * ((s.N + kSeedS * kSeedS - 1) / (kSeedS * kSeedS));
    const int rdf = std::min(items, seed_resident(kmeanspp_round_full_dyn<T, D, false>, &e));
    if (e != cudaSuccess) return e;
    const int rds = std::min(items, seed_resident(kmeanspp_round_full_dyn<T, D, true>, &e));
    if (e != cudaSuccess) return e;
    const int chg = seed_block_positions(kmeanspp_round_grouped<T, D>, true, 256, H, s.N, &e);
    if (e != cudaSuccess) return e;
    const int N = s.N, K = s.K;
    const dim3 pgrid((N + 255) / 256, H);
    const dim3 gfull((N + chf - 1) / chf, H), ggrp((N + chg - 1) / chg, H);
    // first regrouping by centres at 3K/16 (at least 256); static groups from
    // a third of max(256, K/8) (measured at the build shape: regrouping at
    // 1024, 1280, 1536, 1792 or 2048 gave 239.8, 232.1, 229.0, 229.9 and
    // 231.9 ms; static groups from round 256, 341 or 448: 230.6, 229.0, 229.5)
    int G = 0, next = std::max(256, (3 * K) / 16);
    const int sstart = std::max(2, std::max(256, K / 8) / 3);
    // no regrouping after round K/4: more groups mean more pieces to test in
    // every round, which cost more than the finer groups save (last
    // regrouping at 1792, 2048, 2560, 3072, 4096 or 7168: 220.2, 219.1,
    // 220.4, 221.6, 224.5 and 228.8 ms)
    const int last = std::max(next, K / 4);
    for (int r = 0; r < K; ++r) {
        int pre = 1;
        if (r == sstart && s.A > 0 && next > sstart) {
            // static groups until the first regrouping by centres (earlier,
            // most points still move each round and the full update is
            // cheaper): each point joins its nearest of A anchors (every
            // (N / A)-th point); R is the exact largest distance to the
            // anchor, M starts at +inf
            const int A = s.A;
            G = A;
            pre = 0;
            seed_gather_anchors<T, D><<<dim3(A, H), 128, 0, st>>>(x, s);
            if ((e = asm_kmeans_assign_launch(x, s.anc, H, N, D, A, 0, ASM_BF16, s.skey, s.aws, 0, st)) != cudaSuccess)
                return e;
            if ((e = cudaMemsetAsync(s.gcnt, 0, sizeof(int) * (size_t)H * A, st)) != cudaSuccess) return e;
            if ((e = cudaMemsetAsync(s.r2, 0, sizeof(double) * (size_t)H * A, st)) != cudaSuccess) return e;
            seed_group_hist_static<T, D><<<dim3((N + 255) / 256, H), 256, 0, st>>>(x, s);
            scan_kernel<<<H, 1024, 0, st>>>(s.gcnt, A, s.seg, s.cur);
            seed_group_scatter<<<pgrid, 256, 0, st>>>(s, A, s.skey);
            seed_group_anchor<T, D><<<dim3((A + 7) / 8, H), 256, 0, st>>>(x, s, A, 1);
            seed_group_pieces<<<ggrp, kSeedThreads, 0, st>>>(s, A, chg, 1);
        }
        if (r == next) {
            // regroup by the nearest of the r - 1 centres applied so far;
            // then again each time the centres grow by a quarter of the
            // largest power of two below r (at least 256 rounds apart), up
            // to round `last`
            G = r - 1;
            pre = 0;
            if ((e = cudaMemsetAsync(s.gcnt, 0, sizeof(int) * (size_t)H * G, st)) != cudaSuccess) return e;
            if ((e = cudaMemsetAsync(s.r2, 0, sizeof(double) * (size_t)H * G, st)) != cudaSuccess) return e;
            seed_group_hist<<<pgrid, 256, 0, st>>>(s, G);
            scan_kernel<<<H, 1024, 0, st>>>(s.gcnt, G, s.seg, s.cur);
            seed_group_scatter<<<pgrid, 256, 0, st>>>(s, G, s.near);
            seed_group_anchor<T, D><<<dim3((G + 7) / 8, H), 256, 0, st>>>(x, s, G, 0);
            seed_group_pieces<<<ggrp, kSeedThreads, 0, st>>>(s, G, chg, 0);
            int p2 = 1;
            while (p2 * 2 <= r) p2 *= 2;
            next = r >= last ? K : r + std::max(256, p2 / 4);
        }
        if (G > 0) e = seed_launch(kmeanspp_round_grouped<T, D>, ggrp, seed_grouped_smem(chg), st, x, s, r, G, pre, chg);
        else if (r == 0) e = seed_launch(kmeanspp_round_full<T, D, false>, gfull, 0, st, x, s, r, chf);
        else if (r < kSeedScreen) e = seed_launch(kmeanspp_round_full_dyn<T, D, false>, dim3(rdf), 0, st, x, s, r, H);
        else e = seed_launch(kmeanspp_round_full_dyn<T, D, true>, dim3(rds), 0, st, x, s, r, H);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}
}  // namespace

cudaError_t asm_kmeanspp_launch(const void *x, int H, int N, int d, int K, const double *u,
                                asm_dtype dt, int32_t *init_idx, void *ws, cudaStream_t st) {
    if (N > kSeedMaxN) return cudaErrorInvalidValue;
    const SeedWs w = seed_ws(H, N, d, K);
    char *b = static_cast<char *>(ws);
    SeedArgs s{};
    s.u = u;
    s.idx = init_idx;
    s.d2 = reinterpret_cast<double *>(b + w.off_d2);
    s.bs1 = reinterpret_cast<double *>(b + w.off_bs1);
    s.bs2 = reinterpret_cast<double *>(b + w.off_bs2);
    s.r2 = reinterpret_cast<double *>(b + w.off_r2);
    s.gs = reinterpret_cast<float *>(b + w.off_gs);
    s.ge = reinterpret_cast<float *>(b + w.off_ge);
    s.gr = reinterpret_cast<float *>(b + w.off_gr);
    s.gn = reinterpret_cast<int32_t *>(b + w.off_gn);
    s.gq = reinterpret_cast<int8_t *>(b + w.off_gq);
    s.near = reinterpret_cast<int32_t *>(b + w.off_near);
    s.perm = reinterpret_cast<int32_t *>(b + w.off_perm);
    s.gcnt = reinterpret_cast<int32_t *>(b + w.off_gcnt);
    s.seg = reinterpret_cast<int32_t *>(b + w.off_seg);
    s.cur = reinterpret_cast<int32_t *>(b + w.off_cur);
    s.pg = reinterpret_cast<int32_t *>(b + w.off_pg);
    s.pm = reinterpret_cast<float *>(b + w.off_pm);
    s.plo = reinterpret_cast<uint16_t *>(b + w.off_plo);
    s.phi = reinterpret_cast<uint16_t *>(b + w.off_phi);
    s.pcnt = reinterpret_cast<int32_t *>(b + w.off_pcnt);
    s.dirty = reinterpret_cast<unsigned char *>(b + w.off_dirty);
    s.taken = reinterpret_cast<unsigned char *>(b + w.off_taken);
    s.cnt = reinterpret_cast<int *>(b + w.off_cnt);
    s.ctr = reinterpret_cast<int *>(b + w.off_ctr);
    s.cen = reinterpret_cast<unsigned char *>(b + w.off_cen);
    s.A = (dt == ASM_BF16) ? w.anchors : 0;
    s.skey = reinterpret_cast<int32_t *>(b + w.off_skey);
    s.anc = b + w.off_anc;
    s.aws = b + w.off_aws;
    s.N = N;
    s.K = K;
    s.NR1 = w.nr1;
    s.NR2 = w.nr2;
    s.DSTRIDE = w.dstride;
    s.NBMAX = w.nbmax;
    s.CAP = w.cap;
    cudaError_t e = cudaMemsetAsync(s.cnt, 0, sizeof(int) * (size_t)H, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s.ctr, 0, sizeof(int) * (size_t)K, st);
    if (e != cudaSuccess) return e;
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        return d == 128 ? seed_all<T, 128>((const T *)x, s, H, st) : seed_all<T, 64>((const T *)x, s, H, st);
    }
    return d == 128 ? seed_all<float, 128>((const float *)x, s, H, st) : seed_all<float, 64>((const float *)x, s, H, st);
}

// ---- batched seeding: workspace and the host loop of rounds
namespace {
struct BSeedWs {
    size_t off_d2, off_bs1, off_xn, off_taken, off_st, off_key, off_cb, off_aws, total;
    int nr1, nr2;
};
BSeedWs bseed_ws(int H, int N, int d, int K, int B) {
    (void)K;
    const size_t h = (size_t)H, n = (size_t)N;
    BSeedWs w;
    w.nr1 = (N + kSeedS - 1) / kSeedS;
    w.nr2 = (w.nr1 + kSeedS - 1) / kSeedS;
    // the assignment's workspace first: its error word (word 0) is this one's
    w.off_aws = 0;
    w.off_d2 = al256(w.off_aws + asm_kmeans_ws_bytes(H, N, d, B));
    w.off_bs1 = al256(w.off_d2 + sizeof(double) * h * n);
    w.off_xn = al256(w.off_bs1 + sizeof(double) * h * w.nr1);
    w.off_taken = al256(w.off_xn + sizeof(float) * h * n);
    w.off_st = al256(w.off_taken + h * n);
    w.off_key = al256(w.off_st + sizeof(int) * 4 * h);
    w.off_cb = al256(w.off_key + sizeof(int32_t) * h * n);
    w.total = al256(w.off_cb + sizeof(float) * h * (size_t)B * d);
    return w;
}

template <typename T, int D>
cudaError_t bseed_all(const T *x, BSeedArgs &a, int H, asm_dtype dt, void *aws, int num_sms, cudaStream_t st) {
    const int N = a.N;
    bseed_first<T, D><<<dim3((N + kSeedThreads - 1) / kSeedThreads, H), kSeedThreads, 0, st>>>(x, a);
    bseed_sums<<<dim3((a.NR1 + kSeedThreads - 1) / kSeedThreads, H), kSeedThreads, 0, st>>>(a);
    const int sms = num_sms;
    auto round = [&]() -> cudaError_t {
        bseed_pick<T, D><<<H, kSeedThreads, 0, st>>>(x, a);
        if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
            // fused: tensor-core nearest centre, screened exact D2 update, S1 sums
            // (the pick wrote the centres' bias parts)
            return asm_bseed_round_tc_launch(x, a.cb, a.cbias, a.xn, a.d2, a.bs1, a.st, H, N, a.B, a.NR1, sms,
                                             a.err, st);
        } else {
            (void)sms;
            cudaError_t e = asm_kmeans_assign_launch(x, a.cb, H, N, D, a.B, 0, dt, a.key, aws, 0, st);
            if (e != cudaSuccess) return e;
            bseed_update<T, D><<<dim3(a.NR2, H), kSeedThreads, 0, st>>>(x, a);
            return cudaGetLastError();
        }
    };
    const int main_rounds = (a.K - 1 + a.B - 1) / a.B;
    cudaError_t e = cudaGetLastError();
    for (int r = 0; r < main_rounds && e == cudaSuccess; ++r) e = round();
    if (e != cudaSuccess) return e;
    // repeated draws leave a head short: up to 16 more rounds while any is
    {
        std::vector<int> hst(4 * (size_t)H);
        for (int extra = 0; extra <= 16; ++extra) {
            if ((e = cudaMemcpyAsync(hst.data(), a.st, sizeof(int) * 4 * (size_t)H, cudaMemcpyDeviceToHost, st)) !=
                    cudaSuccess ||
                (e = cudaStreamSynchronize(st)) != cudaSuccess)
                return e;
            bool short_ = false;
            for (int h = 0; h < H; ++h) short_ |= hst[4 * (size_t)h] < a.K;
            if (!short_) break;
            if (extra == 16) {
                bseed_fill<<<H, 32, 0, st>>>(a);
                break;
            }
            if ((e = round()) != cudaSuccess) return e;
        }
    }
    return cudaGetLastError();
}
}  // namespace

size_t asm_kmeanspp_batched_ws_bytes(int H, int N, int d, int K, int batch) {
    return bseed_ws(H, N, d, K, batch).total;
}

cudaError_t asm_kmeanspp_batched_launch(const void *x, int H, int N, int d, int K, int batch, const double *u,
                                        int U, asm_dtype dt, int32_t *init_idx, void *ws, int num_sms,
                                        cudaStream_t st) {
    const BSeedWs w = bseed_ws(H, N, d, K, batch);
    if (w.nr2 > kBSeedMaxNR2 || batch > kBSeedMaxB) return cudaErrorInvalidValue;
    char *b = static_cast<char *>(ws);
    BSeedArgs a{};
    a.u = u;
    a.idx = init_idx;
    a.d2 = reinterpret_cast<double *>(b + w.off_d2);
    a.bs1 = reinterpret_cast<double *>(b + w.off_bs1);
    const bool fused = dt == ASM_BF16 && d == 128;
    a.xn = fused ? reinterpret_cast<float *>(b + w.off_xn) : nullptr;
    a.cbias = fused ? reinterpret_cast<__nv_bfloat16 *>(b + w.off_aws + km_ws(H, N, batch).off_bias) : nullptr;
    a.taken = reinterpret_cast<unsigned char *>(b + w.off_taken);
    a.st = reinterpret_cast<int *>(b + w.off_st);
    a.key = reinterpret_cast<int32_t *>(b + w.off_key);
    a.cb = b + w.off_cb;
    a.err = reinterpret_cast<int *>(b);
    a.N = N;
    a.K = K;
    a.B = batch;
    a.U = U;
    a.NR1 = w.nr1;
    a.NR2 = w.nr2;
    cudaError_t e = cudaMemsetAsync(a.taken, 0, (size_t)H * N, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        return d == 128 ? bseed_all<T, 128>((const T *)x, a, H, dt, b + w.off_aws, num_sms, st)
                        : bseed_all<T, 64>((const T *)x, a, H, dt, b + w.off_aws, num_sms, st);
    }
    return d == 128 ? bseed_all<float, 128>((const float *)x, a, H, dt, b + w.off_aws, num_sms, st)
                    : bseed_all<float, 64>((const float *)x, a, H, dt, b + w.off_aws, num_sms, st);
}

size_t asm_kmeans_ws_bytes(int H, int N, int d, int K) {
    (void)d;
    return km_ws(H, N, K).total;
}

cudaError_t asm_kmeans_init_launch(const void *x, int H, int N, int d, int K, asm_dtype dt,
                                   const int32_t *init_idx, float *centroids, void *centroids_dt,
                                   cudaStream_t st) {
    const int per_block = 256 / d;
    dim3 grid((K + per_block - 1) / per_block, H);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) kmeans_init<T, 128><<<grid, 256, 0, st>>>((const T *)x, N, K, init_idx, centroids, (T *)centroids_dt);
        else kmeans_init<T, 64><<<grid, 256, 0, st>>>((const T *)x, N, K, init_idx, centroids, (T *)centroids_dt);
    } else {
        if (d == 128) kmeans_init<float, 128><<<grid, 256, 0, st>>>((const float *)x, N, K, init_idx, centroids, (float *)centroids_dt);
        else kmeans_init<float, 64><<<grid, 256, 0, st>>>((const float *)x, N, K, init_idx, centroids, (float *)centroids_dt);
    }
    return cudaGetLastError();
}


cudaError_t asm_kmeans_assign_launch(const void *x, const void *centroids_dt, int H, int N, int d,
                                     int K, int metric, asm_dtype dt, int32_t *assign, void *ws,
                                     int num_sms, cudaStream_t st) {
    (void)num_sms;
    KmWs w = km_ws(H, N, K);
    float *norms = reinterpret_cast<float *>(static_cast<char *>(ws) + w.off_norm);
    const bool tc = dt == ASM_BF16 && d == 128;
    __nv_bfloat16 *bias = (tc && metric == 0)
                              ? reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + w.off_bias) : nullptr;
    const int HK = H * K;
    const int nb = (HK * 32 + 255) / 256;
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) centroid_norms<T, 128><<<nb, 256, 0, st>>>((const T *)centroids_dt, HK, norms, bias);
        else centroid_norms<T, 64><<<nb, 256, 0, st>>>((const T *)centroids_dt, HK, norms, nullptr);
    } else {
        if (d == 128) centroid_norms<float, 128><<<nb, 256, 0, st>>>((const float *)centroids_dt, HK, norms, nullptr);
        else centroid_norms<float, 64><<<nb, 256, 0, st>>>((const float *)centroids_dt, HK, norms, nullptr);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (tc)
        return asm_assign_tc_launch(x, centroids_dt, norms, bias, H, N, K, metric, assign, static_cast<int *>(ws), st);
    dim3 grid((N + kAsP - 1) / kAsP, H);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) assign_simple<T, 128><<<grid, 256, 0, st>>>((const T *)x, (const T *)centroids_dt, norms, N, K, metric, assign);
        else assign_simple<T, 64><<<grid, 256, 0, st>>>((const T *)x, (const T *)centroids_dt, norms, N, K, metric, assign);
    } else {
        if (d == 128) assign_simple<float, 128><<<grid, 256, 0, st>>>((const float *)x, (const float *)centroids_dt, norms, N, K, metric, assign);
        else assign_simple<float, 64><<<grid, 256, 0, st>>>((const float *)x, (const float *)centroids_dt, norms, N, K, metric, assign);
    }
    return cudaGetLastError();
}

cudaError_t asm_kmeans_update_launch(const void *x, const int32_t *assign, int H, int N, int d,
                                     int K, asm_dtype dt, float *centroids, void *centroids_dt,
                                     int32_t *counts, int32_t *perm, int32_t *seg_off, void *ws,
                                     cudaStream_t st) {
    KmWs w = km_ws(H, N, K);
    int32_t *cursor = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.off_cursor);
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)H * K, st);
    if (e != cudaSuccess) return e;
    const size_t HN = (size_t)H * N, HK = (size_t)H * K;
    hist_kernel<<<(unsigned)((HN + 255) / 256), 256, 0, st>>>(assign, H, N, K, counts);
    scan_kernel<<<H, 1024, 0, st>>>(counts, K, seg_off, cursor);
    scatter_kernel<<<(unsigned)((HN + 255) / 256), 256, 0, st>>>(assign, H, N, K, cursor, perm);
    segsort_kernel<<<(unsigned)((HK + 255) / 256), 256, 0, st>>>(seg_off, H, N, K, perm);
    const unsigned nb = (unsigned)((HK * 32 + 255) / 256);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) means_kernel<T, 128><<<nb, 256, 0, st>>>((const T *)x, perm, seg_off, H, N, K, centroids, (T *)centroids_dt);
        else means_kernel<T, 64><<<nb, 256, 0, st>>>((const T *)x, perm, seg_off, H, N, K, centroids, (T *)centroids_dt);
    } else {
        if (d == 128) means_kernel<float, 128><<<nb, 256, 0, st>>>((const float *)x, perm, seg_off, H, N, K, centroids, (float *)centroids_dt);
        else means_kernel<float, 64><<<nb, 256, 0, st>>>((const float *)x, perm, seg_off, H, N, K, centroids, (float *)centroids_dt);
    }
    return cudaGetLastError();
}
