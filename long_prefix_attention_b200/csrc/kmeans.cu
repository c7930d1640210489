// kmeans.cu -- clustering of the calibration queries into K centroids.
//
// "Context Memorization for Efficient Long Context Generation", Metodologia,
// "Agrupamiento" (the query vectors are clustered, e.g. by k-means, into K
// centroids) and "Agregacion" (a centroid's query vector is the mean of its
// cluster's queries).  Seeding is k-means++ (D^2 sampling) with the uniform
// draws supplied by the caller.
#include <cuda_runtime.h>
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
// waiting) refreshes the partial sums of the ranges whose D2 changed, finds
// the range holding the threshold u * sum(D2) and the first point inside it
// whose running sum exceeds the threshold, and records the pick.
//
// Exact pruning.  From round kSeedFirstGroup on, the points are grouped by the
// chosen centre nearest to them (regrouped on a schedule as centres are
// added).  Group g has anchor a_g (its centre) and radius R_g = max |x - a_g|
// over its members; a piece (the part of a group inside one block's range of
// positions) also keeps M = max sqrt(D2) over its members.  By the triangle
// inequality every member has |x - c| >= |c - a_g| - R_g, so when
// |c - a_g| > (R_g + M)(1 + 1e-12) no member's D2 can fall and the piece is
// skipped; the margin covers the rounding of the fp64 distances, so the D2
// values, and therefore the picks, are those of the unpruned update.

constexpr int kSeedThreads = 256;
constexpr int kSeedWarps = kSeedThreads / 32;
constexpr int kSeedCh = 1024;        // positions per block
constexpr int kSeedRange = 128;      // points per partial sum of D2
constexpr int kSeedFirstGroup = 256; // first regrouping round
constexpr double kSeedMargin = 1e-12;

struct SeedWs {
    size_t off_d2, off_mdp, off_rr, off_bsum, off_r2, off_near, off_perm, off_apos, off_gcnt, off_seg,
        off_cur, off_pofs, off_dirty, off_taken, off_cnt, total;
};
SeedWs seed_ws(int H, int N, int K) {
    const size_t h = (size_t)H, n = (size_t)N, k = (size_t)K;
    const size_t nr = (n + kSeedRange - 1) / kSeedRange;
    SeedWs w;
    w.off_d2 = 0;
    w.off_mdp = al256(w.off_d2 + sizeof(double) * h * n);
    w.off_rr = al256(w.off_mdp + sizeof(double) * h * n);
    w.off_bsum = al256(w.off_rr + sizeof(double) * h * n);
    w.off_r2 = al256(w.off_bsum + sizeof(double) * h * nr);
    w.off_near = al256(w.off_r2 + sizeof(double) * h * k);
    w.off_perm = al256(w.off_near + sizeof(int) * h * n);
    w.off_apos = al256(w.off_perm + sizeof(int) * h * n);
    w.off_gcnt = al256(w.off_apos + sizeof(int) * h * n);
    w.off_seg = al256(w.off_gcnt + sizeof(int) * h * k);
    w.off_cur = al256(w.off_seg + sizeof(int) * h * (k + 1));
    w.off_pofs = al256(w.off_cur + sizeof(int) * h * k);
    w.off_dirty = al256(w.off_pofs + sizeof(uint16_t) * h * n);
    w.off_taken = al256(w.off_dirty + h * nr);
    w.off_cnt = al256(w.off_taken + h * n);
    w.total = al256(w.off_cnt + sizeof(int) * h);
    return w;
}

struct SeedArgs {
    const double *u;
    int32_t *idx;           // [H][K] picks
    double *d2;             // [H][N] D2 by point
    double *mdp;            // [H][N] piece max of D2, at the piece's first position
    double *rr;             // [H][N] R^2 of the group of each position
    double *bsum;           // [H][NR] partial sums of D2 by range of points
    double *r2;             // [H][G] group R^2 (regrouping scratch)
    int32_t *near;          // [H][N] round of the nearest chosen centre
    int32_t *perm;          // [H][N] point at each position (grouped order)
    int32_t *apos;          // [H][N] anchor point of the group of each position
    int32_t *gcnt, *seg, *cur;  // regrouping scratch: [H][G], [H][G+1], [H][G]
    uint16_t *pofs;         // [H][N] offset of the piece's first position in its block
    unsigned char *dirty;   // [H][NR] range touched this round
    unsigned char *taken;   // [H][N] point already chosen
    int *cnt;               // [H] arrival counters
    int N, K, NR;
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

// D2 update geometry: a point is LPP lanes x 16 bytes; one 16-byte load per
// lane covers PPL = 32 / LPP points, so a warp reads its 32 points with LPP
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

// |x_row - c|^2 (fp64) of 32 rows at once: lane j names row `row` (rows whose
// bit in `mask` is clear are not read), lane l reads 16-byte chunk l % LPP of
// rows i * PPL + l / LPP, and a transpose-reduction over the LPP lanes of a
// row leaves in every lane the distance of row (l % LPP) * PPL + l / LPP.
template <typename T, int D, bool STREAM>
__device__ __forceinline__ double dist32(const T *__restrict__ xh, const double *cv, int row, unsigned mask,
                                         int lane) {
    using G = SeedGeo<T, D>;
    const int sub = lane % G::LPP, grp = lane / G::LPP;
    uint4 buf[G::LPP];
#pragma unroll
    for (int i = 0; i < G::LPP; ++i) {
        const int q = i * G::PPL + grp;
        const int src = __shfl_sync(0xffffffffu, row, q);
        const uint4 *pp = reinterpret_cast<const uint4 *>(xh + (size_t)src * D + sub * G::E16);
        buf[i] = ((mask >> q) & 1u) ? (STREAM ? __ldcs(pp) : __ldg(pp)) : make_uint4(0, 0, 0, 0);
    }
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

// G = number of groups (0: no grouping yet, every point is updated).
template <typename T, int D>
__global__ void __launch_bounds__(kSeedThreads)
kmeanspp_round(const T *__restrict__ x, const SeedArgs s, int r, int G) {
    using Gm = SeedGeo<T, D>;
    const int h = blockIdx.y, N = s.N, K = s.K, NR = s.NR;
    const size_t hN = (size_t)h * N;
    const T *xh = x + hN * D;
    double *d2h = s.d2 + hN;
    unsigned char *tk = s.taken + hN;
    unsigned char *dh = s.dirty + (size_t)h * NR;
    __shared__ unsigned long long pmax[kSeedCh];  // piece max of D2 (bits), by first offset
    __shared__ int list[kSeedCh];                 // piece first offsets / dirty ranges
    __shared__ uint16_t lead[kSeedCh];            // piece first offset of each position
    __shared__ unsigned char act[kSeedCh];        // piece is updated, by first offset
    __shared__ double sh[kSeedWarps];
    __shared__ int nlist, last, pick_blk;
    __shared__ double sh_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p0 = blockIdx.x * kSeedCh;
    const int p1 = min(N, p0 + kSeedCh);

    if (r == 0) {
        // round 0: clear the state; the last block records floor(u * N)
        for (int i = p0 + tid; i < p1; i += kSeedThreads) {
            d2h[i] = __longlong_as_double(0x7ff0000000000000LL);  // +inf
            tk[i] = 0;
            s.near[hN + i] = 0;
        }
        for (int k = p0 / kSeedRange + tid; k < (p1 + kSeedRange - 1) / kSeedRange; k += kSeedThreads) dh[k] = 0;
    } else {
        const int c = s.idx[(size_t)h * K + r - 1];
        const int sub = lane % Gm::LPP;
        double cv[Gm::E16];
        widen16<T>(__ldg(reinterpret_cast<const uint4 *>(xh + (size_t)c * D + sub * Gm::E16)), cv);
        const bool grouped = G > 0;
        if (grouped) {
            // the block's pieces, then the triangle test of each
            if (tid == 0) nlist = 0;
            __syncthreads();
            const uint16_t *po = s.pofs + hN;
            for (int o = tid; o < p1 - p0; o += kSeedThreads) {
                const int f = po[p0 + o];
                lead[o] = (uint16_t)f;
                if (f == o) list[atomicAdd(&nlist, 1)] = o;
            }
            __syncthreads();
            const int nl = nlist;
            for (int j0 = warp * 32; j0 < nl; j0 += kSeedWarps * 32) {
                const int j = j0 + lane;
                const int o = j < nl ? list[j] : 0;
                const int arow = j < nl ? __ldg(s.apos + hN + p0 + o) : 0;
                const unsigned m = __ballot_sync(0xffffffffu, j < nl);
                const double dc2 = dist32<T, D, false>(xh, cv, arow, m, lane);
                const int q = (lane % Gm::LPP) * Gm::PPL + lane / Gm::LPP;  // the row this lane holds
                const int oq = __shfl_sync(0xffffffffu, o, q);
                if ((m >> q) & 1u) {
                    const double R = sqrt(s.rr[hN + p0 + oq]);
                    const double M = sqrt(s.mdp[hN + p0 + oq]);
                    act[oq] = sqrt(dc2) > (R + M) * (1.0 + kSeedMargin) ? 0 : 1;
                    pmax[oq] = 0ull;
                }
            }
            __syncthreads();
        }
        // D2 update of the positions in updated pieces, 32 at a time per warp
        for (int base = p0 + warp * 32; base < p1; base += kSeedWarps * 32) {
            const int qp = base + lane;
            const bool al = qp < p1 && (!grouped || act[lead[qp - p0]]);
            const unsigned m = __ballot_sync(0xffffffffu, al);
            if (m == 0u) continue;
            const int pt = grouped ? (al ? s.perm[hN + qp] : 0) : qp;
            const double dist = dist32<T, D, true>(xh, cv, pt, m, lane);
            const int q = (lane % Gm::LPP) * Gm::PPL + lane / Gm::LPP;
            const int i = __shfl_sync(0xffffffffu, pt, q);
            if ((m >> q) & 1u) {
                const double old = d2h[i];
                const double nd = fmin(old, dist);
                if (nd < old) {
                    d2h[i] = nd;
                    s.near[hN + i] = r - 1;
                    dh[i / kSeedRange] = 1;
                }
                if (grouped) atomicMax(&pmax[lead[base + q - p0]], (unsigned long long)__double_as_longlong(nd));
            }
        }
        if (grouped) {
            __syncthreads();
            for (int j = tid; j < nlist; j += kSeedThreads) {
                const int o = list[j];
                if (act[o]) s.mdp[hN + p0 + o] = __longlong_as_double((long long)pmax[o]);
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int old = atomicAdd(&s.cnt[h], 1);
        last = (old == (int)gridDim.x - 1);
        __threadfence();
    }
    __syncthreads();
    if (!last) return;

    // ---------------- last block of head h: choose this round's centre
    const double ur = s.u[(size_t)h * K + r];
    if (r == 0) {
        if (tid == 0) {
            int pk = (int)floor(ur * (double)N);
            pk = min(max(pk, 0), N - 1);
            s.idx[(size_t)h * K] = pk;
            tk[pk] = 1;
            s.cnt[h] = 0;
        }
        return;
    }
    double *bs = s.bsum + (size_t)h * NR;
    // refresh the sums of the ranges whose D2 changed (fixed order per range:
    // lane-strided partials, then a butterfly, so every refresh is the same)
    for (int k0 = 0; k0 < NR; k0 += kSeedThreads) {
        if (tid == 0) nlist = 0;
        __syncthreads();
        const int k = k0 + tid;
        if (k < NR && __ldcg(dh + k)) list[atomicAdd(&nlist, 1)] = k;
        __syncthreads();
        const int nd = nlist;
        for (int j = warp; j < nd; j += kSeedWarps) {
            const int kk = list[j];
            const int q0 = kk * kSeedRange;
            double v = 0.0;
#pragma unroll
            for (int e = 0; e < kSeedRange / 32; ++e) {
                const int i = q0 + e * 32 + lane;
                v += i < N ? __ldcg(d2h + i) : 0.0;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
            if (lane == 0) {
                bs[kk] = v;
                dh[kk] = 0;
            }
        }
        __syncthreads();
    }
    double total = 0.0;
    {
        double v = 0.0;
        for (int k = tid; k < NR; k += kSeedThreads) v += __ldcg(bs + k);
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
        // inclusive running sums of the range sums, chunk by chunk; the first
        // range whose running sum exceeds thr holds the pick
        double carry = 0.0;
        for (int c0 = 0; c0 < NR; c0 += kSeedThreads) {
            const int kk = c0 + tid;
            const double v = kk < NR ? __ldcg(bs + kk) : 0.0;
            const double inc = block_scan_d(v, sh) + carry;
            __syncthreads();
            if (kk < NR && inc > thr) atomicMin(&pick_blk, kk);
            if (tid == kSeedThreads - 1) sh[0] = inc;  // carry into the next chunk
            __syncthreads();
            carry = sh[0];
            if (kk == pick_blk) sh_base = inc - v;  // exclusive running sum of the range
            __syncthreads();
        }
        int blk = pick_blk;
        const bool crossed = blk != 0x7fffffff;
        const double base_run = crossed ? sh_base : 0.0;
        __syncthreads();
        if (tid == 0) pick_blk = 0x7fffffff;
        __syncthreads();
        if (crossed) {
            // inside the range: the first point whose running sum exceeds thr
            const int q0 = blk * kSeedRange;
            const int i = q0 + tid;
            const double dv = (tid < kSeedRange && i < N) ? __ldcg(d2h + i) : 0.0;
            const double inc = block_scan_d(dv, sh);
            if (tid < kSeedRange && i < N && base_run + inc > thr) atomicMin(&pick_blk, i);
            __syncthreads();
            if (pick_blk == 0x7fffffff) {
                // rounding: the range's own running sum stayed at or below
                // thr; take the range's last point with D2 > 0
                if (tid == 0) pick_blk = -1;
                __syncthreads();
                if (tid < kSeedRange && i < N && dv > 0.0) atomicMax(&pick_blk, i);
                __syncthreads();
                if (tid == 0 && pick_blk < 0) pick_blk = 0x7fffffff;
                __syncthreads();
            }
        }
        if (pick_blk == 0x7fffffff) {
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
    if (tid == 0) {
        const int pk = pick_blk;
        s.idx[(size_t)h * K + r] = pk;
        tk[pk] = 1;
        s.cnt[h] = 0;
    }
}

// ---- regrouping (before round r, with G = r - 1 chosen centres applied)
//
// Group g holds the points whose nearest applied centre is centre g; its
// radius is the largest of their D2 (D2 is exactly the distance to that
// centre).  Counting sort: histogram and radius, exclusive scan, scatter of
// the points with their piece offsets and group data.

__global__ void seed_group_hist(const SeedArgs s, int G) {
    const int h = blockIdx.y, i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= s.N) return;
    const size_t hi = (size_t)h * s.N + i;
    const int g = s.near[hi];
    atomicAdd(&s.gcnt[(size_t)h * G + g], 1);
    atomicMax(reinterpret_cast<unsigned long long *>(s.r2 + (size_t)h * G + g),
              (unsigned long long)__double_as_longlong(s.d2[hi]));
}

__global__ void seed_group_scatter(const SeedArgs s, int G) {
    const int h = blockIdx.y, i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= s.N) return;
    const size_t hN = (size_t)h * s.N;
    const int g = s.near[hN + i];
    const int pos = atomicAdd(&s.cur[(size_t)h * G + g], 1);
    const int cs = pos - pos % kSeedCh;
    const double R2 = s.r2[(size_t)h * G + g];
    s.perm[hN + pos] = i;
    s.apos[hN + pos] = s.idx[(size_t)h * s.K + g];
    s.rr[hN + pos] = R2;
    s.mdp[hN + pos] = R2;
    s.pofs[hN + pos] = (uint16_t)(max(s.seg[(size_t)h * (G + 1) + g], cs) - cs);
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

// |c|^2 of every storage-dtype centre (fp32), one warp per centre.
template <typename T, int D>
__global__ void centroid_norms(const T *__restrict__ c, int HK, float *norms) {
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
    size_t off_norm, off_cursor, total;
};
KmWs km_ws(int H, int N, int K) {
    (void)N;
    KmWs w;
    w.off_norm = 256;
    w.off_cursor = al256(w.off_norm + sizeof(float) * (size_t)H * K);
    w.total = al256(w.off_cursor + sizeof(int) * (size_t)H * K);
    return w;
}

}  // namespace asmk

// ============================================================== host side ==
using namespace asmk;

size_t asm_kmeanspp_ws_bytes(int H, int N, int d, int K) {
    (void)d;
    return seed_ws(H, N, K).total;
}

template <typename T, int D>
static void seed_round(const T *x, const SeedArgs &s, int r, int G, int H, cudaStream_t st) {
    dim3 grid((s.N + kSeedCh - 1) / kSeedCh, H);
    kmeanspp_round<T, D><<<grid, kSeedThreads, 0, st>>>(x, s, r, G);
}

cudaError_t asm_kmeanspp_launch(const void *x, int H, int N, int d, int K, const double *u,
                                asm_dtype dt, int32_t *init_idx, void *ws, cudaStream_t st) {
    const SeedWs w = seed_ws(H, N, K);
    char *b = static_cast<char *>(ws);
    SeedArgs s{};
    s.u = u;
    s.idx = init_idx;
    s.d2 = reinterpret_cast<double *>(b + w.off_d2);
    s.mdp = reinterpret_cast<double *>(b + w.off_mdp);
    s.rr = reinterpret_cast<double *>(b + w.off_rr);
    s.bsum = reinterpret_cast<double *>(b + w.off_bsum);
    s.r2 = reinterpret_cast<double *>(b + w.off_r2);
    s.near = reinterpret_cast<int32_t *>(b + w.off_near);
    s.perm = reinterpret_cast<int32_t *>(b + w.off_perm);
    s.apos = reinterpret_cast<int32_t *>(b + w.off_apos);
    s.gcnt = reinterpret_cast<int32_t *>(b + w.off_gcnt);
    s.seg = reinterpret_cast<int32_t *>(b + w.off_seg);
    s.cur = reinterpret_cast<int32_t *>(b + w.off_cur);
    s.pofs = reinterpret_cast<uint16_t *>(b + w.off_pofs);
    s.dirty = reinterpret_cast<unsigned char *>(b + w.off_dirty);
    s.taken = reinterpret_cast<unsigned char *>(b + w.off_taken);
    s.cnt = reinterpret_cast<int *>(b + w.off_cnt);
    s.N = N;
    s.K = K;
    s.NR = (N + kSeedRange - 1) / kSeedRange;
    cudaError_t e = cudaMemsetAsync(s.cnt, 0, sizeof(int) * (size_t)H, st);
    if (e != cudaSuccess) return e;
    const dim3 pgrid((N + 255) / 256, H);
    int G = 0, next = kSeedFirstGroup;
    for (int r = 0; r < K; ++r) {
        if (r == next) {
            // regroup by the nearest of the r - 1 centres applied so far;
            // then again each time the centres grow by a quarter of the
            // largest power of two below r (at least 256 rounds apart)
            G = r - 1;
            if ((e = cudaMemsetAsync(s.gcnt, 0, sizeof(int) * (size_t)H * G, st)) != cudaSuccess) return e;
            if ((e = cudaMemsetAsync(s.r2, 0, sizeof(double) * (size_t)H * G, st)) != cudaSuccess) return e;
            seed_group_hist<<<pgrid, 256, 0, st>>>(s, G);
            scan_kernel<<<H, 1024, 0, st>>>(s.gcnt, G, s.seg, s.cur);
            seed_group_scatter<<<pgrid, 256, 0, st>>>(s, G);
            int p2 = 1;
            while (p2 * 2 <= r) p2 *= 2;
            next = r + max(256, p2 / 4);
        }
        if (dt == ASM_BF16) {
            using T = __nv_bfloat16;
            if (d == 128) seed_round<T, 128>((const T *)x, s, r, G, H, st);
            else seed_round<T, 64>((const T *)x, s, r, G, H, st);
        } else {
            if (d == 128) seed_round<float, 128>((const float *)x, s, r, G, H, st);
            else seed_round<float, 64>((const float *)x, s, r, G, H, st);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
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
    const int HK = H * K;
    const int nb = (HK * 32 + 255) / 256;
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) centroid_norms<T, 128><<<nb, 256, 0, st>>>((const T *)centroids_dt, HK, norms);
        else centroid_norms<T, 64><<<nb, 256, 0, st>>>((const T *)centroids_dt, HK, norms);
    } else {
        if (d == 128) centroid_norms<float, 128><<<nb, 256, 0, st>>>((const float *)centroids_dt, HK, norms);
        else centroid_norms<float, 64><<<nb, 256, 0, st>>>((const float *)centroids_dt, HK, norms);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (dt == ASM_BF16 && d == 128)
        return asm_assign_tc_launch(x, centroids_dt, norms, H, N, K, metric, assign, static_cast<int *>(ws), st);
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
