/*
 * asm_oracle.c -- plain fp64 CPU oracle for Attention State Memory (ASM).
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package's
 * smoke check and the benchmark's CPU-baseline leg may load this library.  It
 * shares no code, header, table or helper with the CUDA path.
 *
 * Every function is the definition written out, loop by loop, in double
 * precision, with no blocking, fusion or reordering beyond the definition.
 * Inputs are the exact storage-dtype values (bf16 or fp32) upcast to double
 * by the caller.  OpenMP only distributes independent outputs (one query, one
 * head, one cluster) over threads; the arithmetic of each output is serial.
 *
 * Source: "Context Memorization for Efficient Long Context Generation"
 * (gist.science technical summary of arXiv 2605.18226), section
 * "Metodologia: Memoria de Estado de Atencion (ASM)".  Conventions the page
 * leaves open are stated at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Attention state (a, Z) of one query q over a key block K, V of L rows
 * ("Metodologia", paragraph 2: the attention output plus its normalisation
 * term suffice to rebuild the block's contribution).
 *   l_j  = scale * <q, k_j>
 *   Z    = sum_j exp(l_j)            stored as logZ = m + ln sum_j exp(l_j - m)
 *   a    = sum_j exp(l_j - logZ) v_j (the normalised output)
 * An empty block (L == 0) has a = 0 and logZ = -inf.
 */
void oracle_state(const double *q, const double *K, const double *V, int L,
                  int d, double scale, double *a, double *logz)
{
    int i, j;
    for (i = 0; i < d; i++) a[i] = 0.0;
    if (L <= 0) {
        *logz = -INFINITY;
        return;
    }
    double *logit = (double *)malloc(sizeof(double) * (size_t)L);
    double m = -INFINITY;
    for (j = 0; j < L; j++) {
        double s = 0.0;
        for (i = 0; i < d; i++) s += q[i] * K[(size_t)j * d + i];
        logit[j] = scale * s;
        if (logit[j] > m) m = logit[j];
    }
    double l = 0.0;
    for (j = 0; j < L; j++) l += exp(logit[j] - m);
    double lz = m + log(l);
    for (j = 0; j < L; j++) {
        double p = exp(logit[j] - lz);
        for (i = 0; i < d; i++) a[i] += p * V[(size_t)j * d + i];
    }
    *logz = lz;
    free(logit);
}

/*
 * Merge operator of the online-softmax identity ("Metodologia", paragraph 1,
 * and the "Fusion" bullet): two states over disjoint key blocks combine into
 * the state over their union.
 *   Z = Z1 + Z2                      (logZ by max-shifted log-sum-exp)
 *   a = (Z1 a1 + Z2 a2) / Z
 * Two empty states give the empty state (a = 0, logZ = -inf).
 * The output may alias either input.
 */
void oracle_merge(const double *a1, double z1, const double *a2, double z2,
                  int d, double *a, double *z)
{
    int i;
    if (z1 == -INFINITY && z2 == -INFINITY) {
        for (i = 0; i < d; i++) a[i] = 0.0;
        *z = -INFINITY;
        return;
    }
    double m = z1 > z2 ? z1 : z2;
    double zz = m + log(exp(z1 - m) + exp(z2 - m));
    double w1 = exp(z1 - zz), w2 = exp(z2 - zz);
    for (i = 0; i < d; i++) a[i] = w1 * a1[i] + w2 * a2[i];
    *z = zz;
}

/*
 * Prefix states of every calibration query ("Recoleccion" bullet: for each
 * query token the query vector and its state over the prefix are recorded;
 * "Eficiencia" bullet: a long prefix is split into chunks whose states are
 * merged by the identity).  Non-causal: every query sees the whole block.
 *   Q[Hq,N,d], K,V[Hkv,L,d], A[Hq,N,d] and logZ[Hq,N] are in/out.
 * Query head h reads KV head h / (Hq / Hkv).  With accumulate != 0 the block's
 * state is merged into the stored (A, logZ) (one chunk of a longer prefix);
 * otherwise it overwrites them.
 */
void oracle_build_states(const double *Q, const double *K, const double *V,
                         int Hq, int Hkv, int N, int L, int d, double scale,
                         int accumulate, double *A, double *logZ)
{
    int G = Hq / Hkv;
    long hn;
#pragma omp parallel for schedule(dynamic, 16)
    for (hn = 0; hn < (long)Hq * N; hn++) {
        int h = (int)(hn / N);
        int g = h / G;
        double *a_new = (double *)malloc(sizeof(double) * (size_t)d);
        double z_new;
        oracle_state(Q + (size_t)hn * d, K + (size_t)g * L * d,
                     V + (size_t)g * L * d, L, d, scale, a_new, &z_new);
        double *a_out = A + (size_t)hn * d;
        if (accumulate) {
            oracle_merge(a_out, logZ[hn], a_new, z_new, d, a_out, &logZ[hn]);
        } else {
            memcpy(a_out, a_new, sizeof(double) * (size_t)d);
            logZ[hn] = z_new;
        }
        free(a_new);
    }
}

static double sqdist(const double *x, const double *c, int d)
{
    double s = 0.0;
    int i;
    for (i = 0; i < d; i++) {
        double t = x[i] - c[i];
        s += t * t;
    }
    return s;
}

static double dot(const double *x, const double *c, int d)
{
    double s = 0.0;
    int i;
    for (i = 0; i < d; i++) s += x[i] * c[i];
    return s;
}

/*
 * k-means++ seeding of one head's points X[N,d] with K centres (Arthur and
 * Vassilvitskii 2007).  The pages only say the queries are clustered "e.g.
 * by k-means"; the seeding rule and its random draws are inputs here.
 *   u[K] are uniform draws in [0,1), one per round.
 *   round 0: the point floor(u[0] * N);
 *   round r: D2_i = min(D2_i, |x_i - c_{r-1}|^2) over every point, then the
 *            smallest i whose running sum of D2 (in index order) exceeds
 *            u[r] * sum(D2).  If sum(D2) == 0 the smallest index not yet
 *            chosen is taken.
 */
static void kmeanspp_one(const double *X, int N, int d, int K,
                         const double *u, int32_t *idx)
{
    double *D2 = (double *)malloc(sizeof(double) * (size_t)N);
    unsigned char *taken = (unsigned char *)calloc((size_t)N, 1);
    int i, r;
    for (i = 0; i < N; i++) D2[i] = INFINITY;
    int first = (int)floor(u[0] * (double)N);
    if (first >= N) first = N - 1;
    if (first < 0) first = 0;
    idx[0] = first;
    taken[first] = 1;
    for (r = 1; r < K; r++) {
        const double *c = X + (size_t)idx[r - 1] * d;
        double total = 0.0;
        for (i = 0; i < N; i++) {
            double t = sqdist(X + (size_t)i * d, c, d);
            if (t < D2[i]) D2[i] = t;
        }
        for (i = 0; i < N; i++) total += D2[i];
        int pick = -1;
        if (total > 0.0) {
            double thr = u[r] * total;
            double run = 0.0;
            int last_pos = -1;
            for (i = 0; i < N; i++) {
                run += D2[i];
                if (D2[i] > 0.0) last_pos = i;
                if (run > thr) {
                    pick = i;
                    break;
                }
            }
            if (pick < 0) pick = last_pos; /* thr at the very top of the CDF */
        } else {
            for (i = 0; i < N; i++)
                if (!taken[i]) {
                    pick = i;
                    break;
                }
            if (pick < 0) pick = 0;
        }
        idx[r] = pick;
        taken[pick] = 1;
    }
    free(D2);
    free(taken);
}

/* X[H,N,d], u[H,K] -> idx[H,K]; heads are independent. */
void oracle_kmeanspp_seed(const double *X, int H, int N, int d, int K,
                          const double *u, int32_t *idx)
{
    int h;
#pragma omp parallel for schedule(dynamic, 1)
    for (h = 0; h < H; h++)
        kmeanspp_one(X + (size_t)h * N * d, N, d, K, u + (size_t)h * K,
                     idx + (size_t)h * K);
}

/*
 * Batched k-means++ seeding (the batched seeding of k-means|| by Bahmani et
 * al. 2012, without its final reclustering; the pages leave the seeding
 * open).  Rounds draw up to b centres at once from the same D2 distribution
 * and only then update D2, so K centres take about K / b rounds instead of K.
 *   u[U]: uniform draws in [0,1), consumed in order (draw p uses u[p % U]).
 *   round 0: the point floor(u[0] * N).
 *   round r >= 1, with m centres chosen: nb = min(b, K - m) draws; draw j
 *            takes the smallest i whose running sum of D2 (index order)
 *            exceeds u_j * sum(D2), or the last point with D2 > 0 if none
 *            does; if sum(D2) == 0, draw j takes the j-th smallest index not
 *            yet chosen.  A draw equal to an earlier draw of the same round
 *            is dropped.  The kept draws are appended in draw order, then
 *            D2_i = min(D2_i, |x_i - c|^2) over them.
 *   after ceil((K - 1) / b) + 16 rounds the remaining centres, if any, are
 *   the smallest indices not yet chosen.
 * With b = 1 this is oracle_kmeanspp_seed with u[r] for round r.
 */
static void kmeanspp_batched_one(const double *X, int N, int d, int K, int b,
                                 const double *u, int U, int32_t *idx)
{
    double *D2 = (double *)malloc(sizeof(double) * (size_t)N);
    unsigned char *taken = (unsigned char *)calloc((size_t)N, 1);
    int32_t *batch = (int32_t *)malloc(sizeof(int32_t) * (size_t)(b > 0 ? b : 1));
    int i, j, q, m = 0, p = 0, round, cap = (K - 1 + b - 1) / b + 16;
    for (i = 0; i < N; i++) D2[i] = INFINITY;
    {
        int first = (int)floor(u[p % U] * (double)N);
        p++;
        if (first >= N) first = N - 1;
        if (first < 0) first = 0;
        idx[m++] = first;
        taken[first] = 1;
        for (i = 0; i < N; i++) {
            double t = sqdist(X + (size_t)i * d, X + (size_t)first * d, d);
            if (t < D2[i]) D2[i] = t;
        }
    }
    for (round = 1; m < K && round <= cap; round++) {
        int nb = K - m < b ? K - m : b, kept = 0;
        double total = 0.0;
        for (i = 0; i < N; i++) total += D2[i];
        for (j = 0; j < nb; j++) {
            int pick = -1;
            double uj = u[p % U];
            p++;
            if (total > 0.0) {
                double thr = uj * total, run = 0.0;
                int last_pos = -1;
                for (i = 0; i < N; i++) {
                    run += D2[i];
                    if (D2[i] > 0.0) last_pos = i;
                    if (run > thr) {
                        pick = i;
                        break;
                    }
                }
                if (pick < 0) pick = last_pos;
            } else {
                int seen = 0;
                for (i = 0; i < N; i++)
                    if (!taken[i]) {
                        if (seen == j) {
                            pick = i;
                            break;
                        }
                        seen++;
                    }
                if (pick < 0) pick = 0;
            }
            for (q = 0; q < kept; q++)
                if (batch[q] == pick) break;
            if (q == kept) batch[kept++] = pick;
        }
        for (q = 0; q < kept; q++) {
            idx[m++] = batch[q];
            taken[batch[q]] = 1;
        }
        for (i = 0; i < N; i++)
            for (q = 0; q < kept; q++) {
                double t = sqdist(X + (size_t)i * d, X + (size_t)batch[q] * d, d);
                if (t < D2[i]) D2[i] = t;
            }
    }
    for (i = 0; m < K && i < N; i++)
        if (!taken[i]) {
            idx[m++] = i;
            taken[i] = 1;
        }
    free(D2);
    free(taken);
    free(batch);
}

/* X[H,N,d], u[H,U] -> idx[H,K] (batched seeding, b draws per round). */
void oracle_kmeanspp_seed_batched(const double *X, int H, int N, int d, int K,
                                  int b, const double *u, int U, int32_t *idx)
{
    int h;
#pragma omp parallel for schedule(dynamic, 1)
    for (h = 0; h < H; h++)
        kmeanspp_batched_one(X + (size_t)h * N * d, N, d, K, b, u + (size_t)h * U, U,
                             idx + (size_t)h * K);
}

/*
 * Nearest centre of each point ("Agrupamiento" bullet for k-means; the
 * "Recuperacion" bullet for the decode-time lookup).
 *   metric 0 (L2):     argmin_c |x - c|^2, computed as the squared distance.
 *   metric 1 (cosine): argmax_c <x, c> / |c|.
 * Ties go to the smallest centre index.  gap[i] is the relative separation
 * of the best and second-best candidate: (d2 - d1) / max(|d1|, 1e-30) for L2,
 * (s1 - s2) / max(|s1|, 1e-30) for cosine; +inf when K == 1.
 * X[N,d], C[K,d] -> assign[N], gap[N] (gap may be NULL).
 */
void oracle_assign(const double *X, const double *C, int N, int K, int d,
                   int metric, int32_t *assign, double *gap)
{
    long n;
#pragma omp parallel for schedule(dynamic, 64)
    for (n = 0; n < N; n++) {
        const double *x = X + (size_t)n * d;
        int best = -1;
        double b1 = 0.0, b2 = 0.0;
        int c;
        for (c = 0; c < K; c++) {
            const double *cc = C + (size_t)c * d;
            double v;
            if (metric == 0) {
                v = sqdist(x, cc, d); /* smaller is better */
            } else {
                double nc = sqrt(dot(cc, cc, d));
                v = nc > 0.0 ? -dot(x, cc, d) / nc : 0.0; /* negated: smaller is better */
            }
            if (best < 0 || v < b1) {
                if (best >= 0) b2 = b1;
                else b2 = INFINITY;
                b1 = v;
                best = c;
            } else if (v < b2) {
                b2 = v;
            }
        }
        if (K == 1) b2 = INFINITY;
        assign[n] = best;
        if (gap) {
            double den = fabs(b1) > 1e-30 ? fabs(b1) : 1e-30;
            gap[n] = (b2 - b1) / den;
        }
    }
}

/*
 * Centroid update ("Agregacion" bullet: a cluster's query vector is the mean
 * of its members' queries).  Sums run over members in index order.  An empty
 * cluster keeps its previous centre.  X[N,d], assign[N], Cin[K,d] ->
 * Cout[K,d] (may alias Cin), counts[K].
 */
void oracle_update(const double *X, const int32_t *assign, int N, int K, int d,
                   const double *Cin, double *Cout, int32_t *counts)
{
    double *sum = (double *)calloc((size_t)K * d, sizeof(double));
    int n, c, i;
    for (c = 0; c < K; c++) counts[c] = 0;
    for (n = 0; n < N; n++) {
        c = assign[n];
        counts[c] += 1;
        for (i = 0; i < d; i++) sum[(size_t)c * d + i] += X[(size_t)n * d + i];
    }
    for (c = 0; c < K; c++)
        for (i = 0; i < d; i++)
            Cout[(size_t)c * d + i] = counts[c] > 0
                ? sum[(size_t)c * d + i] / (double)counts[c]
                : Cin[(size_t)c * d + i];
    free(sum);
}

/* Storage-dtype rounding of a centre: fp32, or fp32 then bf16 (nearest, ties
 * to even), matching an fp32 master copy with a bf16 working copy. */
static double round_storage(double v, int dtype)
{
    float f = (float)v;
    if (dtype == 0) return (double)f;
    if (isnan(f)) return (double)f;
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

void oracle_round_storage(const double *x, long n, int dtype, double *y)
{
    long i;
    for (i = 0; i < n; i++) y[i] = round_storage(x[i], dtype);
}

/*
 * Lloyd iterations of one head, starting from the points X[init_idx].
 * Iteration t: assign every point to its nearest storage-rounded centre,
 * record the inertia sum |x - c_assign|^2 against those rounded centres, then
 * move every centre to the mean of its members.  The returned assignment is
 * the last iteration's; the returned centres are the means of exactly those
 * members (fp64 master C and its storage rounding Cq).
 */
static void kmeans_one(const double *X, int N, int d, int K, int iters,
                       int metric, int dtype, const int32_t *init_idx,
                       double *C, double *Cq, int32_t *assign,
                       int32_t *counts, double *inertia)
{
    int c, t, i;
    long n;
    for (c = 0; c < K; c++)
        for (i = 0; i < d; i++)
            C[(size_t)c * d + i] = X[(size_t)init_idx[c] * d + i];
    for (t = 0; t < iters; t++) {
        oracle_round_storage(C, (long)K * d, dtype, Cq);
        for (n = 0; n < N; n++) {
            /* one point at a time, serial (threads are spent across heads) */
            const double *x = X + (size_t)n * d;
            int best = 0;
            double bv = 0.0;
            for (c = 0; c < K; c++) {
                const double *cc = Cq + (size_t)c * d;
                double v;
                if (metric == 0) {
                    v = sqdist(x, cc, d);
                } else {
                    double nc = sqrt(dot(cc, cc, d));
                    v = nc > 0.0 ? -dot(x, cc, d) / nc : 0.0;
                }
                if (c == 0 || v < bv) {
                    bv = v;
                    best = c;
                }
            }
            assign[n] = best;
        }
        if (inertia) {
            double s = 0.0;
            for (n = 0; n < N; n++)
                s += sqdist(X + (size_t)n * d, Cq + (size_t)assign[n] * d, d);
            inertia[t] = s;
        }
        oracle_update(X, assign, N, K, d, C, C, counts);
    }
    oracle_round_storage(C, (long)K * d, dtype, Cq);
}

/* X[H,N,d], init_idx[H,K] -> C,Cq[H,K,d], assign[H,N], counts[H,K],
 * inertia[H,iters] (may be NULL). */
void oracle_kmeans(const double *X, int H, int N, int d, int K, int iters,
                   int metric, int dtype, const int32_t *init_idx, double *C,
                   double *Cq, int32_t *assign, int32_t *counts,
                   double *inertia)
{
    int h;
#pragma omp parallel for schedule(dynamic, 1)
    for (h = 0; h < H; h++)
        kmeans_one(X + (size_t)h * N * d, N, d, K, iters, metric, dtype,
                   init_idx + (size_t)h * K, C + (size_t)h * K * d,
                   Cq + (size_t)h * K * d, assign + (size_t)h * N,
                   counts + (size_t)h * K,
                   inertia ? inertia + (size_t)h * iters : NULL);
}

/*
 * Attention-aware aggregation of the member states of each cluster
 * ("Agregacion" bullet: the members' states are fused by the online-softmax
 * update rule into one lossless average).  Members are taken in index order.
 *   m      = max_i logZ_i
 *   w_i    = exp(logZ_i - m)
 *   a_bar  = sum_i w_i a_i / sum_i w_i            (the Z-weighted mean of a)
 *   logZ_bar = m + ln sum_i w_i                   (zmode 1: the merged sum)
 *            = m + ln sum_i w_i - ln |members|    (zmode 0: the mean of Z)
 * An empty cluster, or one whose members are all empty states, gets a_bar = 0
 * and logZ_bar = -inf.
 * A[N,d], logZ[N], assign[N] -> Abar[K,d], logZbar[K].
 */
void oracle_aggregate(const double *A, const double *logZ,
                      const int32_t *assign, int N, int K, int d, int zmode,
                      double *Abar, double *logZbar)
{
    int c;
#pragma omp parallel for schedule(dynamic, 16)
    for (c = 0; c < K; c++) {
        int n, i, cnt = 0;
        double m = -INFINITY;
        double *ab = Abar + (size_t)c * d;
        for (i = 0; i < d; i++) ab[i] = 0.0;
        for (n = 0; n < N; n++)
            if (assign[n] == c) {
                cnt++;
                if (logZ[n] > m) m = logZ[n];
            }
        if (cnt == 0 || m == -INFINITY) {
            logZbar[c] = -INFINITY;
            continue;
        }
        double S = 0.0;
        for (n = 0; n < N; n++)
            if (assign[n] == c) {
                double w = exp(logZ[n] - m);
                S += w;
                for (i = 0; i < d; i++) ab[i] += w * A[(size_t)n * d + i];
            }
        for (i = 0; i < d; i++) ab[i] /= S;
        logZbar[c] = m + log(S) - (zmode == 0 ? log((double)cnt) : 0.0);
    }
}

/*
 * Score of centre c for query x by the retrieval rule of oracle_assign,
 * oriented so that smaller is better: |x - c|^2 (L2) or -<x, c>/|c| (cosine).
 */
static double retrieval_score(const double *x, const double *c, int d, int metric)
{
    if (metric == 0) return sqdist(x, c, d);
    {
        double nc = sqrt(dot(c, c, d));
        return nc > 0.0 ? -dot(x, c, d) / nc : 0.0;
    }
}

/*
 * Two-level centroid search, the hierarchical lookup the pages name
 * ("Complejidad": retrieval in O(log K) with a hierarchical index) without
 * giving its construction; the plainest two-level reading is taken.  The K
 * centres of a head are grouped into K1 clusters whose members are the rows
 * seg_off[j] .. seg_off[j+1]-1 of the centre array (ordered by cluster), each
 * cluster with a super-centre S[j].  The query scores every super-centre
 * with the retrieval rule, keeps the P best clusters (ties to the smaller
 * cluster index), and returns the best row among the members of those
 * clusters by the same rule (ties to the smaller row).
 * q[d], S[K1,d], seg_off[K1+1], C[K,d] -> idx, sel[P] (best cluster first),
 * gap_sel: relative gap between the P-th and (P+1)-th cluster score (+inf
 * when P >= K1), gap_idx: relative gap between the best and second-best
 * member score (+inf with a single member).
 */
static void index_search_one(const double *q, const double *S, const int32_t *seg_off, const double *C,
                             int K1, int d, int P, int metric, int32_t *idx, int32_t *sel, double *gap_sel,
                             double *gap_idx)
{
    double *sc = (double *)malloc(sizeof(double) * (size_t)K1);
    unsigned char *used = (unsigned char *)calloc((size_t)K1, 1);
    int j, p, Psel = P < K1 ? P : K1;
    double last = 0.0, next = INFINITY;
    for (j = 0; j < K1; j++) sc[j] = retrieval_score(q, S + (size_t)j * d, d, metric);
    for (p = 0; p < Psel; p++) {
        int bj = -1;
        for (j = 0; j < K1; j++)
            if (!used[j] && (bj < 0 || sc[j] < sc[bj])) bj = j;
        used[bj] = 1;
        sel[p] = bj;
        last = sc[bj];
    }
    for (p = Psel; p < P; p++) sel[p] = -1;
    for (j = 0; j < K1; j++)
        if (!used[j] && sc[j] < next) next = sc[j];
    *gap_sel = (next - last) / (fabs(last) > 1e-30 ? fabs(last) : 1e-30);
    {
        int best = -1, r;
        double b1 = INFINITY, b2 = INFINITY;
        /* rows of the selected clusters, in row order (clusters are ordered) */
        for (j = 0; j < K1; j++) {
            if (!used[j]) continue;
            for (r = seg_off[j]; r < seg_off[j + 1]; r++) {
                double v = retrieval_score(q, C + (size_t)r * d, d, metric);
                if (best < 0 || v < b1) {
                    b2 = b1;
                    b1 = v;
                    best = r;
                } else if (v < b2) {
                    b2 = v;
                }
            }
        }
        *idx = best < 0 ? 0 : best;
        *gap_idx = (b2 - b1) / (fabs(b1) > 1e-30 ? fabs(b1) : 1e-30);
    }
    free(sc);
    free(used);
}

/*
 * index_search_one for every batch row b and query head h:
 * q[B,Hq,d], S[Hq,K1,d], seg_off[Hq,K1+1], C[Hq,K,d] -> idx[B,Hq],
 * sel[B,Hq,P], gap_sel[B,Hq], gap_idx[B,Hq].
 */
void oracle_index_search(const double *q, const double *S, const int32_t *seg_off, const double *C, int B,
                         int Hq, int K, int K1, int d, int P, int metric, int32_t *idx, int32_t *sel,
                         double *gap_sel, double *gap_idx)
{
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * Hq; bh++) {
        int h = (int)(bh % Hq);
        index_search_one(q + (size_t)bh * d, S + (size_t)h * K1 * d, seg_off + (size_t)h * (K1 + 1),
                         C + (size_t)h * K * d, K1, d, P, metric, idx + bh, sel + (size_t)bh * P,
                         gap_sel + bh, gap_idx + bh);
    }
}

/*
 * One decode step ("Fase de Inferencia Online": Recuperacion, then Fusion).
 * For every batch row b and query head h (KV head g = h / (Hq / Hkv)):
 *   idx      = nearest centre of q[b,h] among C[h,0:K) (oracle_assign rule),
 *              or idx_in[b,h] when idx_in is not NULL;
 *   local    = state of q[b,h] over Kc[b,g,0:T_b), Vc[b,g,0:T_b), T_b =
 *              local_len[b] (the query's own non-prefix tokens);
 *   out, lse = merge((Abar[h,idx], logZbar[h,idx]), local).
 * q[B,Hq,d], C/Abar[Hq,K,d], logZbar[Hq,K], Kc/Vc[B,Hkv,Tmax,d] ->
 * out[B,Hq,d], lse[B,Hq], idx_out[B,Hq], gap[B,Hq] (idx_out, gap may be NULL).
 */
void oracle_decode(const double *q, const double *C, const double *Abar,
                   const double *logZbar, const double *Kc, const double *Vc,
                   const int32_t *local_len, int B, int Hq, int Hkv, int K,
                   int Tmax, int d, double scale, int metric,
                   const int32_t *idx_in, double *out, double *lse,
                   int32_t *idx_out, double *gap)
{
    int G = Hq / Hkv;
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * Hq; bh++) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        const double *qq = q + (size_t)bh * d;
        int32_t idx;
        double gp = INFINITY;
        if (idx_in) {
            idx = idx_in[bh];
        } else {
            oracle_assign(qq, C + (size_t)h * K * d, 1, K, d, metric, &idx, &gp);
        }
        double *al = (double *)malloc(sizeof(double) * (size_t)d);
        double zl;
        size_t kv = ((size_t)b * Hkv + g) * (size_t)Tmax * d;
        oracle_state(qq, Kc + kv, Vc + kv, local_len[b], d, scale, al, &zl);
        oracle_merge(Abar + ((size_t)h * K + idx) * d, logZbar[(size_t)h * K + idx],
                     al, zl, d, out + (size_t)bh * d, &lse[bh]);
        if (idx_out) idx_out[bh] = idx;
        if (gap) gap[bh] = gp;
        free(al);
    }
}

/*
 * Full attention of the decode queries over an explicit shared prefix
 * Kp,Vp[Hkv,Lp,d] followed by each row's local tokens Kc,Vc[b,g,0:T_b): the
 * quantity the memory lookup stands in for ("Fusion" bullet: the exact output
 * as if the prefix were present).  The keys are concatenated, then one state
 * is taken over them.
 */
void oracle_full_attention(const double *q, const double *Kp, const double *Vp,
                           int Lp, const double *Kc, const double *Vc,
                           const int32_t *local_len, int B, int Hq, int Hkv,
                           int Tmax, int d, double scale, double *out,
                           double *lse)
{
    int G = Hq / Hkv;
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * Hq; bh++) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        int T = local_len[b];
        int L = Lp + T;
        double *Kcat = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
        double *Vcat = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
        memcpy(Kcat, Kp + (size_t)g * Lp * d, sizeof(double) * (size_t)Lp * d);
        memcpy(Vcat, Vp + (size_t)g * Lp * d, sizeof(double) * (size_t)Lp * d);
        size_t kv = ((size_t)b * Hkv + g) * (size_t)Tmax * d;
        memcpy(Kcat + (size_t)Lp * d, Kc + kv, sizeof(double) * (size_t)T * d);
        memcpy(Vcat + (size_t)Lp * d, Vc + kv, sizeof(double) * (size_t)T * d);
        oracle_state(q + (size_t)bh * d, Kcat, Vcat, L, d, scale,
                     out + (size_t)bh * d, &lse[bh]);
        free(Kcat);
        free(Vcat);
    }
}
