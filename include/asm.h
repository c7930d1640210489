/*
 * asm.h -- C ABI of the Attention State Memory (ASM) hot path on NVIDIA B200
 * (sm_100a).
 *
 * Method: "Context Memorization for Efficient Long Context Generation"
 * (technical summary of arXiv 2605.18226), section "Metodologia: Memoria de
 * Estado de Atencion (ASM)".  A long conditioning prefix is replaced by a
 * lookup memory of K query centroids per head, each carrying a precomputed
 * attention state (a, Z) of the prefix; every decode step retrieves the
 * nearest centroid and merges its state with attention over the locally
 * generated tokens by the online-softmax identity.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every array argument is a DEVICE pointer unless marked "host".  The caller
 *   allocates and owns every buffer; the library never allocates, frees or
 *   keeps state between calls.
 * - Layouts are row-major and contiguous with the head dimension d innermost.
 *   Hq query heads share Hkv key/value heads; query head h reads KV head
 *   h / (Hq / Hkv) (grouped-query attention).
 * - Storage dtype `dt` (fp32 or bf16) applies to q, k, v, a, centroids_dt,
 *   a_bar and out.  logZ-type arrays and the centroid master copy are fp32.
 *   Arithmetic is fp32 (k-means++ distances: fp64).
 * - Z is stored as its natural logarithm logZ = ln sum_j exp(scale <q, k_j>),
 *   and `a` is the normalised attention output.  The empty state is
 *   (a = 0, logZ = -inf).
 * - Calls are asynchronous on `stream`.  All arguments are validated on the
 *   host before anything is enqueued; an invalid call returns an error code
 *   and touches no buffer.  Kernel launch failures return ASM_ERR_CUDA;
 *   faults inside a kernel surface at the caller's next synchronisation.
 * - Pointers must be 16-byte aligned; d must be 64 or 128; Hq % Hkv == 0 and
 *   Hq / Hkv must be 1, 2, 4 or 8.
 * - Calls that take a workspace `ws` of `ws_bytes` bytes document its size
 *   function.  Workspaces of asm_decode_step and asm_flash_decode hold
 *   self-resetting counters: zero them once with asm_workspace_init before
 *   the first call, then reuse them for any number of calls on one stream.
 *   The k-means workspace (asm_kmeans_workspace_size) starts with the same
 *   error word; zero it once too if that word is to be read.
 *   Two calls that overlap on the GPU must not share a workspace.
 */
#ifndef ASM_B200_H
#define ASM_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ASM_OK = 0,
    ASM_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or enum   */
    ASM_ERR_UNSUPPORTED = 2, /* valid but unsupported shape (d, group size) */
    ASM_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
    ASM_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    ASM_ERR_TIMEOUT = 5      /* a device-side bounded wait gave up          */
} asm_status;

typedef enum { ASM_F32 = 0, ASM_BF16 = 1 } asm_dtype;

/* Retrieval metric ("Recuperacion" bullet).  The page names cosine
 * similarity; squared L2 is the default here, matching k-means.
 *   ASM_L2:     argmax_c <q, c> - |c|^2 / 2   (== argmin |q - c|^2)
 *   ASM_COSINE: argmax_c <q, c> / |c|         (0 for a zero centre)
 * Ties go to the smallest centre index. */
typedef enum { ASM_L2 = 0, ASM_COSINE = 1 } asm_metric;

/* Normalisation term of an aggregated cluster ("Agregacion" bullet).
 *   ASM_ZBAR_MEAN: Z_bar = mean of the members' Z (default)
 *   ASM_ZBAR_SUM:  Z_bar = sum of the members' Z (plain state merge) */
typedef enum { ASM_ZBAR_MEAN = 0, ASM_ZBAR_SUM = 1 } asm_zbar_mode;

/* ------------------------------------------------------------------------ */
/* Offline memory build                                                     */
/* ------------------------------------------------------------------------ */

/*
 * asm_build_states -- attention state of every calibration query over one
 * block of the prefix ("Recoleccion" bullet: for each query its state over
 * the prefix; "Eficiencia" bullet: a long prefix is encoded chunk by chunk and
 * the chunk states are merged with the online-softmax identity).
 *   q      [Hq, N, d]  dt   calibration queries
 *   k, v   [Hkv, L, d] dt   the prefix block (non-causal: all L keys are seen)
 *   scale               softmax scale (typically 1/sqrt(d))
 *   accumulate          0: overwrite (a, logz) with this block's state;
 *                       1: merge this block's state into the stored (a, logz)
 *                          (a is re-rounded to dt after each merge)
 *   a      [Hq, N, d]  dt   output / in-out when accumulate
 *   logz   [Hq, N]     fp32 output / in-out when accumulate
 * L == 0 with accumulate == 0 writes the empty state.  No workspace.
 * bf16 with d = 128 runs on the tcgen05 tensor cores (bf16 products, fp32
 * accumulators and softmax statistics); a tensor-core pipeline wait that times
 * out writes NaN into logz of the rows it covers.  Other cases run on CUDA
 * cores in fp32.
 */
asm_status asm_build_states(const void *q, const void *k, const void *v,
                            int Hq, int Hkv, int N, int L, int d, float scale,
                            asm_dtype dt, int accumulate, void *a, float *logz,
                            cudaStream_t stream);

/*
 * asm_merge_states -- merge a second set of attention states into a first,
 * row by row, by the online-softmax identity ("Eficiencia" bullet: the
 * states of a long prefix's chunks are combined by the identity; with the
 * chunks encoded on several GPUs, the gathered chunk states are folded with
 * this call in chunk order):
 *   z = ln(e^z_acc + e^z_in),  a_acc = e^(z_acc - z) a_acc + e^(z_in - z) a_in
 * The empty state (0, -inf) is the identity; a_acc is rounded to dt.
 *   a_acc  [R, d] dt   in/out     logz_acc [R] fp32 in/out
 *   a_in   [R, d] dt              logz_in  [R] fp32
 * R rows (for example heads x queries).  The two sets must not overlap
 * (ASM_ERR_INVALID_ARG).  No workspace; one kernel launch, HBM-bound.
 */
asm_status asm_merge_states(void *a_acc, float *logz_acc, const void *a_in,
                            const float *logz_in, int64_t R, int d,
                            asm_dtype dt, cudaStream_t stream);

/*
 * asm_kmeanspp_seed -- k-means++ initial centres of every head's points
 * (the clustering of the "Agrupamiento" bullet; seeding by D^2 sampling,
 * Arthur & Vassilvitskii 2007).  Round 0 takes point floor(u[h,0] * N); round
 * r takes the smallest i whose running sum of D2 (index order) exceeds
 * u[h,r] * sum(D2), where D2_i is the squared distance (fp64) of point i to
 * its nearest chosen centre; if sum(D2) == 0 the smallest unchosen index.
 *   x        [H, N, d] dt   points
 *   u        [H, K]    fp64 uniform draws in [0, 1), one per round
 *   init_idx [H, K]    int32 output
 *   ws       asm_kmeanspp_workspace_size(H, N, d, K) bytes
 * Requires 1 <= K <= N; N > 2^24 returns ASM_ERR_UNSUPPORTED.  The update
 * skips groups of points that the triangle inequality shows cannot move (a
 * work saving only: the D2 values and picks are those of the full update).
 * The groups are, first, the points nearest to each of a fixed set of
 * anchor points (bf16, d = 128, from a third of max(256, K/8) rounds), then
 * the points nearest to each chosen centre (from 3K/16 rounds, regrouped on
 * a schedule).  One kernel launch per round, plus a few launches at each
 * regrouping; all are queued on `stream` without synchronising.
 */
size_t asm_kmeanspp_workspace_size(int H, int N, int d, int K);

/*
 * asm_kmeanspp_seed_batched -- batched k-means++ seeding: each round draws
 * up to `batch` centres from the same D2 distribution and only then updates
 * D2 (the batched seeding of k-means||, Bahmani et al. 2012, without its
 * reclustering), so K centres take about K / batch rounds instead of K.  It
 * changes the seeds: with batch = 1 it is asm_kmeanspp_seed.
 *   round 0: point floor(u[h,0] * N).  Round r: nb = min(batch, K - m) draws
 *   (m centres chosen), draw j taking the smallest i whose running sum of D2
 *   (index order) exceeds u_j * sum(D2) (the last point with D2 > 0 if
 *   rounding leaves none; the j-th smallest unchosen index if sum(D2) = 0); a
 *   draw equal to an earlier one of the same round is dropped; the kept
 *   draws are appended in draw order; then D2_i = min(D2_i, |x_i - c|^2)
 *   over them.  After ceil((K - 1) / batch) + 16 rounds any remaining
 *   centres are the smallest unchosen indices.  D2 is exact fp64 to the
 *   centre the tensor-core (bf16, d = 128) or CUDA-core assignment finds
 *   nearest among the round's centres.
 *   x        [H, N, d] dt   points
 *   u        [H, U]    fp64 uniform draws in [0, 1), consumed in order
 *                           (draw p of a head uses u[h, p % U])
 *   init_idx [H, K]    int32 output
 *   ws       asm_kmeanspp_batched_workspace_size(H, N, d, K, batch) bytes;
 *            its word 0 is the error word (asm_workspace_error)
 * Requires 1 <= K <= N, 1 <= batch <= 256, U >= 1; N > 2^21 returns
 * ASM_ERR_UNSUPPORTED.  Two launches per round for bf16 with d = 128 (the
 * draws, then one fused pass: tensor-core nearest centre, D2 update, sums),
 * four otherwise.  Synchronises `stream` after about K / batch rounds to see
 * whether repeated draws left any head short, and again after each of the
 * (at most 16) extra rounds that then run.
 */
size_t asm_kmeanspp_batched_workspace_size(int H, int N, int d, int K, int batch);
asm_status asm_kmeanspp_seed_batched(const void *x, int H, int N, int d, int K, int batch,
                                     const double *u, int U, asm_dtype dt, int32_t *init_idx,
                                     void *ws, size_t ws_bytes, cudaStream_t stream);
asm_status asm_kmeanspp_seed(const void *x, int H, int N, int d, int K,
                             const double *u, asm_dtype dt, int32_t *init_idx,
                             void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * asm_kmeans_assign -- nearest centre of every point ("Agrupamiento"
 * bullet), with the metric rule above, against the storage-dtype centres.
 *   x [H, N, d] dt, centroids_dt [H, K, d] dt -> assign [H, N] int32.
 *   ws asm_kmeans_workspace_size(H, N, d, K) bytes (error word, centre norms).
 * bf16 with d = 128 runs on the tcgen05 tensor cores (bf16 products, fp32
 * accumulation); other cases on CUDA cores in fp32.  A tensor-core pipeline
 * wait that times out sets the workspace error word to ASM_ERR_TIMEOUT.
 */
asm_status asm_kmeans_assign(const void *x, const void *centroids_dt, int H,
                             int N, int d, int K, asm_metric metric,
                             asm_dtype dt, int32_t *assign, void *ws,
                             size_t ws_bytes, cudaStream_t stream);

/*
 * asm_kmeans_update -- every centre moves to the mean of its members
 * ("Agregacion" bullet: a cluster's query vector is the mean of its
 * members' queries); an empty cluster keeps its centre.  Also produces the
 * members of each cluster in index order: perm[h, seg_off[h,c] ..
 * seg_off[h,c+1]) lists the points of cluster c ascending.
 *   x [H,N,d] dt, assign [H,N]
 *   centroids    [H, K, d] fp32 in/out (master copy)
 *   centroids_dt [H, K, d] dt   out (storage rounding of the master)
 *   counts [H, K], perm [H, N], seg_off [H, K+1] int32 out
 *   ws asm_kmeans_workspace_size(H, N, d, K) bytes
 */
asm_status asm_kmeans_update(const void *x, const int32_t *assign, int H,
                             int N, int d, int K, asm_dtype dt,
                             float *centroids, void *centroids_dt,
                             int32_t *counts, int32_t *perm, int32_t *seg_off,
                             void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * asm_kmeans -- Lloyd's algorithm from the points x[h, init_idx[h, :]]:
 * `iters` rounds of asm_kmeans_assign then asm_kmeans_update.  On return the
 * assignment is the last round's and the centres are the means of exactly
 * those members.  Arguments as in the two calls above; iters >= 1.
 */
size_t asm_kmeans_workspace_size(int H, int N, int d, int K);
asm_status asm_kmeans(const void *x, int H, int N, int d, int K, int iters,
                      asm_metric metric, asm_dtype dt, const int32_t *init_idx,
                      float *centroids, void *centroids_dt, int32_t *assign,
                      int32_t *counts, int32_t *perm, int32_t *seg_off,
                      void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * asm_aggregate -- attention-aware aggregation of each cluster's member
 * states ("Agregacion" bullet: members are fused by the online-softmax update
 * rule into one lossless average):
 *   m = max_i logz_i,  w_i = exp(logz_i - m)
 *   a_bar = sum_i w_i a_i / sum_i w_i           (Z-weighted mean of a)
 *   logz_bar = m + ln sum_i w_i [- ln |members| in ASM_ZBAR_MEAN mode]
 * Members come from perm / seg_off of asm_kmeans_update.  An empty cluster
 * gets (0, -inf).
 *   a [H, N, d] dt, logz [H, N] fp32 -> a_bar [H, K, d] dt, logz_bar [H, K]
 * No workspace.
 */
asm_status asm_aggregate(const void *a, const float *logz, const int32_t *perm,
                         const int32_t *seg_off, int H, int N, int d, int K,
                         asm_zbar_mode zmode, asm_dtype dt, void *a_bar,
                         float *logz_bar, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Online decode                                                            */
/* ------------------------------------------------------------------------ */

/*
 * asm_decode_step -- one decode step for a batch ("Fase de Inferencia
 * Online": Recuperacion then Fusion).  For every row b and query head h
 * (KV head g = h / (Hq / Hkv)):
 *   idx      = nearest centre of q[b,h] in centroids[h] (metric rule above)
 *   local    = state of q[b,h] over k_cache[b,g,0:T_b), v_cache[b,g,0:T_b)
 *              with T_b = local_len[b] (the row's non-prefix tokens)
 *   out, lse = merge((a_bar[h,idx], logz_bar[h,idx]), local)
 * so the prefix is never read: per-step cost depends on K and T_b only.
 *   q         [B, Hq, d]       dt
 *   centroids [Hq, K, d]       dt
 *   a_bar     [Hq, K, d]       dt
 *   logz_bar  [Hq, K]          fp32
 *   k_cache, v_cache [B, Hkv, Tmax, d] dt
 *   local_len [B]              int32, device, 0 <= T_b <= Tmax
 *   out       [B, Hq, d]       dt   output
 *   lse_out   [B, Hq]          fp32 output (natural log of the merged Z), or NULL
 *   idx_out   [B, Hq]          int32 output, or NULL
 *   flags     0, or ASM_DECODE_PREFETCH_CENTROIDS
 *   ws        asm_decode_workspace_size(...) bytes, zeroed once by
 *             asm_workspace_init.
 * One (fp32) or two (bf16) kernel launches, with programmatic dependent
 * launch enabled: a kernel may start while the preceding kernel in `stream`
 * finishes, and reads no argument before that kernel has completed --
 * except, with
 * ASM_DECODE_PREFETCH_CENTROIDS, the `centroids` array, which it may start
 * streaming early.  Pass that flag only when the preceding kernel in the
 * stream does not write `centroids` (the memory is normally built once and
 * then only read).  T_b == 0 returns the retrieved state itself.
 */
#define ASM_DECODE_PREFETCH_CENTROIDS 1u
size_t asm_decode_workspace_size(int B, int Hq, int Hkv, int K, int Tmax,
                                 int d, asm_dtype dt);
asm_status asm_decode_step(const void *q, const void *centroids,
                           const void *a_bar, const float *logz_bar,
                           const void *k_cache, const void *v_cache,
                           const int32_t *local_len, int B, int Hq, int Hkv,
                           int K, int Tmax, int d, float scale,
                           asm_metric metric, asm_dtype dt, void *out,
                           float *lse_out, int32_t *idx_out, unsigned flags,
                           void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * asm_decode_step_launches -- kernel launches one asm_decode_step (or
 * asm_decode_step_search) call with these sizes makes, or -1 for sizes the
 * call rejects or when no device is present: bf16 2 (split units, then a
 * merge kernel), fp32 1 (streaming CTAs, merged by the last to finish).
 */
int asm_decode_step_launches(int B, int Hq, int Hkv, int K, int Tmax, int d,
                             asm_dtype dt);

/*
 * asm_decode_step_noalloc -- asm_decode_step without a caller workspace.
 * The paper has no counterpart: this is a convenience of the library.
 * It exists for callers that cannot allocate device memory at the point where
 * they decode -- for example a plug-in inside a host framework that owns all
 * device allocations and hands none to extensions, or a latency-critical loop
 * where cudaMalloc is ruled out because it may synchronise the device.
 * Instead of `ws`, the call uses a scratch array of 8 MiB compiled into the
 * library (a file-scope __device__ array: every GPU that loads the library
 * holds it until the process exits).  Problems whose
 * asm_decode_workspace_size(...) exceeds 8 MiB are rejected with
 * ASM_ERR_WORKSPACE.  The call allocates and frees nothing.
 * Arguments, outputs and errors are those of asm_decode_step; every argument
 * is checked before anything is enqueued.  A device-side timeout is recorded
 * in the array's error word, which asm_decode_noalloc_error reads.
 * - The first call on a device looks up the array's device address for that
 *   device (with the device current); make that first call before any stream
 *   capture.
 * - Every call on a device shares the one array and it keeps the previous
 *   call's contents; the call clears the part that must start at zero.  Calls
 *   that overlap on the GPU (other streams, other host threads) race on it and
 *   must be serialised by the caller.
 */
asm_status asm_decode_step_noalloc(const void *q, const void *centroids,
                                   const void *a_bar, const float *logz_bar,
                                   const void *k_cache, const void *v_cache,
                                   const int32_t *local_len, int B, int Hq,
                                   int Hkv, int K, int Tmax, int d,
                                   float scale, asm_metric metric,
                                   asm_dtype dt, void *out, float *lse_out,
                                   int32_t *idx_out, unsigned flags,
                                   cudaStream_t stream);

/*
 * asm_decode_noalloc_error -- the error word of the built-in scratch of
 * asm_decode_step_noalloc on the current device, copied to the host pointer
 * `code`: 0, or ASM_ERR_TIMEOUT when a bounded device-side wait of the last
 * asm_decode_step_noalloc call on this device gave up (its outputs are then
 * not valid).  Each call clears the word when it starts, so this reports the
 * most recent call.  Synchronises `stream`.
 */
asm_status asm_decode_noalloc_error(int *code, cudaStream_t stream);

/*
 * asm_flash_decode -- the quantity the memory stands in for: decode attention
 * over an explicit prefix shared by the whole batch followed by each row's
 * local tokens ("Fusion" bullet: the exact output as if the prefix were
 * present).  Used as the full-attention comparison.
 *   k_prefix, v_prefix [Hkv, Lp, d] dt (read once per call for all rows)
 *   other arguments as asm_decode_step; lse_out may be NULL.
 *   ws asm_flash_decode_workspace_size(...) bytes, zeroed once by
 *   asm_workspace_init.
 * bf16 with d = 128 and B >= 2: the prefix runs on the tcgen05 tensor cores
 * in chunks, with the B * (Hq / Hkv) query rows of each KV head as the rows
 * of one tile, then the local tokens and the merge: three kernel launches.
 * Otherwise the prefix and local tokens are split into units that each
 * serve one row (the rows of one prefix unit run together): two launches.
 */
size_t asm_flash_decode_workspace_size(int B, int Hq, int Hkv, int Lp,
                                       int Tmax, int d, asm_dtype dt);
asm_status asm_flash_decode(const void *q, const void *k_prefix,
                            const void *v_prefix, int Lp, const void *k_cache,
                            const void *v_cache, const int32_t *local_len,
                            int B, int Hq, int Hkv, int Tmax, int d,
                            float scale, asm_dtype dt, void *out,
                            float *lse_out, void *ws, size_t ws_bytes,
                            cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Two-level (hierarchical) memory                                           */
/* ------------------------------------------------------------------------ */

/*
 * The retrieval the pages describe is hierarchical, in O(log K)
 * ("Complejidad"), without its construction; the plainest two-level reading
 * is provided.  Index build: cluster each head's K centres into K1 clusters
 * with asm_kmeanspp_seed + asm_kmeans run on the centres themselves (points =
 * centroids_dt [Hq, K, d], clusters = K1); their centroids_dt are the
 * super-centres, their perm / seg_off the members, their counts give
 * max_seg.  Then asm_index_reorder lays the memory out by cluster.
 *
 * asm_index_reorder -- row i of head h of each output is row perm[h, i] of
 * the corresponding input, so that cluster j occupies rows
 * seg_off[h, j] .. seg_off[h, j+1]-1.
 *   perm [H, K] int32; centroids, a_bar [H, K, d] dt; logz_bar [H, K] fp32
 *   -> centroids_ord, a_bar_ord, logz_bar_ord of the same shapes (distinct
 *   buffers).
 */
asm_status asm_index_reorder(const int32_t *perm, int H, int K, int d,
                             asm_dtype dt, const void *centroids,
                             const void *a_bar, const float *logz_bar,
                             void *centroids_ord, void *a_bar_ord,
                             float *logz_bar_ord, cudaStream_t stream);

/*
 * asm_decode_step_indexed -- asm_decode_step with the two-level search: each
 * query head scores the K1 super-centres, keeps the P best clusters (ties to
 * the smaller cluster index) and retrieves the best member of those clusters
 * (ties to the smaller row), both by the retrieval metric; then the local
 * attention and the merge as in asm_decode_step.  With P = K1 it is the flat
 * search.
 *   supers   [Hq, K1, d] dt   super-centres
 *   seg_off  [Hq, K1 + 1]     int32, cluster j = rows seg_off[j] .. seg_off[j+1]-1
 *   K1, P    1 <= P <= min(K1, 32), K1 <= min(K, 4096)
 *   max_seg  at least the largest cluster (members beyond it are not read)
 *   centroids, a_bar, logz_bar: the memory ordered by asm_index_reorder
 *   idx_out  the retrieved row of the ordered memory (perm maps it back)
 *   other arguments as asm_decode_step (no flags).  bf16 only.
 *   ws asm_decode_indexed_workspace_size(...) bytes, zeroed once by
 *   asm_workspace_init.
 * Three kernel launches: the cluster choice, then the member and local units,
 * then the merge.
 */
size_t asm_decode_indexed_workspace_size(int B, int Hq, int Hkv, int K1, int P,
                                         int max_seg, int Tmax, int d,
                                         asm_dtype dt);
asm_status asm_decode_step_indexed(const void *q, const void *supers,
                                   const int32_t *seg_off, int K1, int P,
                                   int max_seg, const void *centroids,
                                   const void *a_bar, const float *logz_bar,
                                   const void *k_cache, const void *v_cache,
                                   const int32_t *local_len, int B, int Hq,
                                   int Hkv, int K, int Tmax, int d, float scale,
                                   asm_metric metric, asm_dtype dt, void *out,
                                   float *lse_out, int32_t *idx_out, void *ws,
                                   size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Whitened retrieval                                                       */
/* ------------------------------------------------------------------------ */

/*
 * The retrieval may whiten the vectors first ("Recuperacion" bullet of "Fase
 * de Inferencia Online"; the pages give no recipe).  Reading: ZCA whitening
 * from each head's calibration queries.  Build the clusters on the whitened
 * queries (asm_whiten, then asm_kmeanspp_seed / asm_kmeans on the result);
 * build the states from the original queries (asm_build_states) and aggregate
 * them over those clusters (asm_aggregate); at decode, search with the
 * whitened query against the whitened centres while the local attention uses
 * the original query (asm_decode_step_search).
 *
 * asm_whitening -- per head h, from its N points x[h]:
 *   mu[h] = mean of the points, C = (1/N) sum (x - mu)(x - mu)^T,
 *   W[h]  = (C + eps I)^(-1/2), eps = eps_rel * trace(C) / d (symmetric).
 *   x  [H, N, d] dt;  mu [H, d] fp32 output;  W [H, d, d] fp32 output.
 *   ws asm_whitening_workspace_size(H, d) bytes; the error word (read with
 *   asm_workspace_error) becomes ASM_ERR_TIMEOUT if the iteration for the
 *   inverse square root has not converged after 100 steps.  That happens
 *   for an exactly zero or a negative eigenvalue, which eps_rel > 0
 *   excludes; a covariance singular only up to rounding has tiny positive
 *   eigenvalues, and W then holds their (huge) inverse square roots, as the
 *   exact definition does.  Use eps_rel > 0 for rank-deficient data.
 * Moments in fp64, then a Newton-Schulz iteration in fp64 (two launches).
 */
size_t asm_whitening_workspace_size(int H, int d);
asm_status asm_whitening(const void *x, int H, int N, int d, asm_dtype dt,
                         float eps_rel, float *mu, float *W, void *ws,
                         size_t ws_bytes, cudaStream_t stream);

/*
 * asm_whiten -- y = W[h] (x - mu[h]) for R rows of every head h: row r of
 * head h starts at element h * head_stride + r * row_stride of x (and of y
 * with the y strides).  [H, N, d] points: strides (N d, d); decode queries
 * [B, Hq, d] (H = Hq, R = B): strides (d, Hq d).  fp32 arithmetic, output
 * rounded to dt.  x and y must not overlap.
 */
asm_status asm_whiten(const void *x, int H, int R, int d, asm_dtype dt,
                      int64_t head_stride, int64_t row_stride, const float *mu,
                      const float *W, void *y, int64_t y_head_stride,
                      int64_t y_row_stride, cudaStream_t stream);

/*
 * asm_decode_step_search -- asm_decode_step whose centroid search uses
 * q_search [B, Hq, d] (dt) in place of q; the local attention and the merge
 * use q.  Same arguments, workspace and launches otherwise.
 */
asm_status asm_decode_step_search(const void *q, const void *q_search,
                                  const void *centroids, const void *a_bar,
                                  const float *logz_bar, const void *k_cache,
                                  const void *v_cache, const int32_t *local_len,
                                  int B, int Hq, int Hkv, int K, int Tmax, int d,
                                  float scale, asm_metric metric, asm_dtype dt,
                                  void *out, float *lse_out, int32_t *idx_out,
                                  unsigned flags, void *ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Utilities                                                                */
/* ------------------------------------------------------------------------ */

/* Zero a decode / flash-decode / k-means workspace (counters, error word). */
asm_status asm_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * asm_wait_spin_limit -- how many unsuccessful mbarrier try_wait polls any
 * wait in the library's kernels makes before it gives up, sets the error
 * word to ASM_ERR_TIMEOUT and lets its CTA finish.
 */
uint32_t asm_wait_spin_limit(void);

/*
 * asm_wait_selftest -- run the give-up path of a bounded wait on purpose: one
 * CTA waits on an mbarrier that nothing arrives at, `polls` try_wait polls
 * (0: the library's own bounded wait, asm_wait_spin_limit() polls), then
 * completes the barrier's phase itself.  No copy is in flight and no tensor
 * memory is held, so the context stays usable.
 *   ws          >= 256 bytes, 16-byte aligned: its error word (read with
 *               asm_workspace_error) is cleared, then set to ASM_ERR_TIMEOUT
 *               when the wait gives up
 *   elapsed_ns  host: how long the wait took (device %globaltimer)
 * Synchronises `stream`.  ASM_ERR_INVALID_ARG for polls < 0, a short or
 * misaligned ws, or a null elapsed_ns.
 */
asm_status asm_wait_selftest(int polls, void *ws, size_t ws_bytes, uint64_t *elapsed_ns,
                             cudaStream_t stream);

/* Error word of a decode / flash-decode / k-means / whitening workspace, copied to the host
 * pointer `code` (0 = no device-side error; otherwise ASM_ERR_TIMEOUT).
 * Synchronises `stream`. */
asm_status asm_workspace_error(const void *ws, size_t ws_bytes, int *code,
                               cudaStream_t stream);

/* The CUDA runtime's message for the last CUDA error behind an ASM_ERR_CUDA
 * returned on the calling thread ("no error" if there was none).  Static
 * storage, never NULL. */
const char *asm_last_cuda_error(void);

/* Static description of a status code (never NULL). */
const char *asm_status_string(asm_status s);

/* Library version, "major.minor.patch". */
const char *asm_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ASM_B200_H */
