// whiten.cu -- ZCA whitening of the retrieval vectors.
//
// "Context Memorization for Efficient Long Context Generation", Fase de
// Inferencia Online, Recuperacion: the retrieval may whiten the vectors
// first; the pages give no recipe.  Reading: ZCA whitening from each head's
// calibration queries, W = (C + eps I)^(-1/2) with C the (1/N) covariance and
// eps = eps_rel * trace(C) / d, applied to a vector as y = W (x - mu).
//
//   whiten_moments   column sums and second moments of a head's points in
//                    fp64 (products of bf16 or fp32 values are exact in fp64),
//                    accumulated over blocks of rows with fp64 atomics
//   whiten_invsqrt   one CTA per head: C, eps, then the coupled Newton-Schulz
//                    iteration Y <- Y T, Z <- T Z with T = (3I - Z Y) / 2,
//                    from Y = A / s, Z = I (s = |A|_F, so the spectrum of A / s
//                    lies in (0, 1]); Z -> (A / s)^(-1/2), W = Z / sqrt(s).
//                    fp64 throughout; the iteration stops when
//                    max |I - Z Y| < 1e-13 and flags an error if it has not
//                    after kMaxIter iterations.
//   whiten_apply     y = (x - mu) W for rows given by a head stride and a row
//                    stride (W is symmetric), fp32 accumulation, output in the
//                    storage type; whiten_apply_small for a few rows per head
//                    (decode queries).
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {
namespace wh {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = 2048;  // rows of one head per moments block
constexpr int kStage = 16;           // rows staged in shared memory at a time
constexpr int kMaxIter = 100;
constexpr double kTol = 1e-13;

// ---------------------------------------------------------------- moments --
// Thread (ti, tj) of a 16 x 16 grid owns the TL x TL tile (TL = D / 16) of the
// second-moment matrix at rows ti * TL, columns tj * TL.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
whiten_moments(const T *__restrict__ x, int N, double *S, double *colsum) {
    constexpr int TL = D / 16;
    const int h = blockIdx.y, tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
    const int r0 = blockIdx.x * kRowsPerBlock, r1 = min(N, r0 + kRowsPerBlock);
    const T *xh = x + (size_t)h * N * D;
    __shared__ double xs[kStage][D];
    double acc[TL][TL];
#pragma unroll
    for (int i = 0; i < TL; ++i)
#pragma unroll
        for (int j = 0; j < TL; ++j) acc[i][j] = 0.0;
    double cs = 0.0;  // column tid's sum (tid < D)
    for (int rb = r0; rb < r1; rb += kStage) {
        const int nr = min(kStage, r1 - rb);
        for (int e = tid; e < kStage * D; e += kThreads) {
            const int rr = e / D, cc = e % D;
            xs[rr][cc] = rr < nr ? (double)Elem<T>::to_f(xh[(size_t)(rb + rr) * D + cc]) : 0.0;
        }
        __syncthreads();
        for (int rr = 0; rr < nr; ++rr) {
            double a[TL], b[TL];
#pragma unroll
            for (int i = 0; i < TL; ++i) a[i] = xs[rr][ti * TL + i];
#pragma unroll
            for (int j = 0; j < TL; ++j) b[j] = xs[rr][tj * TL + j];
#pragma unroll
            for (int i = 0; i < TL; ++i)
#pragma unroll
                for (int j = 0; j < TL; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
            if (tid < D) cs += xs[rr][tid];
        }
        __syncthreads();
    }
    double *Sh = S + (size_t)h * D * D;
#pragma unroll
    for (int i = 0; i < TL; ++i)
#pragma unroll
        for (int j = 0; j < TL; ++j) atomicAdd(&Sh[(ti * TL + i) * D + tj * TL + j], acc[i][j]);
    if (tid < D) atomicAdd(&colsum[(size_t)h * D + tid], cs);
}

// --------------------------------------------------- CTA-wide fp64 GEMM ----
// C = A B for D x D row-major matrices in global memory; thread (ti, tj) of a
// 16 x 16 grid computes the TL x TL tile at rows ti * TL, columns tj * TL.
template <int D>
__device__ void gemm_cta(const double *A, const double *B, double (&acc)[D / 16][D / 16], double *As,
                         double *Bs) {
    constexpr int TL = D / 16, KC = 16;
    const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
#pragma unroll
    for (int i = 0; i < TL; ++i)
#pragma unroll
        for (int j = 0; j < TL; ++j) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < D; k0 += KC) {
        // As[k][row] (k-major) and Bs[k][col]
        for (int e = tid; e < D * KC; e += kThreads) {
            const int row = e / KC, k = e % KC;
            As[k * D + row] = A[row * D + k0 + k];
            const int kb = e / D, col = e % D;
            Bs[kb * D + col] = B[(k0 + kb) * D + col];
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < KC; ++k) {
            double a[TL], b[TL];
#pragma unroll
            for (int i = 0; i < TL; ++i) a[i] = As[k * D + ti * TL + i];
#pragma unroll
            for (int j = 0; j < TL; ++j) b[j] = Bs[k * D + tj * TL + j];
#pragma unroll
            for (int i = 0; i < TL; ++i)
#pragma unroll
                for (int j = 0; j < TL; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
}

__device__ __forceinline__ double block_max_d(double v, double *sh) {
    for (int m = 16; m >= 1; m >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, m));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
    __syncthreads();
    double r = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) r = fmax(r, sh[w]);
    return r;
}
__device__ __forceinline__ double block_sum_d(double v, double *sh) {
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
    __syncthreads();
    double r = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) r += sh[w];
    return r;
}

// ------------------------------------------------------------ inverse root --
// scratch per head: Y0, Z0, Y1, Z1, Tm (D x D fp64 each)
template <int D>
__global__ void __launch_bounds__(kThreads)
whiten_invsqrt(const double *S, const double *colsum, int N, float eps_rel, double *scratch, float *mu_out,
               float *w_out, int *err) {
    constexpr int TL = D / 16, DD = D * D;
    const int h = blockIdx.x, tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
    extern __shared__ double wsm[];
    double *As = wsm, *Bs = wsm + D * 16;
    __shared__ double sh[kThreads / 32];
    __shared__ double mus[D];
    double *Y = scratch + (size_t)h * 5 * DD, *Z = Y + DD, *Y2 = Z + DD, *Z2 = Y2 + DD, *Tm = Z2 + DD;
    const double *Sh = S + (size_t)h * DD;
    const double inv_n = 1.0 / (double)N;
    for (int i = tid; i < D; i += kThreads) {
        mus[i] = colsum[(size_t)h * D + i] * inv_n;
        mu_out[(size_t)h * D + i] = (float)mus[i];
    }
    __syncthreads();
    // A = S / N - mu mu^T + eps I, eps = eps_rel * trace(C) / D; s = |A|_F
    double tr = 0.0;
    for (int i = tid; i < D; i += kThreads) tr += Sh[i * D + i] * inv_n - mus[i] * mus[i];
    tr = block_sum_d(tr, sh);
    const double eps = (double)eps_rel * tr / D;
    double fro = 0.0;
    for (int e = tid; e < DD; e += kThreads) {
        const int i = e / D, j = e % D;
        const double a = Sh[e] * inv_n - mus[i] * mus[j] + (i == j ? eps : 0.0);
        Y[e] = a;
        fro += a * a;
    }
    fro = sqrt(block_sum_d(fro, sh));
    const double sc = fro > 0.0 ? fro : 1.0;
    for (int e = tid; e < DD; e += kThreads) {
        Y[e] /= sc;
        Z[e] = (e / D == e % D) ? 1.0 : 0.0;
    }
    __syncthreads();
    double acc[TL][TL];
    bool done = false;
    for (int it = 0; it < kMaxIter && !done; ++it) {
        // Tm = (3I - Z Y) / 2, and the distance of Z Y from I
        gemm_cta<D>(Z, Y, acc, As, Bs);
        double dev = 0.0;
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int j = 0; j < TL; ++j) {
                const int r = ti * TL + i, c = tj * TL + j;
                const double id = r == c ? 1.0 : 0.0;
                dev = fmax(dev, fabs(id - acc[i][j]));
                Tm[r * D + c] = 0.5 * (3.0 * id - acc[i][j]);
            }
        dev = block_max_d(dev, sh);  // also orders the Tm stores before the reads below
        if (dev < kTol) {
            done = true;
            break;
        }
        gemm_cta<D>(Y, Tm, acc, As, Bs);
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int j = 0; j < TL; ++j) Y2[(ti * TL + i) * D + tj * TL + j] = acc[i][j];
        gemm_cta<D>(Tm, Z, acc, As, Bs);
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int j = 0; j < TL; ++j) Z2[(ti * TL + i) * D + tj * TL + j] = acc[i][j];
        __syncthreads();
        double *t = Y;
        Y = Y2;
        Y2 = t;
        t = Z;
        Z = Z2;
        Z2 = t;
    }
    if (!done && tid == 0) atomicExch(err, (int)ASM_ERR_TIMEOUT);
    const double rs = 1.0 / sqrt(sc);
    float *Wh = w_out + (size_t)h * DD;
    for (int e = tid; e < DD; e += kThreads) {
        // symmetrise the rounding of the iteration
        const int i = e / D, j = e % D;
        Wh[e] = (float)(0.5 * (Z[i * D + j] + Z[j * D + i]) * rs);
    }
}

// ------------------------------------------------------------------ apply --
// Block: one head, kApplyRows rows at a time; W in shared memory (fp32).
// Thread t computes row t / 8 of the 32-row tile, columns (t % 8) * D / 8.
constexpr int kApplyRows = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
whiten_apply(const T *__restrict__ x, int R, long long sh_in, long long sr_in, const float *__restrict__ mu,
             const float *__restrict__ w, T *y, long long sh_out, long long sr_out, int tiles_per_block) {
    constexpr int CW = D / 8;  // columns per thread
    extern __shared__ float asm_wsm[];
    float *Ws = asm_wsm;                 // [D][D]
    float *xs = asm_wsm + D * D;         // [kApplyRows][D] centred rows
    const int h = blockIdx.y, tid = threadIdx.x;
    for (int e = tid; e < D * D; e += kThreads) Ws[e] = w[(size_t)h * D * D + e];
    const float *muh = mu + (size_t)h * D;
    const int row = tid / 8, c0 = (tid % 8) * CW;
    for (int tb = 0; tb < tiles_per_block; ++tb) {
        const int base = (blockIdx.x * tiles_per_block + tb) * kApplyRows;
        if (base >= R) break;
        __syncthreads();
        for (int e = tid; e < kApplyRows * D; e += kThreads) {
            const int rr = e / D, cc = e % D;
            const int r = base + rr;
            xs[e] = r < R ? Elem<T>::to_f(x[h * sh_in + (long long)r * sr_in + cc]) - muh[cc] : 0.f;
        }
        __syncthreads();
        float acc[CW];
#pragma unroll
        for (int j = 0; j < CW; ++j) acc[j] = 0.f;
        for (int k = 0; k < D; ++k) {
            const float xv = xs[row * D + k];
#pragma unroll
            for (int j = 0; j < CW; ++j) acc[j] = fmaf(xv, Ws[k * D + c0 + j], acc[j]);
        }
        const int r = base + row;
        if (r < R) {
#pragma unroll
            for (int j = 0; j < CW; ++j) y[h * sh_out + (long long)r * sr_out + c0 + j] = Elem<T>::from_f(acc[j]);
        }
    }
}

// Few rows (decode queries): one block of 4 x D threads per head.  Thread
// (kq, j) holds column j of W over the quarter kq of the input dimension in
// registers (all its loads in flight at once), forms its partial dot product
// for every row, and the four partials are added in a fixed order.  Chained by
// programmatic dependent launch like the decode kernels.
constexpr int kSmallRows = 64;

template <typename T, int D>
__global__ void __launch_bounds__(4 * D)
whiten_apply_small(const T *__restrict__ x, int R, long long sh_in, long long sr_in, const float *__restrict__ mu,
                   const float *__restrict__ w, T *y, long long sh_out, long long sr_out) {
    constexpr int KQ = D / 4;
    const int h = blockIdx.x, t = threadIdx.x, kq = t / D, j = t % D;
    __shared__ float xs[kSmallRows][D];
    __shared__ float part[4][D];
    // W and mu may be written by the preceding kernel (asm_whitening): read
    // after the dependency wait like x
    pdl_wait();
    pdl_launch_dependents();
    float wr[KQ];
    const float *Wh = w + (size_t)h * D * D;
#pragma unroll
    for (int i = 0; i < KQ; ++i) wr[i] = Wh[(size_t)(kq * KQ + i) * D + j];
    for (int e = t; e < R * D; e += 4 * D) {
        const int r = e / D, c = e % D;
        xs[r][c] = Elem<T>::to_f(x[h * sh_in + (long long)r * sr_in + c]) - mu[(size_t)h * D + c];
    }
    __syncthreads();
    for (int r = 0; r < R; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < KQ; ++i) acc = fmaf(xs[r][kq * KQ + i], wr[i], acc);
        part[kq][j] = acc;
        __syncthreads();
        if (kq == 0) {
            const float v = ((part[0][j] + part[1][j]) + part[2][j]) + part[3][j];
            y[h * sh_out + (long long)r * sr_out + j] = Elem<T>::from_f(v);
        }
        __syncthreads();
    }
}

}  // namespace wh
}  // namespace asmk

using namespace asmk;

size_t asm_whitening_ws_bytes(int H, int d) {
    const size_t dd = (size_t)d * d;
    // error word, S, column sums, Newton-Schulz scratch (5 matrices)
    return 256 + sizeof(double) * ((size_t)H * dd + (size_t)H * d + (size_t)H * 5 * dd);
}

cudaError_t asm_whitening_launch(const void *x, int H, int N, int d, asm_dtype dt, float eps_rel, float *mu,
                                 float *W, void *ws, cudaStream_t st) {
    char *b = static_cast<char *>(ws);
    int *err = reinterpret_cast<int *>(b);
    double *S = reinterpret_cast<double *>(b + 256);
    double *colsum = S + (size_t)H * d * d;
    double *scratch = colsum + (size_t)H * d;
    cudaError_t e = cudaMemsetAsync(b, 0, 256 + sizeof(double) * ((size_t)H * d * d + (size_t)H * d), st);
    if (e != cudaSuccess) return e;
    dim3 g1((N + wh::kRowsPerBlock - 1) / wh::kRowsPerBlock, H);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128) wh::whiten_moments<T, 128><<<g1, wh::kThreads, 0, st>>>((const T *)x, N, S, colsum);
        else wh::whiten_moments<T, 64><<<g1, wh::kThreads, 0, st>>>((const T *)x, N, S, colsum);
    } else {
        if (d == 128) wh::whiten_moments<float, 128><<<g1, wh::kThreads, 0, st>>>((const float *)x, N, S, colsum);
        else wh::whiten_moments<float, 64><<<g1, wh::kThreads, 0, st>>>((const float *)x, N, S, colsum);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem = sizeof(double) * 2 * d * 16;
    if (d == 128) wh::whiten_invsqrt<128><<<H, wh::kThreads, smem, st>>>(S, colsum, N, eps_rel, scratch, mu, W, err);
    else wh::whiten_invsqrt<64><<<H, wh::kThreads, smem, st>>>(S, colsum, N, eps_rel, scratch, mu, W, err);
    return cudaGetLastError();
}

namespace {
template <typename T, int D>
cudaError_t apply_t(const T *x, int H, int R, long long shi, long long sri, const float *mu, const float *W, T *y,
                    long long sho, long long sro, cudaStream_t st) {
    if (R <= wh::kSmallRows) {
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(H);
        cfg.blockDim = dim3(4 * D);
        cfg.stream = st;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, wh::whiten_apply_small<T, D>, x, R, shi, sri, mu, W, y, sho, sro);
    }
    const size_t smem = sizeof(float) * ((size_t)D * D + (size_t)wh::kApplyRows * D);
    auto k = wh::whiten_apply<T, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (R + wh::kApplyRows - 1) / wh::kApplyRows;
    const int tpb = tiles >= 8 * 148 ? 8 : 1;  // large inputs: amortise the W load
    dim3 g((tiles + tpb - 1) / tpb, H);
    k<<<g, wh::kThreads, smem, st>>>(x, R, shi, sri, mu, W, y, sho, sro, tpb);
    return cudaGetLastError();
}
}  // namespace

cudaError_t asm_whiten_launch(const void *x, int H, int R, int d, asm_dtype dt, long long sh_in, long long sr_in,
                              const float *mu, const float *W, void *y, long long sh_out, long long sr_out,
                              cudaStream_t st) {
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        return d == 128 ? apply_t<T, 128>((const T *)x, H, R, sh_in, sr_in, mu, W, (T *)y, sh_out, sr_out, st)
                        : apply_t<T, 64>((const T *)x, H, R, sh_in, sr_in, mu, W, (T *)y, sh_out, sr_out, st);
    }
    return d == 128 ? apply_t<float, 128>((const float *)x, H, R, sh_in, sr_in, mu, W, (float *)y, sh_out, sr_out, st)
                    : apply_t<float, 64>((const float *)x, H, R, sh_in, sr_in, mu, W, (float *)y, sh_out, sr_out, st);
}
