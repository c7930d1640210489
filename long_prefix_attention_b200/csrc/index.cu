// index.cu -- order a memory by the clusters of its two-level index.
//
// "Context Memorization for Efficient Long Context Generation", Complejidad:
// retrieval through a hierarchical index.  The K centres of each head are
// clustered (the library's k-means run on the centres); this gather puts the
// members of every cluster in consecutive rows, so the second level of the
// search reads each kept cluster as one contiguous range:
//   row i of head h  <-  row perm[h, i] of the flat memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

// One warp per output row: D elements of the centre and of the state, 16-byte chunks.
template <typename T, int D>
__global__ void index_reorder_kernel(const int32_t *__restrict__ perm, int H, int K, const T *__restrict__ c,
                                     const T *__restrict__ abar, const float *__restrict__ lz, T *c_out, T *abar_out,
                                     float *lz_out) {
    constexpr int CH = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
    const long w = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long)H * K) return;
    const int h = (int)(w / K);
    const int src = perm[w];
    const size_t si = ((size_t)h * K + src) * D, di = (size_t)w * D;
    for (int i = lane; i < CH; i += 32) {
        reinterpret_cast<uint4 *>(c_out + di)[i] = __ldg(reinterpret_cast<const uint4 *>(c + si) + i);
        reinterpret_cast<uint4 *>(abar_out + di)[i] = __ldg(reinterpret_cast<const uint4 *>(abar + si) + i);
    }
    if (lane == 0) lz_out[w] = lz[(size_t)h * K + src];
}

}  // namespace asmk

cudaError_t asm_index_reorder_launch(const int32_t *perm, int H, int K, int d, asm_dtype dt, const void *c,
                                     const void *abar, const float *lz, void *c_out, void *abar_out, float *lz_out,
                                     cudaStream_t st) {
    using namespace asmk;
    const long rows = (long)H * K;
    const unsigned nb = (unsigned)((rows * 32 + 255) / 256);
    if (dt == ASM_BF16) {
        using T = __nv_bfloat16;
        if (d == 128)
            index_reorder_kernel<T, 128><<<nb, 256, 0, st>>>(perm, H, K, (const T *)c, (const T *)abar, lz, (T *)c_out,
                                                             (T *)abar_out, lz_out);
        else
            index_reorder_kernel<T, 64><<<nb, 256, 0, st>>>(perm, H, K, (const T *)c, (const T *)abar, lz, (T *)c_out,
                                                            (T *)abar_out, lz_out);
    } else {
        if (d == 128)
            index_reorder_kernel<float, 128><<<nb, 256, 0, st>>>(perm, H, K, (const float *)c, (const float *)abar, lz,
                                                                 (float *)c_out, (float *)abar_out, lz_out);
        else
            index_reorder_kernel<float, 64><<<nb, 256, 0, st>>>(perm, H, K, (const float *)c, (const float *)abar, lz,
                                                                (float *)c_out, (float *)abar_out, lz_out);
    }
    return cudaGetLastError();
}
