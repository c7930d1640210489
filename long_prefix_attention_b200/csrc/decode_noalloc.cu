// decode_noalloc.cu -- asm_decode_step for callers that cannot allocate.
//
// Some callers have no way to obtain device memory at the point where they
// decode: a plug-in running inside a host framework that owns every device
// allocation and offers none to extensions, or a latency-critical loop where
// cudaMalloc is not allowed because it can synchronise the device.  For them
// this entry point takes its scratch from one fixed array compiled into the
// library instead of a caller-provided workspace.
//
// The array below is a file-scope __device__ variable: every GPU that loads
// the library holds it, zero-initialised, until the process exits.  In host
// code its name is only a host-side stand-in, so its device address is
// fetched once per device with cudaGetSymbolAddress (with that device
// current) and the decode kernel is given that address.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "asm.h"
#include "launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of g_decode_scratch on the current device (set up on the
// first call for that device), or nullptr on failure.
void *scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" asm_status asm_decode_step_noalloc(const void *q, const void *centroids, const void *a_bar,
                                              const float *logz_bar, const void *k_cache,
                                              const void *v_cache, const int32_t *local_len, int B,
                                              int Hq, int Hkv, int K, int Tmax, int d, float scale,
                                              asm_metric metric, asm_dtype dt, void *out, float *lse_out,
                                              int32_t *idx_out, unsigned flags, cudaStream_t stream) {
    // every argument is checked before anything touches the stream
    const asm_status v = asm_decode_check_args(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, B, Hq,
                                               Hkv, K, Tmax, d, scale, (int)metric, dt, out, lse_out, idx_out, flags);
    if (v != ASM_OK) return v;
    const size_t need = asm_decode_workspace_size(B, Hq, Hkv, K, Tmax, d, dt);
    if (need == 0) return ASM_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return ASM_ERR_WORKSPACE;  // beyond the fixed scratch
    void *ws = scratch_on_current_device();
    if (ws == nullptr) return ASM_ERR_CUDA;
    // The array keeps the previous call's contents: clear the error word (and
    // for fp32 the arrival counters), which must start at zero.
    if (cudaMemsetAsync(ws, 0, asm_decode_ws_header_bytes(B, Hkv, dt), stream) != cudaSuccess) return ASM_ERR_CUDA;
    return asm_decode_step(q, centroids, a_bar, logz_bar, k_cache, v_cache, local_len, B, Hq, Hkv, K, Tmax, d,
                           scale, metric, dt, out, lse_out, idx_out, flags, ws, kNoAllocScratchBytes, stream);
}

// The error word of the built-in scratch on the current device: the device-side
// status of the last asm_decode_step_noalloc call there.
extern "C" asm_status asm_decode_noalloc_error(int *code, cudaStream_t stream) {
    if (code == nullptr) return ASM_ERR_INVALID_ARG;
    void *ws = scratch_on_current_device();
    if (ws == nullptr) return ASM_ERR_CUDA;
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return ASM_ERR_CUDA;
    *code = v;
    return ASM_OK;
}
