// selftest.cu -- the device-side timeout path, made to run out on purpose.
//
// Every mbarrier wait of the library is bounded (mbar_wait gives up after
// kSpinLimit unsuccessful try_wait polls) and reports ASM_ERR_TIMEOUT in the
// caller's error word instead of hanging.  This kernel waits on an mbarrier
// that nothing ever arrives at -- the one way to exercise that path without
// a fault -- records how long the wait took, and then completes the phase
// itself so that the CTA leaves the barrier settled.  No copy is in flight
// and no tensor memory is held, so giving up is clean.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace asmk {

__device__ __forceinline__ unsigned long long wall_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// polls > 0: that many try_wait polls; polls == 0: the library's mbar_wait.
__global__ void wait_selftest_kernel(int polls, int *err, unsigned long long *elapsed_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = wall_ns();
    bool done = false;
    if (polls == 0) {
        done = mbar_wait(&bar, 0);
    } else {
        for (int i = 0; i < polls && !done; ++i) done = mbar_try_wait(&bar, 0);
    }
    *elapsed_ns = wall_ns() - t0;
    if (!done) atomicExch(err, (int)ASM_ERR_TIMEOUT);
    mbar_arrive(&bar);  // the phase nobody completed
}

}  // namespace asmk

cudaError_t asm_selftest_wait_launch(int polls, int *err, unsigned long long *elapsed_ns, cudaStream_t st) {
    asmk::wait_selftest_kernel<<<1, 32, 0, st>>>(polls, err, elapsed_ns);
    return cudaGetLastError();
}

uint32_t asm_wait_spin_limit_value() { return asmk::kSpinLimit; }
