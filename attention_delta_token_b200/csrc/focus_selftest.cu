// focus_selftest.cu -- focus_selftest_wait_timeout: exercises the library's
// bounded mbarrier wait on a barrier that nothing ever arrives at.
//
// Every wait in the eviction kernels is bounded: when its limit passes it sets
// FOCUS_DEV_TIMEOUT in the device status word and returns false, and the kernel
// unwinds instead of hanging the GPU.  This entry point runs that same wait on a
// barrier with no arrivals, so tests can check the timeout path end to end on a
// real device without faulting, trapping or hanging it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "focus.h"
#include "focus_device.cuh"

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t *status, uint64_t limit_ns,
                                                          unsigned long long *elapsed_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        focus::mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        focus::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = focus::global_timer_ns();
        const bool ok = focus::mbar_wait(&bar, 0, status, &abort_flag, limit_ns);
        *elapsed_ns = focus::global_timer_ns() - t0;
        if (ok) atomicOr(status, 0x80000000u);  // would mean the barrier completed: a bug
    }
}

}  // namespace

extern "C" focus_status_t focus_selftest_wait_timeout(uint32_t *status, uint64_t limit_ns,
                                                      unsigned long long *elapsed_ns,
                                                      void *stream) {
    if (!status || !elapsed_ns || (reinterpret_cast<uintptr_t>(status) & 3u) ||
        (reinterpret_cast<uintptr_t>(elapsed_ns) & 7u))
        return FOCUS_ERR_INVALID_ARGUMENT;
    if (limit_ns == 0 || limit_ns > FOCUS_WAIT_LIMIT_NS) return FOCUS_ERR_INVALID_ARGUMENT;
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, limit_ns,
                                                                       elapsed_ns);
    return cudaGetLastError() == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
}
