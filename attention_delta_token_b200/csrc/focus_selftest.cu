// focus_selftest.cu -- self-tests of device mechanisms that a normal call cannot
// reach on one GPU.
//
// focus_selftest_wait_timeout: exercises the library's bounded mbarrier wait on a
// barrier that nothing ever arrives at.
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
#include "focus_exchange.cuh"

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

// focus_selftest_exchange: `world` ranks emulated by block groups of ONE
// cooperative launch (blockIdx.z = rank; every block resident, so a block may
// wait for flags that other blocks raise).  Each block pushes one (layer,
// request) row of its rank's sums, the rank's last block raises its flags, then
// each block waits for its rank's buffer to hold every rank's row and writes the
// rank-ordered sum -- the push, signal, wait and summation of the real kernels.
__global__ void __launch_bounds__(128) exchange_selftest_kernel(const float *partials,
                                                                void *const *bufs, float *out,
                                                                uint32_t *scratch, int R, int B,
                                                                int W, uint32_t epoch) {
    const int r = blockIdx.x, l = blockIdx.y, rank = blockIdx.z, j = threadIdx.x;
    const size_t row = (static_cast<size_t>(rank) * 2 + l) * R * B + static_cast<size_t>(r) * B;
    if (j < B) focus::ex_push(bufs, R, B, W, rank, epoch, l, r, j, partials[row + j]);
    const size_t flags_off = focus::ex_layout(R, B, W).flags;
    focus::ex_signal(bufs, flags_off, W, rank, epoch, scratch + 1 + rank, gridDim.x * gridDim.y);
    const uint8_t *mine = static_cast<const uint8_t *>(bufs[rank]);
    focus::ex_wait(reinterpret_cast<const uint32_t *>(mine + flags_off), W, epoch, scratch);
    if (j < B) {
        const float *slots = reinterpret_cast<const float *>(mine);
        float s = 0.f;
        for (int q = 0; q < W; ++q) s += __ldcg(slots + focus::ex_index(R, B, W, epoch, l, r, q, j));
        out[row + j] = s;
    }
}

}  // namespace

extern "C" focus_status_t focus_selftest_exchange(const float *partials, void *const *buffers,
                                                  float *out, uint32_t *scratch, int32_t R,
                                                  int32_t B, int32_t world, uint32_t epoch,
                                                  void *stream) {
    if (!partials || !buffers || !out || !scratch || (reinterpret_cast<uintptr_t>(partials) & 3u) ||
        (reinterpret_cast<uintptr_t>(buffers) & 7u) || (reinterpret_cast<uintptr_t>(out) & 3u) ||
        (reinterpret_cast<uintptr_t>(scratch) & 3u))
        return FOCUS_ERR_INVALID_ARGUMENT;
    if (R < 1 || B < 1 || B > 128 || world < 1 || world > focus::kMaxExchangeWorld || epoch == 0 ||
        static_cast<long long>(R) * 2 * world > 1024)
        return FOCUS_ERR_INVALID_ARGUMENT;
    void *args[] = {&partials, &buffers, &out, &scratch, &R, &B, &world, &epoch};
    const cudaError_t e = cudaLaunchCooperativeKernel(
        reinterpret_cast<const void *>(exchange_selftest_kernel),
        dim3(static_cast<unsigned>(R), 2, static_cast<unsigned>(world)), dim3(128), args, 0,
        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
}

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
