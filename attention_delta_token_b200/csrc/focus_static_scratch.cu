// focus_static_scratch.cu -- focus_evict_static_scratch: the fused eviction step
// for callers that cannot allocate device memory.
//
// focus_evict needs a caller-provided workspace (device status word, request
// order, per-kv-head column sums).  Some callers cannot provide one: a serving
// engine that reserved nearly all HBM for its KV cache at start-up and must not
// ask the allocator for more while it decodes, or a plug-in that reaches the GPU
// through this C ABI alone and has no access to its host framework's memory
// pool (a raw cudaMalloc there would also synchronise the device).  This entry
// point keeps that scratch in a fixed array that the library itself owns in
// device memory (FOCUS_STATIC_SCRATCH_BYTES, 8 MiB, held by every GPU that loads
// the library until the process exits), so the caller passes only inputs and
// outputs.  It then runs exactly the focus_evict kernels on that array.
#include <cuda_runtime.h>
#include <stdint.h>

#include <string.h>

#include <mutex>

#include "focus.h"

namespace focus {
// The fused step's host validation (focus_api.cu): every check focus_evict_ex makes
// before it enqueues work, with nothing enqueued.
focus_status_t evict_check(const focus_dims_t *dims, const focus_evict_args_t *args);
}  // namespace focus

namespace {

// The scratch array.  In host code `g_scratch` is only a host-side handle for
// the symbol; its device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_scratch[FOCUS_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per device and
// kept for the life of the process.  A cudaDeviceReset (or anything else that tears
// down and rebuilds the device's primary context) reloads the module and may move the
// array, so the library must not be used on a device across such a reset.
focus_status_t scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return FOCUS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return FOCUS_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return FOCUS_OK;
}

}  // namespace

extern "C" focus_status_t focus_evict_static_scratch(
    const focus_dims_t *dims, const void *q0, const void *k0_prefix, const void *k0_block,
    const void *q1, const void *k1_prefix, const void *k1_block, const int32_t *cu_prefix,
    int64_t total_prefix, const void *hidden, const uint8_t *decoded, const int32_t *budget,
    int32_t *kept_idx, int32_t *cu_seqlens, void *packed, int64_t capacity, float *delta_out,
    float *i0_out, float *i1_out, uint32_t *device_status, void *stream) {
    const size_t need = focus_workspace_size(dims);
    if (need == 0)  // invalid dims: let the shared validation name the problem, no CUDA call
        return focus_evict(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix,
                           total_prefix, hidden, decoded, budget, kept_idx, cu_seqlens, packed,
                           capacity, delta_out, i0_out, i1_out, nullptr, 0, stream);
    if (need > FOCUS_STATIC_SCRATCH_BYTES) return FOCUS_ERR_WORKSPACE;
    if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u))
        return FOCUS_ERR_INVALID_ARGUMENT;

    void *scratch = nullptr;
    focus_status_t st = scratch_address(&scratch);
    if (st != FOCUS_OK) return st;
    focus_evict_args_t x;
    memset(&x, 0, sizeof x);
    x.q0 = q0;
    x.k0_prefix = k0_prefix;
    x.k0_block = k0_block;
    x.q1 = q1;
    x.k1_prefix = k1_prefix;
    x.k1_block = k1_block;
    x.cu_prefix = cu_prefix;
    x.total_prefix = total_prefix;
    x.hidden = hidden;
    x.decoded = decoded;
    x.budget = budget;
    x.kept_idx = kept_idx;
    x.cu_seqlens = cu_seqlens;
    x.packed = packed;
    x.capacity = capacity;
    x.delta_out = delta_out;
    x.i0_out = i0_out;
    x.i1_out = i1_out;
    x.workspace = scratch;
    x.workspace_bytes = FOCUS_STATIC_SCRATCH_BYTES;
    x.stream = stream;
    // Every argument is checked before anything is enqueued: a call that is refused
    // leaves the array, and the status word another call may still report, untouched.
    st = focus::evict_check(dims, &x);
    if (st != FOCUS_OK) return st;
    // The array keeps the previous call's contents; only the status word must
    // start at zero (everything else is fully rewritten before it is read).
    st = focus_clear_device_status(scratch, FOCUS_STATIC_SCRATCH_BYTES, stream);
    if (st != FOCUS_OK) return st;
    st = focus_evict_ex(dims, &x);
    if (st != FOCUS_OK) return st;
    if (device_status &&
        cudaMemcpyAsync(device_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return FOCUS_ERR_CUDA;
    return FOCUS_OK;
}
