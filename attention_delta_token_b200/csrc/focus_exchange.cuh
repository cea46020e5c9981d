// focus_exchange.cuh -- device side of the peer exchange of partial importance.
//
// In a head-sharded (tensor-parallel) group every rank computes I over its own
// heads; the ranks need the sum.  Instead of a separate all-reduce, the kernel
// that reduces a rank's column sums stores them straight into every rank's
// exchange buffer (peer-mapped device memory: over NVLink for other GPUs), and
// the selection kernel of each rank waits for all ranks' flags and sums the
// slots in rank order -- so every rank gets bit-identical sums and keeps the
// same tokens.
//
// Buffer of one rank (layout in ex_layout, focus_kernels.cuh):
//   slots [2 parities][2 layers][R][world][B] float32
//   flags [2 parities][world] uint32
// Step `epoch` (>= 1, +1 per step, the same on every rank) uses parity epoch & 1:
// rank q writes slot [p][l][r][q][:] of every buffer, and once all of its stores
// are done, flag [p][q] = epoch in every buffer.  Two parities suffice: a rank
// can only push step e + 2 after its selection of step e + 1, which waited for
// every rank's push of step e + 1, which each rank issued after finishing its
// own selection of step e (stream order) -- so nobody overwrites slots that are
// still being read.
#pragma once

#include "focus_device.cuh"
#include "focus_kernels.cuh"

namespace focus {

__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Index (in floats) of element (l, r, src, j) of the epoch's slots.
__device__ __forceinline__ size_t ex_index(int R, int B, int W, uint32_t epoch, int l, int r,
                                           int src, int j) {
    return (((static_cast<size_t>(epoch & 1u) * 2 + l) * R + r) * W + src) * B + j;
}

// Stores this rank's value of (l, r, j) into the slot `rank` of every rank's buffer.
__device__ __forceinline__ void ex_push(void *const *bufs, int R, int B, int W, int rank,
                                        uint32_t epoch, int l, int r, int j, float v) {
    const size_t i = ex_index(R, B, W, epoch, l, r, rank, j);
    for (int q = 0; q < W; ++q) static_cast<float *>(bufs[q])[i] = v;
}

__device__ __forceinline__ void fence_acq_rel_sys() {
    asm volatile("fence.acq_rel.sys;" ::: "memory");
}

// Every thread of every block of the pushing grid calls this after its stores.
// The block that finishes last (counted on `counter`, which it resets for the
// next launch) raises flag [epoch & 1][rank] = epoch in every rank's buffer.
// Release pattern: the barrier orders the block's peer stores before thread 0's
// system-scope fence, which with the relaxed count releases them; the last
// block's fence after its count acquires every counted block's release, and its
// release store of the flag carries them all to the rank that reads the flag.
__device__ __forceinline__ void ex_signal(void *const *bufs, size_t flags_off, int W, int rank,
                                          uint32_t epoch, unsigned int *counter,
                                          unsigned int n_blocks) {
    __syncthreads();
    if (threadIdx.x == 0) {
        fence_acq_rel_sys();
        if (atomicAdd(counter, 1u) == n_blocks - 1) {
            *counter = 0;
            fence_acq_rel_sys();
            for (int q = 0; q < W; ++q) {
                uint32_t *flags =
                    reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(bufs[q]) + flags_off);
                st_release_sys(flags + (epoch & 1u) * W + rank, epoch);
            }
        }
    }
}

// Thread 0 waits until every rank's flag of this parity in `flags` (this rank's
// own buffer) shows `epoch`; bounded by FOCUS_WAIT_LIMIT_NS and an iteration cap,
// after which FOCUS_DEV_TIMEOUT is set in *status.  Block-wide: every thread
// must call it; returns after a barrier, true when all flags arrived.
__device__ __forceinline__ bool ex_wait(const uint32_t *flags, int W, uint32_t epoch,
                                        uint32_t *status) {
    __shared__ int ok_s;
    if (threadIdx.x == 0) {
        int ok = 1;
        const uint64_t t0 = global_timer_ns();
        uint32_t it = 0;
        for (int q = 0; q < W && ok; ++q) {
            while (ld_acquire_sys(flags + (epoch & 1u) * W + q) != epoch) {
                if (++it > (1u << 26) || global_timer_ns() - t0 > FOCUS_WAIT_LIMIT_NS) {
                    atomicOr(status, FOCUS_DEV_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        ok_s = ok;
    }
    __syncthreads();
    return ok_s != 0;
}

}  // namespace focus
