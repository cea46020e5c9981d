// attn_stats.cu -- attention importance I_j on sm_100a (TMA + tcgen05 + TMEM).
//
// Method: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science
// review page), "What carries the argument": I_j is the column-wise sum of the
// softmax attention weights block token j receives from all query tokens of the
// block; the Referee Report's minor comment on Eq. (2) reads the softmax as
// row (query) wise.  Each query row's softmax runs over the request's prefix
// keys followed by its B block keys; I_j also sums over the query heads.
//
// One CTA handles one (layer, request, kv head, 128-row query tile) in a single
// pass over the keys:
//   warp 0      TMA producer: the Q tile once, then 128-key tiles of the prefix
//               and finally the block keys, through a 2-stage shared-memory ring;
//   warp 1      allocates TMEM and issues tcgen05.mma (M=128 rows, N=128 keys,
//               K=d, bf16 in, fp32 out) into two ping-pong TMEM S buffers;
//   warps 2-5   one TMEM lane (= one query row) per thread: online row max m
//               and sum-exp l over every key tile (exp2 on the SFU).  The block
//               tile comes last, so when it arrives m and l are final and the
//               row's weights p_ij = 2^(s_ij - m)/l of the B block columns are
//               formed straight from the same S values, without a second pass.
//               Column sums over the 128 rows (warp butterfly, then the four
//               warps in fixed order) go to `partial`; no float atomics, so the
//               result is deterministic and equal keys give bit-equal columns.
// Two CTAs fit on an SM (99 KB shared memory and 256 TMEM columns each), so one
// CTA's prologue/epilogue overlaps the other's streaming.
#include <math.h>

#include "focus_device.cuh"
#include "focus_kernels.cuh"

namespace focus {

namespace {

constexpr uint32_t kChunkBytes = kTileRows * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)

template <int HEAD_DIM>
struct AttnSmem {
    static constexpr int kChunks = HEAD_DIM / 64;
    static constexpr uint32_t kTileBytes = kChunkBytes * kChunks;
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kKOff = kTileBytes;
    static constexpr uint32_t kBarOff = kKOff + kStages * kTileBytes;
    static constexpr uint32_t kRedOff = kBarOff + 256;
    static constexpr uint32_t kBytes = kRedOff + 4 * 128 * sizeof(float);
    static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// Loads 32 TMEM columns of this thread's lane into v[OFF .. OFF+31].
template <int OFF>
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    float(&dst)[32] = *reinterpret_cast<float(*)[32]>(v + OFF);
    tmem_ld_32cols(taddr + OFF, dst);
}

// Sum of x[0..31] over the 32 lanes of the warp, transposed: lane c returns the
// sum of column c.  31 shuffles; every column is reduced with the same tree.
__device__ __forceinline__ float warp_colsum32(float *x, int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < off; ++k) {
            const float send = upper ? x[k] : x[k + off];
            const float keep = upper ? x[k + off] : x[k];
            x[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return x[0];
}

template <int HEAD_DIM>
__global__ void __launch_bounds__(kAttnThreads, 2)
attn_stats_kernel(const __grid_constant__ AttnParams p) {
    using S = AttnSmem<HEAD_DIM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem + S::kQOff;
    uint8_t *sK = smem + S::kKOff;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBarOff);
    uint64_t *full = bars;                 // [kStages] key tile landed
    uint64_t *empty = bars + kStages;      // [kStages] key tile consumed by the MMAs
    uint64_t *q_full = bars + 2 * kStages; // Q tile landed
    uint64_t *s_full = q_full + 1;         // [2] S buffer written by the MMAs
    uint64_t *s_empty = s_full + 2;        // [2] S buffer read out by the softmax warps
    uint64_t *red_bar = s_empty + 2;       // column partial sums of the 4 softmax warps ready
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *red = reinterpret_cast<float *>(smem + S::kRedOff);  // [4][128]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item
    const int per_req = p.n_layers * p.Hkv * p.MT;
    const int rank = blockIdx.x / per_req;
    int rem = blockIdx.x - rank * per_req;
    const int layer = rem / (p.Hkv * p.MT);
    rem -= layer * p.Hkv * p.MT;
    const int kvh = rem / p.MT;
    const int mt = rem - kvh * p.MT;
    const int r = p.order ? p.order[rank] : rank;

    int pstart = p.cu_prefix[r];
    int L = p.cu_prefix[r + 1] - pstart;
    if (pstart < 0 || L < 0 || static_cast<long long>(pstart) + L > p.total_prefix) {
        if (threadIdx.x == 0) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
        L = 0;
        pstart = 0;
    }
    const int n_pre = (L + kTileKeys - 1) / kTileKeys;
    const int n_tiles = n_pre + 1;  // + the block tile, always last

    // ---- setup
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(q_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 4);
        }
        mbar_init(red_bar, 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tm_q[layer]);
        tma_prefetch_desc(&p.tm_kp[layer]);
        tma_prefetch_desc(&p.tm_kb[layer]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ======================= TMA producer
        if (lane == 0) {
            // Key tiles of a single row tile are read once: stream them past L2.  With
            // several row tiles per kv head the siblings re-read them from L2.
            const uint64_t pol = p.MT == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
            mbar_arrive_expect_tx(q_full, S::kTileBytes);
#pragma unroll
            for (int c = 0; c < S::kChunks; ++c)
                tma_load_3d(sQ + c * kChunkBytes, &p.tm_q[layer], q_full, c * 64, kvh * p.G,
                            r * p.B + mt * p.tok_per_tile, pol);
            int last = -1;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % kStages;
                const uint32_t ph = (t / kStages) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, p.status, abort_flag)) break;
                uint8_t *dst = sK + s * S::kTileBytes;
                if (t < n_pre) {
                    mbar_arrive_expect_tx(&full[s], S::kTileBytes);
#pragma unroll
                    for (int c = 0; c < S::kChunks; ++c)
                        tma_load_3d(dst + c * kChunkBytes, &p.tm_kp[layer], &full[s], c * 64, kvh,
                                    pstart + t * kTileKeys, pol);
                } else {
                    mbar_arrive_expect_tx(&full[s], p.n_blk * 128 * S::kChunks);
#pragma unroll
                    for (int c = 0; c < S::kChunks; ++c)
                        tma_load_3d(dst + c * kChunkBytes, &p.tm_kb[layer], &full[s], c * 64, kvh,
                                    r * p.B, pol);
                }
                last = t;
            }
            // Drain: every copy this thread issued has landed before the CTA exits.
            mbar_wait_drain(q_full, 0);
            for (int t = last - kStages + 1; t <= last; ++t)
                if (t >= 0) mbar_wait_drain(&full[t % kStages], (t / kStages) & 1);
        }
    } else if (warp == 1) {
        // ======================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pre = umma_idesc_bf16_f32(kTileRows, kTileKeys);
            const uint32_t idesc_blk = umma_idesc_bf16_f32(kTileRows, p.n_blk);
            const uint32_t a_base = smem_u32(sQ);
            int last = -1;
            if (mbar_wait(q_full, 0, p.status, abort_flag)) {
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % kStages;
                    const uint32_t ph = (t / kStages) & 1;
                    const int buf = t & 1;
                    const uint32_t bph = (t >> 1) & 1;
                    if (!mbar_wait(&s_empty[buf], bph ^ 1, p.status, abort_flag)) break;
                    if (!mbar_wait(&full[s], ph, p.status, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t idesc = (t < n_pre) ? idesc_pre : idesc_blk;
                    const uint32_t d_tmem = tmem_base + buf * kTileKeys;
                    const uint32_t b_base = smem_u32(sK + s * S::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < HEAD_DIM / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
                        umma_bf16(d_tmem, umma_desc_sw128(a_base + off),
                                  umma_desc_sw128(b_base + off), idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                    umma_commit(&s_full[buf]);
                    last = t;
                }
            }
            // Drain: the last MMAs have finished writing TMEM.
            if (last >= 0) mbar_wait_drain(&s_full[last & 1], (last >> 1) & 1);
        }
    } else {
        // ======================= softmax statistics, one query row per thread
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const int rows_valid = min(kTileRows, p.G * p.B - mt * kTileRows);
        const float c = p.scale_log2;
        float m = -INFINITY;  // running max of the scaled logits (log2 domain)
        float l = 0.f;        // running sum of 2^(x - m)
        for (int t = 0; t < n_tiles; ++t) {
            const int buf = t & 1;
            const uint32_t bph = (t >> 1) & 1;
            if (!mbar_wait(&s_full[buf], bph, p.status, abort_flag)) break;
            tc_fence_after();
            const uint32_t ta = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                static_cast<uint32_t>(buf * kTileKeys);
            float v[kTileKeys];
            tmem_ld32<0>(ta, v);
            tmem_ld32<32>(ta, v);
            tmem_ld32<64>(ta, v);
            tmem_ld32<96>(ta, v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[buf]);

            if (t < n_pre) {
                const int nv = min(kTileKeys, L - t * kTileKeys);
                float mx = -INFINITY;
                if (nv == kTileKeys) {
#pragma unroll
                    for (int j = 0; j < kTileKeys; ++j) mx = fmaxf(mx, v[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < kTileKeys; ++j)
                        if (j < nv) mx = fmaxf(mx, v[j]);
                }
                const float m_new = fmaxf(m, mx * c);
                const float neg = -m_new;
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                if (nv == kTileKeys) {
#pragma unroll
                    for (int j = 0; j < kTileKeys; j += 4) {
                        a0 += ex2(fmaf(v[j + 0], c, neg));
                        a1 += ex2(fmaf(v[j + 1], c, neg));
                        a2 += ex2(fmaf(v[j + 2], c, neg));
                        a3 += ex2(fmaf(v[j + 3], c, neg));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kTileKeys; j += 4) {
                        a0 += (j + 0 < nv) ? ex2(fmaf(v[j + 0], c, neg)) : 0.f;
                        a1 += (j + 1 < nv) ? ex2(fmaf(v[j + 1], c, neg)) : 0.f;
                        a2 += (j + 2 < nv) ? ex2(fmaf(v[j + 2], c, neg)) : 0.f;
                        a3 += (j + 3 < nv) ? ex2(fmaf(v[j + 3], c, neg)) : 0.f;
                    }
                }
                l = l * ex2(m - m_new) + ((a0 + a1) + (a2 + a3));
                m = m_new;
            } else {
                // Block tile: finish m and l, then the weights of the B block columns.
                const int nb = p.B;
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < kTileKeys; ++j)
                    if (j < nb) mx = fmaxf(mx, v[j]);
                const float m_new = fmaxf(m, mx * c);
                const float neg = -m_new;
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int j = 0; j < kTileKeys; j += 4) {
                    v[j + 0] = (j + 0 < nb) ? ex2(fmaf(v[j + 0], c, neg)) : 0.f;
                    v[j + 1] = (j + 1 < nb) ? ex2(fmaf(v[j + 1], c, neg)) : 0.f;
                    v[j + 2] = (j + 2 < nb) ? ex2(fmaf(v[j + 2], c, neg)) : 0.f;
                    v[j + 3] = (j + 3 < nb) ? ex2(fmaf(v[j + 3], c, neg)) : 0.f;
                    a0 += v[j + 0];
                    a1 += v[j + 1];
                    a2 += v[j + 2];
                    a3 += v[j + 3];
                }
                l = l * ex2(m - m_new) + ((a0 + a1) + (a2 + a3));
                m = m_new;
                const bool row_ok = row < rows_valid;
                const float inv = 1.f / l;
#pragma unroll
                for (int j = 0; j < kTileKeys; ++j) v[j] = row_ok ? v[j] * inv : 0.f;
                // Column sums over this warp's 32 rows, one 32-column group at a time.
#pragma unroll
                for (int g = 0; g < kTileKeys / 32; ++g) {
                    if (g * 32 < nb) {
                        const float col = warp_colsum32(v + g * 32, lane);
                        red[quad * 128 + g * 32 + lane] = col;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(red_bar);
                if (mbar_wait(red_bar, 0, p.status, abort_flag)) {
                    const int j = (warp - 2) * 32 + lane;  // 128 threads cover up to 128 columns
                    if (j < nb) {
                        const float sum = ((red[0 * 128 + j] + red[1 * 128 + j]) + red[2 * 128 + j]) +
                                          red[3 * 128 + j];
                        const size_t idx =
                            ((((size_t)layer * p.R + r) * p.Hkv + kvh) * p.MT + mt) * p.B + j;
                        p.partial[idx] = sum;
                    }
                }
            }
        }
    }

    // ---- teardown: all TMEM reads and MMAs are complete (drained above)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace

size_t attn_smem_bytes(int head_dim) {
    return head_dim == 64 ? AttnSmem<64>::kAlloc : AttnSmem<128>::kAlloc;
}

cudaError_t launch_attn_stats(const AttnParams &p, int head_dim, cudaStream_t stream) {
    const long long grid = static_cast<long long>(p.R) * p.n_layers * p.Hkv * p.MT;
    if (grid <= 0) return cudaSuccess;
    if (head_dim == 64) {
        const int smem = AttnSmem<64>::kAlloc;
        cudaError_t e = cudaFuncSetAttribute(attn_stats_kernel<64>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attn_stats_kernel<64><<<static_cast<unsigned>(grid), kAttnThreads, smem, stream>>>(p);
    } else {
        const int smem = AttnSmem<128>::kAlloc;
        cudaError_t e = cudaFuncSetAttribute(attn_stats_kernel<128>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attn_stats_kernel<128><<<static_cast<unsigned>(grid), kAttnThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace focus
