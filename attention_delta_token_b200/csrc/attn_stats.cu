// attn_stats.cu -- attention importance I_j on sm_100a (TMA + tcgen05 + TMEM).
//
// Method: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science
// review page), "What carries the argument": I_j is the column-wise sum of the
// softmax attention weights block token j receives from all query tokens of the
// block; the Referee Report's minor comment on Eq. (2) reads the softmax as
// row (query) wise.  Each query row's softmax runs over the request's prefix
// keys followed by its B block keys; I_j also sums over the query heads.
//
// Work item = one (layer, request, kv head, 128-row query tile).  The kernel is
// persistent: two CTAs per SM take items from the list (longest prefix first),
// claimed dynamically from a counter when there are at least four per CTA, else
// one per round in snake order across the grid.  Per CTA (10 warps):
//   warp 0      TMA producer: the item's Q tile (once per item, as soon as the
//               previous item's MMAs have released it), then 128-key tiles of the
//               prefix and finally the block keys, through a 2-stage ring;
//   warp 1      allocates TMEM and issues tcgen05.mma (M=128 query rows, N=128
//               keys, K=d; bf16 in, fp32 out) into two ping-pong TMEM S buffers;
//   warps 2-9   two softmax warpgroups.  Warpgroup h reads columns [64h, 64h+64)
//               of every S tile (one TMEM lane = one query row per thread) and
//               keeps an online row max m and sum-exp l over its columns.  The
//               block tile comes last: the two halves' (m, l) are merged through
//               shared memory, the row's weights p_ij = 2^(s_ij - M)/L of the B
//               block columns are formed straight from the S values already in
//               registers (no second pass over the keys), and their column sums
//               over the 128 rows (warp butterfly, then the four lane quadrants in
//               fixed order) go to `partial`.  No float atomics: the result is
//               deterministic, and equal keys weighted by the same warpgroup (the
//               whole block when B <= 64, else each 64-column half) give
//               bit-equal columns.
// Split prefixes (small batches only): when the items would fill at most half of
// the grid, each item's prefix is split into chunks of at least four key tiles,
// one work item per chunk.  The chunks of an item come consecutively in the list,
// the last one also taking the block tile.  The others publish their rows' (m, l)
// and count themselves; the last waits for the count (bounded) and merges the
// chunks' statistics in chunk order before forming the block weights.  A chunk only
// ever waits for chunks listed before it, which never wait, and every CTA of the
// persistent grid is resident (2 per SM: launch bounds cap the registers at 96,
// 2 x 104 KB of shared memory and 2 x 256 TMEM columns fit an SM), so the waits
// end; they are bounded all the same.  Compiled as a separate instantiation
// (SPLIT), so the unsplit kernel is unchanged.
// Exponentials run on the SFU (ex2.approx, fp32).  After a half-row's first full
// tile the exps are taken against the running reference max without computing
// each tile's max (the tile's sum reveals a rise).  At the metric shape the
// kernel runs at the board power cap, so fewer instructions per (row, key) is
// what buys throughput; moving exps to the FMA pipe or packing them as f16
// pairs was measured and did not.
#include <math.h>

#include "focus_device.cuh"
#include "focus_kernels.cuh"

namespace focus {

namespace {

constexpr uint32_t kChunkBytes = kTileRows * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int kHalf = kTileKeys / 2;               // S columns per softmax warpgroup

template <int HEAD_DIM>
struct AttnSmem {
    static constexpr int kChunks = HEAD_DIM / 64;
    static constexpr uint32_t kTileBytes = kChunkBytes * kChunks;
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kKOff = kTileBytes;
    static constexpr uint32_t kBarOff = kKOff + kStages * kTileBytes;
    static constexpr uint32_t kRedOff = kBarOff + 256;
    static constexpr uint32_t kStatOff = kRedOff + 4 * 128 * sizeof(float);
    static constexpr uint32_t kBytes = kStatOff + 2 * 128 * sizeof(float2);
    static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

struct Item {
    int layer, r, kvh, mt, pstart, L, n_pre;
    int chunk, n_chunks;  // this item's chunk of the request's prefix, of n_chunks
    int t0, n_tiles;      // its prefix tiles start at t0; tiles in all (block tile included)
    bool final;           // the last chunk: also takes the block tile and merges
    int group;            // (layer, request, kv head, row tile) index of chunk_cnt/chunk_stat
    bool bad;
};

// Items per request rank: n_layers * Hkv * MT groups, each split into the
// request's prefix chunks (chunk innermost, so a group's last chunk comes after
// its other chunks in the list).
// With SPLIT false (no split prefixes) the chunk fields are compile-time constants
// (one chunk, tiles from 0, final) and the code folds to the unsplit loop.
template <bool SPLIT>
__device__ __forceinline__ Item decode_item(const AttnParams &p, int it) {
    Item w;
    const int per_req = p.n_layers * p.Hkv * p.MT;
    int rank, rem;
    if (SPLIT) {
        int lo = 0, hi = p.R - 1;  // largest rank q with item_base[q] <= it
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.item_base[mid] <= it) lo = mid; else hi = mid - 1;
        }
        rank = lo;
        rem = it - p.item_base[lo];
        // With layer 0's log-sum-exps given its groups stream no prefix: they come
        // first, one item each, then the split groups, chunk innermost.
        const int single = (p.lse0 && p.n_layers == 2) ? p.Hkv * p.MT : 0;
        if (rem < single) {
            w.n_chunks = 1;
            w.chunk = 0;
        } else {
            const int items = p.item_base[lo + 1] - p.item_base[lo];
            w.n_chunks = max(1, (items - single) / (per_req - single));
            const int r2 = rem - single;
            w.chunk = r2 % w.n_chunks;
            rem = single + r2 / w.n_chunks;
        }
    } else {
        rank = it / per_req;
        rem = it - rank * per_req;
        w.n_chunks = 1;
        w.chunk = 0;
    }
    w.layer = rem / (p.Hkv * p.MT);
    rem -= w.layer * p.Hkv * p.MT;
    w.kvh = rem / p.MT;
    w.mt = rem - w.kvh * p.MT;
    w.r = p.order ? p.order[rank] : rank;
    if (p.page_table) {
        w.pstart = 0;
        w.L = p.prefix_len[w.r];
        w.bad = w.L < 0 || static_cast<long long>(w.L) > static_cast<long long>(p.max_pages) * p.page_size;
    } else {
        w.pstart = p.cu_prefix[w.r];
        w.L = p.cu_prefix[w.r + 1] - w.pstart;
        w.bad = w.pstart < 0 || w.L < 0 || static_cast<long long>(w.pstart) + w.L > p.total_prefix;
    }
    if (p.lse0 && w.layer == 0) {  // the row normalisers are given: only the block keys matter
        w.bad = false;
        w.L = 0;
        w.pstart = 0;
    }
    if (w.bad) {
        w.L = 0;
        w.pstart = 0;
    }
    w.n_pre = (w.L + kTileKeys - 1) / kTileKeys;
    // chunk c of C takes prefix tiles [c * n_pre / C, (c + 1) * n_pre / C)
    w.t0 = static_cast<int>(static_cast<long long>(w.chunk) * w.n_pre / w.n_chunks);
    const int t1 = static_cast<int>(static_cast<long long>(w.chunk + 1) * w.n_pre / w.n_chunks);
    w.final = w.chunk == w.n_chunks - 1;
    w.n_tiles = (t1 - w.t0) + (w.final ? 1 : 0);
    w.group = ((w.layer * p.R + w.r) * p.Hkv + w.kvh) * p.MT + w.mt;
    return w;
}

// The work item a CTA takes in its k-th round.  Items come longest request first;
// the rounds alternate direction across the grid (a snake), so the CTA that took
// the longest item of one round takes the shortest of the next and the per-CTA
// totals even out (a plain stride hands CTA 0 the longest item of every round).
// Increasing in k for every CTA, so the first index past the end ends the loop.
__device__ __forceinline__ int item_of_round(int k) {
    const int g = static_cast<int>(gridDim.x);
    const int c = static_cast<int>(blockIdx.x);
    return k * g + ((k & 1) ? g - 1 - c : c);
}

// With at least kDynamicItemsPerCta items per CTA (unsplit kernel) items are claimed
// dynamically: each CTA starts with item blockIdx.x, and its producer claims item
// gridDim.x + atomicAdd(counter) two key tiles before the end of its current item, so
// CTAs take the longest-first list about in the order they become free (a greedy
// longest-first schedule).  The producer passes each index to the MMA and softmax
// warps through a ring of kItemSlots shared-memory slots (full: published; empty: read
// by all nine warps).  With fewer items per CTA the static snake order pairs long and
// short items as well and costs nothing at the end.
constexpr int kItemSlots = 4;
constexpr long long kDynamicItemsPerCta = 4;

// The item a consumer role (the MMA thread, or a softmax warp) takes in its k-th
// round: from the producer's ring when items are claimed dynamically, else the
// static snake order.  A wait that gives up returns an index past every item.
__device__ __forceinline__ int next_item(bool dyn, int k, uint64_t *full, uint64_t *empty,
                                         volatile int *ring, uint32_t *status,
                                         volatile int *abort_flag) {
    if (!dyn) return item_of_round(k);
    const int slot = k & (kItemSlots - 1);
    if (!mbar_wait(&full[slot], (k / kItemSlots) & 1, status, abort_flag)) return 0x7fffffff;
    const int it = ring[slot];
    __syncwarp(__activemask());  // every participating lane has read the slot
    if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
    return it;
}

// One thread waits until the counter reaches `target` (the group's other chunks
// have published their row statistics).  Bounded: on timeout it sets
// FOCUS_DEV_TIMEOUT and the abort flag; it also returns when another role aborted.
__device__ __forceinline__ void wait_chunks(const unsigned int *cnt, unsigned int target,
                                            uint32_t *status, volatile int *abort_flag) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= target) return;
        if ((it & 63u) == 63u) {
            if (*abort_flag) return;
            if (global_timer_ns() - t0 > FOCUS_WAIT_LIMIT_NS) {
                atomicOr(status, FOCUS_DEV_TIMEOUT);
                *abort_flag = 1;
                return;
            }
        }
        __nanosleep(128);
    }
}

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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Max of v[0..63] with three-input max, four independent chains.
__device__ __forceinline__ float max64(const float *v) {
    float a = fmaxf(v[0], v[1]), b = fmaxf(v[2], v[3]), c = fmaxf(v[4], v[5]), d = fmaxf(v[6], v[7]);
#pragma unroll
    for (int j = 8; j < kHalf; j += 8) {
        a = fmax3(a, v[j + 0], v[j + 1]);
        b = fmax3(b, v[j + 2], v[j + 3]);
        c = fmax3(c, v[j + 4], v[j + 5]);
        d = fmax3(d, v[j + 6], v[j + 7]);
    }
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

template <int HEAD_DIM, bool SPLIT>
__global__ void __launch_bounds__(kAttnThreads, 2)
attn_stats_kernel(const __grid_constant__ AttnParams p) {
    using S = AttnSmem<HEAD_DIM>;
    // Items claimed dynamically (see next_item) when the launch has several per CTA;
    // split chunks keep the static order their waits rely on.
    const bool dyn = !SPLIT && p.dynamic;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem + S::kQOff;
    uint8_t *sK = smem + S::kKOff;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBarOff);
    uint64_t *full = bars;                 // [kStages] key tile landed
    uint64_t *empty = bars + kStages;      // [kStages] key tile consumed by the MMAs
    uint64_t *q_full = bars + 2 * kStages; // Q tile landed
    uint64_t *q_empty = q_full + 1;        // Q tile released by the item's last MMAs
    uint64_t *s_full = q_empty + 1;        // [2] S buffer written by the MMAs
    uint64_t *s_empty = s_full + 2;        // [2] S buffer read out by the 8 softmax warps
    uint64_t *stat_bar = s_empty + 2;      // both halves' (m, l) of the item are in smem
    uint64_t *red_bar = stat_bar + 1;      // column partial sums of the item are in smem
    uint64_t *item_full = red_bar + 1;     // [kItemSlots] next item index published
    uint64_t *item_empty = item_full + kItemSlots;  // [kItemSlots] read by MMA + softmax warps
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(item_empty + kItemSlots);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *item_ring = abort_flag + 1;  // [kItemSlots] item indices, in claim order
    float *red = reinterpret_cast<float *>(smem + S::kRedOff);     // [4 quadrants][128 columns]
    float2 *stat = reinterpret_cast<float2 *>(smem + S::kStatOff); // [2 halves][128 rows]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- setup
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], kSoftmaxWarps);
        }
        mbar_init(stat_bar, kSoftmaxWarps);
        mbar_init(red_bar, kSoftmaxWarps);
        for (int q = 0; q < kItemSlots; ++q) {
            mbar_init(&item_full[q], 1);
            mbar_init(&item_empty[q], kSoftmaxWarps + 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int l = 0; l < p.n_layers; ++l) {
            tma_prefetch_desc(&p.tm_q[l]);
            tma_prefetch_desc(&p.tm_kp[l]);
            tma_prefetch_desc(&p.tm_kb[l]);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Everything above overlaps the planner; the request order it writes is read below.
    pdl_launch_dependents();
    pdl_wait();
    const int n_items = SPLIT ? p.item_base[p.R] : p.R * p.n_layers * p.Hkv * p.MT;

    if (warp == 0) {
        // ======================= TMA producer
        if (lane == 0) {
            // Key tiles of a single row tile are read once: stream them past L2.  With
            // several row tiles per kv head the siblings re-read them from L2.
            const uint64_t pol = p.MT == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
            uint32_t kt = 0;   // key tiles issued by this CTA
            int last_q = -1;   // item count of the last Q load issued
            int next = dyn ? static_cast<int>(blockIdx.x) : item_of_round(0);
            for (int k = 0;; ++k) {
                const int it = next;
                if (dyn) {
                    // Publish this CTA's k-th item (or the end) to the MMA and softmax warps.
                    // The next one is claimed two key tiles before this item's last (below).
                    const int slot = k & (kItemSlots - 1);
                    if (!mbar_wait(&item_empty[slot], ((k / kItemSlots) & 1) ^ 1, p.status,
                                   abort_flag))
                        break;
                    item_ring[slot] = it;
                    mbar_arrive(&item_full[slot]);
                    if (it >= n_items) break;
                } else {
                    if (it >= n_items) break;
                    next = item_of_round(k + 1);
                }
                const Item w = decode_item<SPLIT>(p, it);
                if (w.bad) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
                if (!mbar_wait(q_empty, (k & 1) ^ 1, p.status, abort_flag)) break;
                mbar_arrive_expect_tx(q_full, S::kTileBytes);
#pragma unroll
                for (int c = 0; c < S::kChunks; ++c)
                    tma_load_3d(sQ + c * kChunkBytes, &p.tm_q[w.layer], q_full, c * 64, w.kvh * p.G,
                                w.r * p.B + w.mt * p.tok_per_tile, pol);
                last_q = k;
                bool ok = true;
                for (int i = 0; i < w.n_tiles; ++i, ++kt) {
                    // Claim late, so CTAs take the longest-first list close to when they
                    // become free, yet early enough that the atomic's latency stays hidden.
                    if (dyn && i == (w.n_tiles > 2 ? w.n_tiles - 2 : 0))
                        next = static_cast<int>(gridDim.x) +
                               static_cast<int>(atomicAdd(p.item_counter, 1u));
                    const int t = w.t0 + i;                              // prefix tile index
                    const bool blk = w.final && i == w.n_tiles - 1;      // the block tile
                    const int s = kt % kStages;
                    const uint32_t ph = (kt / kStages) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, p.status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *dst = sK + s * S::kTileBytes;
                    if (!blk && p.page_table) {
                        // The tile's keys come from page_rows-row boxes of consecutive pages;
                        // boxes past the prefix are not loaded (their columns are masked).
                        const int first = t * kTileKeys;
                        const int nbox = min(kTileKeys, w.L - first + p.page_rows - 1) / p.page_rows;
                        mbar_arrive_expect_tx(&full[s], nbox * p.page_rows * 128 * S::kChunks);
                        for (int u = 0; u < nbox; ++u) {
                            const int key = first + u * p.page_rows;
                            int page = p.page_table[static_cast<size_t>(w.r) * p.max_pages +
                                                    key / p.page_size];
                            if (page < 0 || page >= p.num_pages) {
                                atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
                                page = 0;  // keep the copy in bounds; the result is flagged
                            }
                            const int row = page * p.page_size + key % p.page_size;
#pragma unroll
                            for (int c = 0; c < S::kChunks; ++c)
                                tma_load_3d(dst + c * kChunkBytes + u * p.page_rows * 128,
                                            &p.tm_kp[w.layer], &full[s], c * 64, w.kvh, row, pol);
                        }
                    } else if (!blk) {
                        mbar_arrive_expect_tx(&full[s], S::kTileBytes);
#pragma unroll
                        for (int c = 0; c < S::kChunks; ++c)
                            tma_load_3d(dst + c * kChunkBytes, &p.tm_kp[w.layer], &full[s], c * 64,
                                        w.kvh, w.pstart + t * kTileKeys, pol);
                    } else {
                        mbar_arrive_expect_tx(&full[s], p.n_blk * 128 * S::kChunks);
#pragma unroll
                        for (int c = 0; c < S::kChunks; ++c)
                            tma_load_3d(dst + c * kChunkBytes, &p.tm_kb[w.layer], &full[s], c * 64,
                                        w.kvh, w.r * p.B, pol);
                    }
                }
                if (!ok) break;
            }
            // Drain: every copy this thread issued has landed before the CTA exits.
            if (last_q >= 0) mbar_wait_drain(q_full, last_q & 1);
            for (uint32_t u = kt > kStages ? kt - kStages : 0; u < kt; ++u)
                mbar_wait_drain(&full[u % kStages], (u / kStages) & 1);
        }
    } else if (warp == 1) {
        // ======================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pre = umma_idesc_bf16_f32(kTileRows, kTileKeys);
            const uint32_t idesc_blk = umma_idesc_bf16_f32(kTileRows, p.n_blk);
            const uint32_t a_base = smem_u32(sQ);
            uint32_t kt = 0;  // key tiles consumed
            uint32_t st = 0;  // S tiles produced
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int it = next_item(dyn, k, item_full, item_empty, item_ring, p.status, abort_flag);
                if (it >= n_items) break;
                const Item w = decode_item<SPLIT>(p, it);
                if (!mbar_wait(q_full, k & 1, p.status, abort_flag)) break;
                for (int i = 0; i < w.n_tiles; ++i, ++kt, ++st) {
                    const bool blk = w.final && i == w.n_tiles - 1;
                    const int s = kt % kStages;
                    const uint32_t ph = (kt / kStages) & 1;
                    const int buf = st & 1;
                    const uint32_t bph = (st >> 1) & 1;
                    if (!mbar_wait(&s_empty[buf], bph ^ 1, p.status, abort_flag) ||
                        !mbar_wait(&full[s], ph, p.status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t idesc = blk ? idesc_blk : idesc_pre;
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
                }
                if (ok) umma_commit(q_empty);  // Q may be overwritten once these MMAs finish
            }
            // Drain: the last MMAs have finished writing TMEM.
            if (st > 0) mbar_wait_drain(&s_full[(st - 1) & 1], ((st - 1) >> 1) & 1);
        }
    } else {
        // ======================= softmax statistics: warpgroup h, one query row per thread
        const int sw = warp - 2;         // 0..7
        const int h = sw >> 2;           // column half of every S tile
        const int quad = warp & 3;       // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const int col0 = h * kHalf;
        const float c = p.scale_log2;
        const float2 c2 = make_float2(c, c);
        uint32_t st = 0;
        int kf = 0;  // final chunks done (the reduction barrier completes once per final chunk)
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int it = next_item(dyn, k, item_full, item_empty, item_ring, p.status, abort_flag);
            if (it >= n_items) break;
            const Item w = decode_item<SPLIT>(p, it);
            const int rows_valid = min(kTileRows, p.G * p.B - w.mt * kTileRows);
            float m = -INFINITY;  // running max of the scaled logits (log2 domain), this half
            float l = 0.f;        // running sum of 2^(x - m), this half
            for (int i = 0; i < w.n_tiles; ++i, ++st) {
                const int t = w.t0 + i;
                const bool blk = w.final && i == w.n_tiles - 1;
                const int buf = st & 1;
                const uint32_t bph = (st >> 1) & 1;
                if (!mbar_wait(&s_full[buf], bph, p.status, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int ncols = blk ? p.B : min(kTileKeys, w.L - t * kTileKeys);
                const int nh = min(max(ncols - col0, 0), kHalf);  // valid columns in this half
                float v[kHalf];
                if (nh > 0) {
                    const uint32_t ta = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                        static_cast<uint32_t>(buf * kTileKeys + col0);
                    tmem_ld32<0>(ta, v);
                    tmem_ld32<32>(ta, v);
                    tmem_wait_ld();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[buf]);

                if (!blk) {
                    if (nh == kHalf && m != -INFINITY) {
                        // Against the running reference m, no tile max is needed: a tile whose
                        // values rose far above m shows up as a large sum (>= 2^20), and only
                        // then is the tile redone against its exact max.  Values that fell far
                        // below m underflow to 0, as they do against the exact max.
                        const float2 nm = make_float2(-m, -m);
                        float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
                        for (int q = 0; q < kHalf / 2; ++q) {
                            const float2 x = __ffma2_rn(make_float2(v[2 * q], v[2 * q + 1]), c2, nm);
                            float2 e; e.x = ex2(x.x); e.y = ex2(x.y);
                            if (q & 1) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
                        }
                        const float sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
                        if (sum <= 1048576.f) {
                            l += sum;
                        } else {
                            const float m_new = fmaxf(m, max64(v) * c);
                            float a0 = 0.f, a1 = 0.f;
#pragma unroll
                            for (int j = 0; j < kHalf; j += 2) {
                                a0 += ex2(fmaf(v[j], c, -m_new));
                                a1 += ex2(fmaf(v[j + 1], c, -m_new));
                            }
                            l = l * ex2(m - m_new) + (a0 + a1);
                            m = m_new;
                        }
                    } else if (nh == kHalf) {
                        const float m_new = fmaxf(m, max64(v) * c);
                        const float2 nm = make_float2(-m_new, -m_new);
                        float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
                        for (int q = 0; q < kHalf / 2; ++q) {
                            const float2 x = __ffma2_rn(make_float2(v[2 * q], v[2 * q + 1]), c2, nm);
                            float2 e; e.x = ex2(x.x); e.y = ex2(x.y);
                            if (q & 1) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
                        }
                        l = l * ex2(m - m_new) + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
                        m = m_new;
                    } else if (nh > 0) {
#pragma unroll
                        for (int j = 0; j < kHalf; ++j)
                            if (j >= nh) v[j] = -INFINITY;
                        const float m_new = fmaxf(m, max64(v) * c);
                        float a0 = 0.f, a1 = 0.f;
#pragma unroll
                        for (int j = 0; j < kHalf; j += 2) {
                            a0 += (j < nh) ? ex2(fmaf(v[j], c, -m_new)) : 0.f;
                            a1 += (j + 1 < nh) ? ex2(fmaf(v[j + 1], c, -m_new)) : 0.f;
                        }
                        l = l * ex2(m - m_new) + (a0 + a1);
                        m = m_new;
                    }
                } else {
                    // ---- block tile: finish this half, merge halves, weights, column sums
                    if (nh > 0) {
#pragma unroll
                        for (int j = 0; j < kHalf; ++j)
                            if (j >= nh) v[j] = -INFINITY;
                        const float m_new = fmaxf(m, max64(v) * c);
                        float a0 = 0.f, a1 = 0.f;
#pragma unroll
                        for (int j = 0; j < kHalf; j += 2) {
                            v[j] = (j < nh) ? ex2(fmaf(v[j], c, -m_new)) : 0.f;
                            v[j + 1] = (j + 1 < nh) ? ex2(fmaf(v[j + 1], c, -m_new)) : 0.f;
                            a0 += v[j];
                            a1 += v[j + 1];
                        }
                        l = l * ex2(m - m_new) + (a0 + a1);
                        m = m_new;
                    }
                    stat[h * 128 + row] = make_float2(m, l);
                    __syncwarp();
                    if (lane == 0) {
                        // With a split prefix the other chunks' statistics must be published
                        // first; the barrier passes the wait on to the other warps.
                        if (sw == 0 && w.n_chunks > 1)
                            wait_chunks(p.chunk_cnt + w.group, w.n_chunks - 1, p.status, abort_flag);
                        mbar_arrive(stat_bar);
                    }
                    if (!mbar_wait(stat_bar, k & 1, p.status, abort_flag) ||
                        (w.n_chunks > 1 && *abort_flag)) {
                        ok = false;
                        break;
                    }
                    const float2 s0 = stat[row], s1 = stat[128 + row];
                    float M = fmaxf(s0.x, s1.x);  // finite: half 0 always has a column
                    // the other chunks' (m, l) of this row, merged in chunk order
                    const int nc = w.n_chunks - 1;
                    const float2 *cs =
                        p.chunk_stat + static_cast<size_t>(w.group) * (p.chunk_max - 1) * 256;
                    for (int q = 0; q < nc; ++q)
                        M = fmax3(M, __ldcg(cs + q * 256 + row).x, __ldcg(cs + q * 256 + 128 + row).x);
                    float Ltot = s0.y * ex2(s0.x - M) + s1.y * ex2(s1.x - M);
                    for (int q = 0; q < nc; ++q) {
                        const float2 a = __ldcg(cs + q * 256 + row), b = __ldcg(cs + q * 256 + 128 + row);
                        Ltot += a.y * ex2(a.x - M) + b.y * ex2(b.x - M);
                    }
                    if (p.lse0 && w.layer == 0 && row < rows_valid) {
                        // Given normaliser: p_ij = exp(s_ij - lse_i) = 2^(x_ij - lse_i log2 e).
                        const int tok = w.mt * p.tok_per_tile + row / p.G;
                        const int h = w.kvh * p.G + row % p.G;
                        M = p.lse0[(static_cast<size_t>(w.r) * p.B + tok) * p.Hq + h] *
                            1.4426950408889634f;
                        Ltot = 1.f;
                    }
                    if (nh > 0) {
                        const float scale = (row < rows_valid) ? ex2(m - M) / Ltot : 0.f;
#pragma unroll
                        for (int j = 0; j < kHalf; ++j) v[j] *= scale;
#pragma unroll
                        for (int g = 0; g < kHalf / 32; ++g) {
                            if (g * 32 < nh) {
                                const float col = warp_colsum32(v + g * 32, lane);
                                red[quad * 128 + col0 + g * 32 + lane] = col;
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(red_bar);
                    if (!mbar_wait(red_bar, kf & 1, p.status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int j = sw * 32 + lane;
                    if (j < p.B) {
                        const float sum = ((red[0 * 128 + j] + red[1 * 128 + j]) + red[2 * 128 + j]) +
                                          red[3 * 128 + j];
                        // (layer, request, kv head, row tile): the item's group
                        const size_t idx =
                            SPLIT ? static_cast<size_t>(w.group) * p.B + j
                                  : ((((size_t)w.layer * p.R + w.r) * p.Hkv + w.kvh) * p.MT + w.mt) * p.B + j;
                        p.partial[idx] = sum;
                    }
                }
            }
            if (!ok) break;
            if (w.final) {
                ++kf;
            } else {
                // A chunk before the last: publish this row's (m, l) of its half, then
                // count the chunk once every softmax warp has (release: barrier, fence,
                // counter).
                p.chunk_stat[(static_cast<size_t>(w.group) * (p.chunk_max - 1) + w.chunk) * 256 +
                             h * 128 + row] = make_float2(m, l);
                __syncwarp();
                if (lane == 0) mbar_arrive(stat_bar);
                if (!mbar_wait(stat_bar, k & 1, p.status, abort_flag)) {
                    ok = false;
                    break;
                }
                if (sw == 0 && lane == 0) {
                    __threadfence();
                    atomicAdd(p.chunk_cnt + w.group, 1u);
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

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

}  // namespace

size_t attn_smem_bytes(int head_dim) {
    return head_dim == 64 ? AttnSmem<64>::kAlloc : AttnSmem<128>::kAlloc;
}

template <int HEAD_DIM, bool SPLIT>
cudaError_t launch_attn_variant(const AttnParams &p, long long grid, cudaStream_t stream, bool pdl) {
    const int smem = AttnSmem<HEAD_DIM>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_stats_kernel<HEAD_DIM, SPLIT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(attn_stats_kernel<HEAD_DIM, SPLIT>, dim3(static_cast<unsigned>(grid)),
                         dim3(kAttnThreads), smem, stream, pdl, p);
}

cudaError_t launch_attn_stats(const AttnParams &p, int head_dim, cudaStream_t stream, bool pdl) {
    // With split prefixes each item has up to chunk_max chunks (the exact count is
    // the planner's); CTAs beyond the items exit at once.
    const bool split = p.chunk_max > 1;
    const long long items = static_cast<long long>(p.R) * p.n_layers * p.Hkv * p.MT *
                            (split ? p.chunk_max : 1);
    if (items <= 0) return cudaSuccess;
    const long long grid = items < 2ll * sm_count() ? items : 2ll * sm_count();
    AttnParams q = p;
    q.dynamic = !split && items >= kDynamicItemsPerCta * grid;
    cudaError_t e;
    if (head_dim == 64)
        e = split ? launch_attn_variant<64, true>(q, grid, stream, pdl)
                  : launch_attn_variant<64, false>(q, grid, stream, pdl);
    else
        e = split ? launch_attn_variant<128, true>(q, grid, stream, pdl)
                  : launch_attn_variant<128, false>(q, grid, stream, pdl);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace focus
