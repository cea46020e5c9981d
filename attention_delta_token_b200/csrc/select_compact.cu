// select_compact.cu -- planning, importance delta, MaxPool1D, mask, top-K and
// compaction kernels of the FOCUS eviction step (sm_100a, CUDA cores / LSU).
//
// Method: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science
// review page), "What carries the argument": dI = I(layer 1) - I(layer 0)
// (Eq. 3), smoothed by MaxPool1D (Free-Parameter Ledger: k = 3, Eq. 15), top-K
// candidates kept under a budget; "The pith": the remaining layers then run
// only on the retained tokens, here packed into a varlen batch with cu_seqlens.
//
// Selection is exact and deterministic: a position's rank is the number of
// positions that beat it under (value desc, position asc), so every tie goes to
// the lower position and the kept set never depends on thread timing.
#include <math.h>

#include "focus_device.cuh"
#include "focus_kernels.cuh"
#include "focus_exchange.cuh"

namespace focus {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kRankSortR = 1024; // up to here the order is a rank count
constexpr int kMaxSortR = 4096;  // up to here a bitonic sort; larger batches keep input order
constexpr int kCompactStagedCu = 4096;  // cu_seqlens entries the compaction stages in smem

// sum over g < n of src[g * stride] in the order g = 0, 1, 2, ... (the fixed order
// every reduction of the column sums uses, so the fused step, the stand-alone
// reduction and the exchange all give the same bits), with eight loads in flight.
// Loads go through L2: the sums were written by another kernel or another GPU.
__device__ __forceinline__ float ordered_sum(const float *src, int n, int stride) {
    float s = 0.f;
    int g = 0;
    for (; g + 8 <= n; g += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = __ldcg(src + static_cast<size_t>(g + u) * stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) s += x[u];
    }
    for (; g < n; ++g) s += __ldcg(src + static_cast<size_t>(g) * stride);
    return s;
}

// masked_r = number of zero bytes in decoded[r*B .. r*B+B); 16-byte loads when
// the row is 16-byte aligned.
__device__ __forceinline__ int masked_count(const uint8_t *decoded, int r, int B) {
    const uint8_t *d = decoded + static_cast<size_t>(r) * B;
    int masked = 0;
    if ((reinterpret_cast<uintptr_t>(d) & 15u) == 0 && (B & 15) == 0) {
        const uint4 *d4 = reinterpret_cast<const uint4 *>(d);
        for (int i = 0; i < B / 16; ++i) {
            const uint4 w = __ldg(d4 + i);
            masked += __popc(__vcmpeq4(w.x, 0u)) + __popc(__vcmpeq4(w.y, 0u)) +
                      __popc(__vcmpeq4(w.z, 0u)) + __popc(__vcmpeq4(w.w, 0u));
        }
        return masked >> 3;  // __vcmpeq4 sets 8 bits per equal byte
    }
    for (int j = 0; j < B; ++j) masked += d[j] == 0;
    return masked;
}

// k_r = min(max(budget_r, 0), masked_r)
__device__ __forceinline__ int kept_count(const uint8_t *decoded, const int32_t *budget, int r,
                                          int B) {
    return min(max(budget[r], 0), masked_count(decoded, r, B));
}

// Prefix length of request r: from the paged lengths or the packed offsets.
__device__ __forceinline__ int prefix_length(const PlanParams &p, int r) {
    return p.prefix_len ? p.prefix_len[r] : p.cu_prefix[r + 1] - p.cu_prefix[r];
}

// Exclusive block-wide scan of one int per thread (kPlanThreads threads).
__device__ __forceinline__ int block_exclusive_scan(int x, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    const int ex = warp_tot[warp] + incl - x;
    total = warp_tot[32];
    __syncthreads();
    return ex;
}

// One CTA: (a) the processing order of the requests, longest prefix first
// (ranks of (L desc, r asc) keys), so the attention CTAs of the longest requests
// start in the first wave; (b) with split prefixes, each request's first
// attention item and zeroed chunk counters; (c) k_r and cu_seqlens (depend only on
// decoded and budget) and the capacity check.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanParams p) {
    __shared__ unsigned long long keys[kMaxSortR];
    __shared__ int warp_tot[33];
    const int R = p.R;
    pdl_launch_dependents();  // the attention kernel may set up while this runs
    if (threadIdx.x == 0 && p.item_counter) *p.item_counter = 0u;

    if (p.order && R <= kRankSortR) {
        // Rank of each request under (L desc, r asc): a plain count, no sort passes.
        for (int i = threadIdx.x; i < R; i += blockDim.x) {
            const int L = max(prefix_length(p, i), 0);
            keys[i] = (static_cast<unsigned long long>(0x7fffffffu - static_cast<uint32_t>(L)) << 32) |
                      static_cast<uint32_t>(i);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < R; i += blockDim.x) {
            const unsigned long long ki = keys[i];
            int rank = 0;
            for (int j = 0; j < R; ++j) rank += keys[j] < ki;
            p.order[rank] = i;
        }
    } else if (p.order) {
        if (R <= kMaxSortR) {
            int n = 1;
            while (n < R) n <<= 1;
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                unsigned long long key = ~0ull;
                if (i < R) {
                    const int L = max(prefix_length(p, i), 0);
                    key = (static_cast<unsigned long long>(0x7fffffffu - static_cast<uint32_t>(L)) << 32) |
                          static_cast<uint32_t>(i);
                }
                keys[i] = key;
            }
            __syncthreads();
            for (int k = 2; k <= n; k <<= 1) {
                for (int j = k >> 1; j > 0; j >>= 1) {
                    for (int i = threadIdx.x; i < n; i += blockDim.x) {
                        const int ixj = i ^ j;
                        if (ixj > i) {
                            const unsigned long long a = keys[i], b = keys[ixj];
                            const bool up = (i & k) == 0;
                            if ((a > b) == up) {
                                keys[i] = b;
                                keys[ixj] = a;
                            }
                        }
                    }
                    __syncthreads();
                }
            }
            for (int i = threadIdx.x; i < R; i += blockDim.x)
                p.order[i] = static_cast<int32_t>(keys[i] & 0xffffffffu);
        } else {
            for (int i = threadIdx.x; i < R; i += blockDim.x) p.order[i] = i;
        }
    }

    if (p.item_base) {
        // Split prefixes: the attention items of request rank q start at item_base[q];
        // the counters the last chunks wait on start from zero.
        __syncthreads();  // the order above was written by other threads of this block
        int running = 0;
        for (int base = 0; base < R; base += kPlanThreads) {
            const int q = base + threadIdx.x;
            int n = 0;
            if (q < R) {
                const int r = p.order ? p.order[q] : q;
                n = p.single_groups + prefix_chunks(prefix_length(p, r), p.chunk_max) * p.per_req;
            }
            int total;
            const int ex = block_exclusive_scan(n, warp_tot, total);
            if (q < R) p.item_base[q] = running + ex;
            running += total;
        }
        if (threadIdx.x == 0) p.item_base[R] = running;
        for (int i = threadIdx.x; i < p.n_groups; i += blockDim.x) p.chunk_cnt[i] = 0;
    }

    if (p.cu_seqlens) {
        int running = 0;
        if (threadIdx.x == 0) p.cu_seqlens[0] = 0;
        for (int base = 0; base < R; base += kPlanThreads) {
            const int r = base + threadIdx.x;
            const int k = r < R ? kept_count(p.decoded, p.budget, r, p.B) : 0;
            int total;
            const int ex = block_exclusive_scan(k, warp_tot, total);
            if (r < R) p.cu_seqlens[r + 1] = running + ex + k;
            running += total;
        }
        if (threadIdx.x == 0 && static_cast<long long>(running) > p.capacity)
            atomicOr(p.status, FOCUS_DEV_CAPACITY);
    }
}

// Rank-based top-k over sv[0..B) (value desc, position asc); thread j < B
// decides position j.  Writes the kept positions, ascending, into kept_s and
// kept_idx[base ..].  Returns nothing; the caller syncs.
__device__ __forceinline__ void select_block(const float *sv, const uint8_t *dec, int B, int k,
                                             long long base, long long capacity, int *sel_s,
                                             int *kept_s, int32_t *kept_idx, uint32_t *status) {
    const int j = threadIdx.x;
    if (j < 128) kept_s[j] = -1;
    if (j < B) {
        const float v = sv[j];
        int rank = 0;
        for (int t = 0; t < B; ++t) {  // only still-masked positions compete
            const float u = sv[t];
            rank += dec[t] == 0 && ((u > v) || (u == v && t < j));
        }
        sel_s[j] = (dec[j] == 0 && rank < k) ? 1 : 0;
    }
    __syncthreads();
    if (j < B && sel_s[j]) {
        int slot = 0;
        for (int t = 0; t < j; ++t) slot += sel_s[t];
        if (slot >= k) return;  // only reachable with non-finite values (out of contract)
        kept_s[slot] = j;
        const long long out = base + slot;
        if (out < capacity)
            kept_idx[out] = j;
        else
            atomicOr(status, FOCUS_DEV_CAPACITY);
    }
}

// MaxPool1D (odd window, stride 1, same padding, padded cells ignored) of
// raw[0..B) at position j, then the decoded mask.
__device__ __forceinline__ float pool_mask(const float *raw, const uint8_t *dec, int B, int w,
                                           int j) {
    const int h = w >> 1;
    float best = -INFINITY;
    const int lo = max(0, j - h), hi = min(B - 1, j + h);
    for (int t = lo; t <= hi; ++t) best = fmaxf(best, raw[t]);
    return dec[j] ? -INFINITY : best;
}

// One CTA per request.  From the per-kv-head column sums of both layers (fused
// path) or from a pooled delta (stand-alone select): I0, I1, dI, MaxPool1D,
// mask, top-k, then the k kept hidden rows copied with 16-byte vectors.
__global__ void __launch_bounds__(256) select_compact_kernel(const SelectParams p) {
    pdl_launch_dependents();
    pdl_wait();  // column sums / delta and cu_seqlens come from the previous kernels
    __shared__ float raw_s[128];
    __shared__ float val_s[128];
    __shared__ uint8_t dec_s[128];
    __shared__ int sel_s[128];
    __shared__ int kept_s[128];
    const int r = blockIdx.x;
    const int B = p.B;
    const int j = threadIdx.x;
    const size_t rb = static_cast<size_t>(r) * B;

    if (j < B) dec_s[j] = p.decoded[rb + j];
    // With the peer exchange the sums arrive from every rank; on a timeout the
    // status says so and the slots are read as they are.
    if (p.ex_flags) ex_wait(p.ex_flags, p.Hkv * p.MT, p.ex_epoch, p.status);
    if (p.partial) {
        if (j < B) {
            const int n = p.Hkv * p.MT;
            const size_t lstride = static_cast<size_t>(p.R) * n * B;
            const float *col = p.partial + rb * n + j;  // group g of column j at col[g * B]
            float i0 = 0.f, i1 = 0.f;
            if (p.layers == 1) {  // only the layer-1 statistics exist: score = I1
                i1 = ordered_sum(col, n, B);
                raw_s[j] = i1;
            } else {
                i0 = ordered_sum(col, n, B);
                i1 = ordered_sum(col + lstride, n, B);
                raw_s[j] = i1 - i0;
                if (p.i0_out) p.i0_out[rb + j] = i0;
            }
            if (p.i1_out) p.i1_out[rb + j] = i1;
            if (p.raw_out) p.raw_out[rb + j] = raw_s[j];
            // I is a sum of softmax weights, finite for any finite Q and K: a non-finite
            // value means non-finite inputs (out of contract), reported, not ranked silently.
            if (!isfinite(raw_s[j])) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
        }
        __syncthreads();
        if (j < B) {
            const float d = pool_mask(raw_s, dec_s, B, p.pool_window, j);
            val_s[j] = d;
            if (p.delta_out) p.delta_out[rb + j] = d;
        }
    } else {
        if (j < B) {
            val_s[j] = p.delta_in[rb + j];
            // still-masked positions carry finite scores; anything else is out of contract
            if (dec_s[j] == 0 && !isfinite(val_s[j])) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
        }
    }
    __syncthreads();

    if (p.constraints || p.decode_avg) {
        // Candidates (under the given or the dynamic budget), then the structural
        // constraints; the retained positions go to a per-request list (their count
        // depends on the data: cu_seqlens comes later).
        __shared__ int rightmost;
        __shared__ int k_dyn;
        const int masked = __syncthreads_count(j < B && dec_s[j] == 0);
        if (p.decode_avg && j == 0) {
            // K = min(max(ceil(alpha * yield), #{masked D > mean + std}, 1), masked),
            // statistics over the masked positions in position order.
            int K = 0;
            if (masked > 0) {
                float sum = 0.f;
                for (int t = 0; t < B; ++t)
                    if (!dec_s[t]) sum += val_s[t];
                const float mu = sum / masked;
                float ss = 0.f;
                for (int t = 0; t < B; ++t)
                    if (!dec_s[t]) ss += (val_s[t] - mu) * (val_s[t] - mu);
                const float thr = mu + sqrtf(ss / masked);
                int n = 0;
                for (int t = 0; t < B; ++t) n += !dec_s[t] && val_s[t] > thr;
                const float want = ceilf(p.budget_alpha * fmaxf(p.decode_avg[r], 0.f));
                K = want >= static_cast<float>(masked) ? masked : max(static_cast<int>(want), n);
                K = min(max(K, 1), masked);
            }
            k_dyn = K;
            if (p.budget_out) p.budget_out[r] = K;
        }
        __syncthreads();
        const int k = p.decode_avg ? k_dyn : min(max(p.budget[r], 0), masked);
        if (j == 0) rightmost = -1;
        if (j < B) {
            const float v = val_s[j];
            int rank = 0;
            for (int t = 0; t < B; ++t) {
                const float u = val_s[t];
                rank += dec_s[t] == 0 && ((u > v) || (u == v && t < j));
            }
            sel_s[j] = (dec_s[j] == 0 && rank < k) ? 1 : 0;
        }
        __syncthreads();
        if (j < B && sel_s[j]) atomicMax(&rightmost, j);
        __syncthreads();
        const bool keep = j < B && (sel_s[j] ||
                                    ((p.constraints & 1) && j + 1 < B && sel_s[j + 1]) ||
                                    ((p.constraints & 2) && dec_s[j] == 0 && j < rightmost));
        if (j < 128) kept_s[j] = keep ? 1 : 0;
        const int n = __syncthreads_count(keep);
        if (keep) {
            int slot = 0;
            for (int t = 0; t < j; ++t) slot += kept_s[t];
            p.lists[rb + slot] = j;
        }
        if (j == 0) p.counts[r] = n;
        return;
    }

    const long long base = p.cu_seqlens[r];
    const int k = static_cast<int>(p.cu_seqlens[r + 1] - base);
    select_block(val_s, dec_s, B, k, base, p.capacity, sel_s, kept_s, p.kept_idx, p.status);
    __syncthreads();

    if (p.hidden) {
        const int rows = static_cast<int>(max(0ll, min(static_cast<long long>(k), p.capacity - base)));
        const int nvec = p.H / 8;  // 16-byte vectors per row
        const uint4 *src = reinterpret_cast<const uint4 *>(p.hidden) + rb * nvec;
        uint4 *dst = reinterpret_cast<uint4 *>(p.packed) + static_cast<size_t>(base) * nvec;
        const int total = rows * nvec;
        for (int v = threadIdx.x; v < total; v += blockDim.x) {
            const int t = v / nvec;
            const int c = v - t * nvec;
            const int jj = kept_s[t];
            if (jj < 0) {  // fewer than k selected: non-finite values (out of contract)
                if (c == 0) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
                continue;
            }
            dst[static_cast<size_t>(t) * nvec + c] = __ldg(src + static_cast<size_t>(jj) * nvec + c);
        }
    }
}

// Stand-alone importance delta + MaxPool1D + mask, one CTA (128 threads) per request.
__global__ void __launch_bounds__(128) delta_kernel(const DeltaParams p) {
    __shared__ float raw_s[128];
    __shared__ uint8_t dec_s[128];
    const int r = blockIdx.x, j = threadIdx.x, B = p.B;
    const size_t rb = static_cast<size_t>(r) * B;
    if (j < B) {
        const float d = p.i1[rb + j] - p.i0[rb + j];
        raw_s[j] = d;
        dec_s[j] = p.decoded[rb + j];
        if (p.raw) p.raw[rb + j] = d;
    }
    __syncthreads();
    if (j < B) p.delta[rb + j] = pool_mask(raw_s, dec_s, B, p.pool_window, j);
}

// importance[l][r][j] = sum over kv heads and row tiles (fixed order) of layer l's
// column sums; one block per (request, layer).  With the peer exchange the sum is
// stored into every rank's exchange buffer and the last block raises this rank's
// flags (focus_exchange.cuh).
__global__ void __launch_bounds__(128) reduce_kernel(const ReduceParams p) {
    pdl_wait();  // the column sums come from the attention kernel
    const int r = blockIdx.x, l = blockIdx.y, j = threadIdx.x, B = p.B;
    if (j < B) {
        const size_t rb = static_cast<size_t>(r) * B;
        const int n = p.Hkv * p.MT;
        const float *part = p.partial + static_cast<size_t>(l) * p.R * n * B;
        const float s = ordered_sum(part + rb * n + j, n, B);
        if (p.ex_world)
            ex_push(p.ex_bufs, p.R, B, p.ex_world, p.ex_rank, p.ex_epoch, l, r, j, s);
        else
            p.importance[static_cast<size_t>(l) * p.R * B + rb + j] = s;
    }
    if (p.ex_world)
        ex_signal(p.ex_bufs, ex_layout(p.R, B, p.ex_world).flags, p.ex_world, p.ex_rank,
                  p.ex_epoch, p.ex_counter, gridDim.x * gridDim.y);
}

// Stand-alone compaction: one warp per packed row, request found by binary search.
__global__ void __launch_bounds__(256) compact_kernel(const CompactParams p) {
    __shared__ int cu_s[kCompactStagedCu];
    pdl_wait();  // kept_idx and cu_seqlens come from the previous kernels
    // The binary search runs in shared memory when cu_seqlens fits (one coalesced
    // load per block instead of a chain of dependent global loads per row).
    const bool staged = p.R + 1 <= kCompactStagedCu;
    if (staged)
        for (int i = threadIdx.x; i <= p.R; i += blockDim.x) cu_s[i] = p.cu_seqlens[i];
    __syncthreads();
    const int32_t *cu = staged ? cu_s : p.cu_seqlens;
    const int warps = blockDim.x >> 5;
    const long long total = min(static_cast<long long>(cu[p.R]), p.capacity);
    if (blockIdx.x == 0 && threadIdx.x == 0 && cu[p.R] > p.capacity)
        atomicOr(p.status, FOCUS_DEV_CAPACITY);
    const int lane = threadIdx.x & 31;
    const int nvec = p.H / 8;
    for (long long row = static_cast<long long>(blockIdx.x) * warps + (threadIdx.x >> 5); row < total;
         row += static_cast<long long>(gridDim.x) * warps) {
        int lo = 0, hi = p.R - 1;  // largest r with cu[r] <= row
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu[mid] <= row) lo = mid; else hi = mid - 1;
        }
        int jj;
        if (p.lists) {  // structural constraints: row t of request lo is its t-th list entry
            const long long t = row - cu[lo];
            jj = (t >= 0 && t < p.B) ? p.lists[static_cast<size_t>(lo) * p.B + t] : -1;
            if (lane == 0 && jj >= 0 && jj < p.B) p.kept_out[row] = jj;
        } else {
            jj = p.kept_idx[row];
        }
        if (jj < 0 || jj >= p.B) {
            if (lane == 0) atomicOr(p.status, FOCUS_DEV_BAD_INPUT);
            continue;
        }
        if (!p.hidden) continue;
        const uint4 *__restrict__ src = reinterpret_cast<const uint4 *>(p.hidden) +
                                        (static_cast<size_t>(lo) * p.B + jj) * nvec;
        uint4 *__restrict__ dst = reinterpret_cast<uint4 *>(p.packed) + static_cast<size_t>(row) * nvec;
        int c = lane;
        for (; c + 7 * 32 < nvec; c += 8 * 32) {  // eight 16-byte loads in flight per lane
            uint4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = __ldg(src + c + 32 * u);
#pragma unroll
            for (int u = 0; u < 8; ++u) dst[c + 32 * u] = x[u];
        }
        for (; c < nvec; c += 32) dst[c] = __ldg(src + c);
    }
}

// cu_seqlens from per-request counts (one CTA; chunks of kPlanThreads), capacity check.
__global__ void __launch_bounds__(kPlanThreads) scan_kernel(const ScanParams p) {
    __shared__ int warp_tot[33];
    pdl_launch_dependents();
    pdl_wait();  // counts come from the selection kernel
    int running = 0;
    if (threadIdx.x == 0) p.cu_seqlens[0] = 0;
    for (int base = 0; base < p.R; base += kPlanThreads) {
        const int r = base + threadIdx.x;
        const int c = r < p.R ? p.counts[r] : 0;
        int total;
        const int ex = block_exclusive_scan(c, warp_tot, total);
        if (r < p.R) p.cu_seqlens[r + 1] = running + ex + c;
        running += total;
    }
    if (threadIdx.x == 0 && static_cast<long long>(running) > p.capacity)
        atomicOr(p.status, FOCUS_DEV_CAPACITY);
}

}  // namespace

cudaError_t launch_scan(const ScanParams &p, cudaStream_t stream, bool pdl) {
    return launch_kernel(scan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, pdl, p);
}

cudaError_t launch_plan(const PlanParams &p, cudaStream_t stream) {
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_select_compact(const SelectParams &p, cudaStream_t stream, bool pdl) {
    // Without a row copy only the B <= 128 column threads have work.
    return launch_kernel(select_compact_kernel, dim3(p.R), dim3(p.hidden ? 256 : 128), 0, stream,
                         pdl, p);
}

cudaError_t launch_delta(const DeltaParams &p, cudaStream_t stream) {
    delta_kernel<<<p.R, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_reduce(const ReduceParams &p, cudaStream_t stream, bool pdl) {
    return launch_kernel(reduce_kernel, dim3(p.R, p.layers), dim3(128), 0, stream, pdl, p);
}

cudaError_t launch_compact(const CompactParams &p, cudaStream_t stream, bool pdl) {
    long long blocks = (p.capacity + 7) / 8;  // one warp per packed row
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_kernel(compact_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                         pdl, p);
}

}  // namespace focus
