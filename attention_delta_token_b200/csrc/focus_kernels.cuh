// focus_kernels.cuh -- launch parameters and launchers of the FOCUS eviction kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace focus {

// Launches `kernel` on `stream`; with `pdl` the launch carries the programmatic
// stream serialization attribute, so it may start while the previous kernel on
// the stream is still running (the kernel itself waits with griddepcontrol.wait
// before touching that kernel's outputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- attention statistics
// Work item = one (layer, request, kv head, 128-row query tile); persistent CTAs
// walk the items.  An item's 128 query rows are the G = Hq/Hkv query heads of
// that kv head for 128/G consecutive block tokens (row = token * G + head-in-
// group), so every key tile that TMA brings in is used by all query heads that
// read it.
constexpr int kTileRows = 128;   // UMMA M: query rows per CTA
constexpr int kTileKeys = 128;   // UMMA N: keys per prefix tile
constexpr int kStages = 2;       // key-tile ring depth (two CTAs share an SM)
constexpr int kAttnThreads = 320;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-9 softmax
constexpr int kSoftmaxWarps = 8;   // two warpgroups, one per half of the S tile columns
constexpr int kTmemCols = 256;   // two 128-column fp32 S buffers

struct AttnParams {
    CUtensorMap tm_q[2];    // per layer: Q  [R*B, Hq, d], box (64, G, 128/G)
    CUtensorMap tm_kp[2];   // per layer: prefix K [total_prefix, Hkv, d], box (64, 1, 128)
    CUtensorMap tm_kb[2];   // per layer: block K  [R*B, Hkv, d], box (64, 1, n_blk)
    const int32_t *cu_prefix;  // [R+1]
    const int32_t *order;      // [R] request processing order (longest prefix first)
    float *partial;            // [n_layers][R][Hkv][MT][B] column sums per kv head / row tile
    uint32_t *status;          // device status word
    unsigned int *item_counter;  // items claimed after the first round (zeroed by the planner)
    int dynamic;               // claim items dynamically (set at launch from the item count)
    long long total_prefix;
    int R, B, Hq, Hkv, G, MT, n_layers;
    int tok_per_tile;          // 128 / G block tokens per row tile
    int n_blk;                 // keys in the block tile: B rounded up to 16
    float scale_log2;          // softmax_scale * log2(e)
    const float *lse0;         // [R, B, Hq] layer-0 row log-sum-exps (natural log) or null:
                               // given, layer-0 items read only the block keys
    // Paged prefix keys (page_table != null): prefix key t of request r is row
    // page_table[r * max_pages + t / page_size] * page_size + t % page_size of the
    // page pool that tm_kp views ([num_pages * page_size, Hkv, d], box rows page_rows).
    const int32_t *page_table;  // [R, max_pages]
    const int32_t *prefix_len;  // [R]
    int page_size, max_pages, num_pages, page_rows;
    // Split prefixes (chunk_max > 1, small batches): a request's prefix tiles are
    // split evenly into prefix_chunks(L, chunk_max) chunks, one work item each, the
    // last of which also takes the block tile.  The items of request rank q are
    // [item_base[q], item_base[q+1]) (chunk innermost).  Every chunk but the last
    // writes its rows' (m, l) to chunk_stat and counts itself in chunk_cnt[group];
    // the last waits for the count and merges in chunk order.
    int chunk_max;
    const int32_t *item_base;   // [R+1] by request rank (written by the planner)
    unsigned int *chunk_cnt;    // [n_layers][R][Hkv][MT] (zeroed by the planner)
    float2 *chunk_stat;         // [n_layers][R][Hkv][MT][chunk_max - 1][2 halves][128 rows]
};

// Prefix chunks of a request with L prefix keys: at most chunk_max, each of at
// least kMinChunkTiles key tiles.
constexpr int kMinChunkTiles = 4;
__host__ __device__ inline int prefix_chunks(int L, int chunk_max) {
    const int n_pre = (L > 0 ? L : 0) / kTileKeys + ((L > 0 && L % kTileKeys) ? 1 : 0);
    const int c = n_pre / kMinChunkTiles;
    return c < 1 ? 1 : (c < chunk_max ? c : chunk_max);
}

size_t attn_smem_bytes(int head_dim);
cudaError_t launch_attn_stats(const AttnParams &p, int head_dim, cudaStream_t stream,
                              bool pdl = false);

// ---------------------------------------------------------------- planning
struct PlanParams {
    const int32_t *cu_prefix;  // [R+1] (packed prefix) or null
    const int32_t *prefix_len; // [R] (paged prefix) or null
    const uint8_t *decoded;    // [R,B] or null (no counts)
    const int32_t *budget;     // [R]   or null
    int32_t *order;            // [R]   or null (no ordering)
    int32_t *cu_seqlens;       // [R+1] or null
    uint32_t *status;
    long long capacity;
    int R, B;
    // Split prefixes (item_base != null): per-rank item offsets of the attention
    // kernel, single_groups + prefix_chunks(L, chunk_max) * per_req items per
    // request (single_groups: layer-0 groups that stream no prefix when layer 0's
    // row log-sum-exps are given), and the chunk counters zeroed.
    int chunk_max, per_req, single_groups, n_groups;
    int32_t *item_base;        // [R+1]
    unsigned int *chunk_cnt;   // [n_groups]
    unsigned int *item_counter;  // the attention kernel's item counter, zeroed (or null)
};
cudaError_t launch_plan(const PlanParams &p, cudaStream_t stream);

// ---------------------------------------------------------------- select / compact
struct SelectParams {
    const float *partial;      // [2][R][Hkv][MT][B] (fused path) or null
    const float *delta_in;     // [R,B] pooled+masked delta (stand-alone select) or null
    const uint8_t *decoded;    // [R,B]
    const int32_t *cu_seqlens; // [R+1] (written by the planner)
    int32_t *kept_idx;         // [capacity]
    const uint16_t *hidden;    // [R,B,H] bf16 bits, null = no compaction
    uint16_t *packed;          // [capacity,H]
    float *delta_out, *i0_out, *i1_out, *raw_out;  // optional [R,B]
    uint32_t *status;
    long long capacity;
    int R, B, Hkv, MT, H, pool_window;
    int layers;                // 2: score = I1 - I0; 1: only I1 was computed (score = I1)
    // Structural constraints (constraints != 0): the retained positions of request r
    // go to lists[r*B ..] and their number to counts[r]; kept_idx/cu_seqlens are
    // written later by the scan and list-driven compaction.
    int constraints;
    const int32_t *budget;     // [R]
    int32_t *lists;            // [R*B]
    int32_t *counts;           // [R]
    // Dynamic budget (decode_avg != null): K_r from the historical yield and the
    // masked delta's mean + std, written to budget_out (nullable).
    const float *decode_avg;   // [R]
    float budget_alpha;
    int32_t *budget_out;       // [R]
    // Peer exchange (ex_flags != null): `partial` is this rank's slots of the epoch
    // ([layers][R][world = Hkv x MT][B]); wait for flags[0 .. world-1] == ex_epoch first.
    const uint32_t *ex_flags;
    uint32_t ex_epoch;
};

struct ScanParams {
    const int32_t *counts;     // [R]
    int32_t *cu_seqlens;       // [R+1]
    uint32_t *status;
    long long capacity;
    int R;
};
cudaError_t launch_scan(const ScanParams &p, cudaStream_t stream, bool pdl = false);
cudaError_t launch_select_compact(const SelectParams &p, cudaStream_t stream, bool pdl = false);

struct DeltaParams {
    const float *i0, *i1;
    const uint8_t *decoded;
    float *delta, *raw;
    int R, B, pool_window;
};
cudaError_t launch_delta(const DeltaParams &p, cudaStream_t stream);

struct ReduceParams {
    const float *partial;  // [layers][R][Hkv][MT][B]
    float *importance;     // [layers][R][B] (null with the peer exchange)
    int R, B, Hkv, MT, layers;
    // Peer exchange (ex_world > 0, focus_exchange.cuh): the sums go to slot ex_rank
    // of every rank's exchange buffer instead of `importance`.
    void *const *ex_bufs;       // device array [ex_world] of peer-mapped buffers
    int ex_rank, ex_world;
    uint32_t ex_epoch;
    unsigned int *ex_counter;   // blocks done (in the workspace), 0 between launches
};

// Exchange buffer of one rank: slots [2 parities][2 layers][R][world][B] float32,
// then flags [2 parities][world] uint32 at `flags` (256-byte aligned).
constexpr int kMaxExchangeWorld = 8;
struct ExLayout {
    size_t flags, total;
};
__host__ __device__ inline ExLayout ex_layout(int R, int B, int world) {
    const size_t slots = 2ull * 2ull * static_cast<size_t>(R) * world * B * sizeof(float);
    const size_t flags = (slots + 255) / 256 * 256;
    return {flags, flags + 256};
}
cudaError_t launch_reduce(const ReduceParams &p, cudaStream_t stream, bool pdl = false);

struct CompactParams {
    const uint16_t *hidden;    // null: write kept_idx from lists only, copy nothing
    const int32_t *kept_idx, *cu_seqlens;
    uint16_t *packed;
    uint32_t *status;
    long long capacity;
    int R, B, H;
    const int32_t *lists;      // non-null: row t of request r is lists[r*B + t], written to kept_out
    int32_t *kept_out;
};
cudaError_t launch_compact(const CompactParams &p, cudaStream_t stream, bool pdl = false);

}  // namespace focus
