// focus_api.cu -- the extern "C" entry points declared in include/focus.h:
// host-side validation, workspace layout, TMA tensor-map encoding, and the
// kernel sequence of each call.  No allocation, no synchronisation (except in
// focus_read_device_status), no state kept between calls.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <mutex>
#include <thread>

#include <nvtx3/nvToolsExt.h>

#include "focus.h"
#include "focus_device.cuh"
#include "focus_kernels.cuh"

namespace {

using focus::AttnParams;

// A named range around each call, for profiler timelines (NVTX; without a tool
// attached it costs a few nanoseconds).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int row_tiles(const focus_dims_t &d) {
    const int G = d.Hq / d.Hkv;
    return (G * d.B + focus::kTileRows - 1) / focus::kTileRows;
}

// Prefix chunks per attention work item.  A batch whose (layer, request, kv head,
// row tile) items would occupy at most half of the B200's persistent grid
// (2 CTAs x 148 SMs) leaves SMs idle, so each item's prefix is split into up to
// enough chunks for about two waves (at most 16 chunks, each of at least
// kMinChunkTiles key tiles).  Larger batches are not split: a chunk costs a Q
// load and a merge, which only pays where SMs would otherwise idle.  Depends on
// the dims only, so the workspace size does.
constexpr long long kSplitMaxItems = 148;
constexpr long long kSplitTargetItems = 2 * 296;
constexpr int kMaxChunks = 16;

int chunk_max_for(const focus_dims_t &d) {
    const long long items = 2ll * d.R * d.Hkv * row_tiles(d);
    if (items > kSplitMaxItems) return 1;
    const long long c = (kSplitTargetItems + items - 1) / items;
    return static_cast<int>(c < kMaxChunks ? c : kMaxChunks);
}

// Workspace: [status 256 B: the status word; at +64 the exchange counter, at +128 the
//            attention kernel's item counter][order: R int32][partial: 2 x R x Hkv x MT x B fp32]
//            [lists: R x B int32][counts: R int32]   (retained positions under constraints)
//            and with split prefixes (chunk_max_for > 1): [item_base: R+1 int32]
//            [chunk_cnt: 2 x R x Hkv x MT uint32][chunk_stat: groups x (chunk_max-1) x 256 float2]
struct WsLayout {
    size_t status, order, partial, lists, counts, item_base, chunk_cnt, chunk_stat, total;
};

WsLayout ws_layout(const focus_dims_t &d) {
    WsLayout w;
    w.status = 0;
    w.order = kAlign;
    w.partial = w.order + round_up(sizeof(int32_t) * static_cast<size_t>(d.R), kAlign);
    const size_t groups = 2ull * d.R * d.Hkv * row_tiles(d);
    w.lists = w.partial + round_up(sizeof(float) * groups * d.B, kAlign);
    w.counts = w.lists + round_up(sizeof(int32_t) * static_cast<size_t>(d.R) * d.B, kAlign);
    w.total = w.counts + round_up(sizeof(int32_t) * static_cast<size_t>(d.R), kAlign);
    w.item_base = w.chunk_cnt = w.chunk_stat = w.total;
    const int cm = chunk_max_for(d);
    if (cm > 1) {
        w.chunk_cnt = w.item_base + round_up(sizeof(int32_t) * (static_cast<size_t>(d.R) + 1), kAlign);
        w.chunk_stat = w.chunk_cnt + round_up(sizeof(uint32_t) * groups, kAlign);
        w.total = w.chunk_stat + round_up(sizeof(float2) * groups * (cm - 1) * 256, kAlign);
    }
    return w;
}

focus_status_t check_dims(const focus_dims_t *d) {
    if (!d) return FOCUS_ERR_INVALID_ARGUMENT;
    if (d->R < 1 || d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->head_dim < 1 || d->hidden < 1 ||
        d->pool_window < 1)
        return FOCUS_ERR_INVALID_ARGUMENT;
    if (!isfinite(d->softmax_scale) || d->softmax_scale < 0.f) return FOCUS_ERR_INVALID_ARGUMENT;
    if (d->constraints < 0 || d->constraints > 3) return FOCUS_ERR_INVALID_ARGUMENT;
    if (d->score < 0 || d->score > 1) return FOCUS_ERR_INVALID_ARGUMENT;
    if (d->B > 128 || (d->head_dim != 64 && d->head_dim != 128) || d->Hq % d->Hkv != 0 ||
        d->hidden % 8 != 0 || d->pool_window % 2 == 0)
        return FOCUS_ERR_UNSUPPORTED_SHAPE;
    const int G = d->Hq / d->Hkv;
    if (G > focus::kTileRows || focus::kTileRows % G != 0) return FOCUS_ERR_UNSUPPORTED_SHAPE;
    const long long rb = static_cast<long long>(d->R) * d->B;
    if (rb > (1ll << 30)) return FOCUS_ERR_UNSUPPORTED_SHAPE;
    // Work items of the attention kernel; the schedule's item index (round x grid +
    // offset) stays below 2^31 with room for one more round of the grid.
    const long long items = static_cast<long long>(d->R) * 2 * d->Hkv * row_tiles(*d);
    if (items > (1ll << 30)) return FOCUS_ERR_UNSUPPORTED_SHAPE;
    return FOCUS_OK;
}

focus_status_t check_ptr(const void *p, size_t align) {
    if (!p || !aligned(p, align)) return FOCUS_ERR_INVALID_ARGUMENT;
    return FOCUS_OK;
}

focus_status_t check_ws(const focus_dims_t &d, const void *ws, size_t bytes) {
    if (!ws || !aligned(ws, kAlign) || bytes < ws_layout(d).total) return FOCUS_ERR_WORKSPACE;
    return FOCUS_OK;
}

#define FOCUS_TRY(x)                          \
    do {                                      \
        focus_status_t _st = (x);             \
        if (_st != FOCUS_OK) return _st;      \
    } while (0)

#define FOCUS_CUDA(x)                                   \
    do {                                                \
        if ((x) != cudaSuccess) return FOCUS_ERR_CUDA;  \
    } while (0)

// ---------------------------------------------------------------- tracing hook

std::atomic<cudaEvent_t> g_trace_start{nullptr};
std::atomic<cudaEvent_t> g_trace_stop{nullptr};

cudaError_t launch_attn_traced(const AttnParams &p, int head_dim, cudaStream_t s, bool pdl = false) {
    cudaEvent_t a = g_trace_start.load(), b = g_trace_stop.load();
    if (a && b && cudaEventRecord(a, s) != cudaSuccess) return cudaErrorInvalidResourceHandle;
    // An event between two kernels would cut the programmatic overlap, so a traced
    // launch is an ordinary one.
    cudaError_t e = focus::launch_attn_stats(p, head_dim, s, pdl && !(a && b));
    if (e != cudaSuccess) return e;
    if (a && b) return cudaEventRecord(b, s);
    return cudaSuccess;
}

// ---------------------------------------------------------------- tensor maps

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

focus_status_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? FOCUS_OK : FOCUS_ERR_CUDA;
}

// bf16 tensor [rows, heads, d] viewed as (d, heads, rows); box (64, box_heads, box_rows),
// 128-byte swizzle (the layout tcgen05 reads as a K-major operand).
focus_status_t encode_rows_heads_d(CUtensorMap *tm, const void *base, long long rows, int heads,
                                   int d, int box_heads, int box_rows) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                          static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(heads) * d * 2};
    cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_heads), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FOCUS_OK : FOCUS_ERR_CUDA;
}

// Fills the tensor maps of one layer.  The prefix map views `total_prefix` rows of
// k_prefix (a packed prefix buffer or a page pool) in boxes of `prefix_box_rows`.
focus_status_t encode_layer(AttnParams &p, int layer, const focus_dims_t &d, const void *q,
                            const void *k_prefix, long long total_prefix, const void *k_block,
                            int prefix_box_rows = focus::kTileKeys) {
    const int G = d.Hq / d.Hkv;
    const long long rb = static_cast<long long>(d.R) * d.B;
    FOCUS_TRY(encode_rows_heads_d(&p.tm_q[layer], q, rb, d.Hq, d.head_dim, G, focus::kTileRows / G));
    // With no prefix rows anywhere the prefix map is never read; point it at the block keys.
    if (total_prefix > 0)
        FOCUS_TRY(encode_rows_heads_d(&p.tm_kp[layer], k_prefix, total_prefix, d.Hkv, d.head_dim, 1,
                                      prefix_box_rows));
    else
        FOCUS_TRY(encode_rows_heads_d(&p.tm_kp[layer], k_block, rb, d.Hkv, d.head_dim, 1,
                                      focus::kTileKeys));
    FOCUS_TRY(encode_rows_heads_d(&p.tm_kb[layer], k_block, rb, d.Hkv, d.head_dim, 1, p.n_blk));
    return FOCUS_OK;
}

void fill_common(AttnParams &p, const focus_dims_t &d, const int32_t *cu_prefix,
                 long long total_prefix, uint8_t *ws, int n_layers) {
    const WsLayout w = ws_layout(d);
    p.cu_prefix = cu_prefix;
    p.order = reinterpret_cast<const int32_t *>(ws + w.order);
    p.partial = reinterpret_cast<float *>(ws + w.partial);
    p.status = reinterpret_cast<uint32_t *>(ws + w.status);
    p.item_counter = reinterpret_cast<unsigned int *>(ws + w.status + 128);
    p.total_prefix = total_prefix;
    p.R = d.R;
    p.B = d.B;
    p.Hq = d.Hq;
    p.Hkv = d.Hkv;
    p.G = d.Hq / d.Hkv;
    p.MT = row_tiles(d);
    p.n_layers = n_layers;
    p.tok_per_tile = focus::kTileRows / p.G;
    p.n_blk = (d.B + 15) / 16 * 16;
    p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
}

// One layer's attention inputs.
struct LayerIn {
    const void *q, *k_prefix, *k_block;
};

// The attention parameters of a call over `layers` layers: with one layer `l1` is
// it (a single-layer call, or the layer-1 score); with two, `l0` then `l1`.  With
// `lse0` (layer 0's row log-sum-exps given) layer 0 streams no prefix, so its
// prefix map is never read.
focus_status_t setup_attention(AttnParams &p, const focus_dims_t &d, int layers, const LayerIn &l0,
                               const LayerIn &l1, const int32_t *cu_prefix,
                               long long total_prefix, uint8_t *ws,
                               int prefix_box = focus::kTileKeys, const float *lse0 = nullptr) {
    memset(&p, 0, sizeof p);
    fill_common(p, d, cu_prefix, total_prefix, ws, layers);
    p.chunk_max = chunk_max_for(d);
    if (p.chunk_max > 1) {
        const WsLayout w = ws_layout(d);
        p.item_base = reinterpret_cast<const int32_t *>(ws + w.item_base);
        p.chunk_cnt = reinterpret_cast<unsigned int *>(ws + w.chunk_cnt);
        p.chunk_stat = reinterpret_cast<float2 *>(ws + w.chunk_stat);
    }
    if (layers == 1) {
        FOCUS_TRY(encode_layer(p, 0, d, l1.q, l1.k_prefix, total_prefix, l1.k_block, prefix_box));
        p.tm_q[1] = p.tm_q[0];
        p.tm_kp[1] = p.tm_kp[0];
        p.tm_kb[1] = p.tm_kb[0];
        return FOCUS_OK;
    }
    if (lse0)
        FOCUS_TRY(encode_layer(p, 0, d, l0.q, nullptr, 0, l0.k_block));
    else
        FOCUS_TRY(encode_layer(p, 0, d, l0.q, l0.k_prefix, total_prefix, l0.k_block, prefix_box));
    FOCUS_TRY(encode_layer(p, 1, d, l1.q, l1.k_prefix, total_prefix, l1.k_block, prefix_box));
    p.lse0 = lse0;
    return FOCUS_OK;
}

// The planner's share of an attention launch: the kernel's item counter zeroed and,
// with split prefixes, per-rank item offsets and zeroed chunk counters.
void plan_attention(focus::PlanParams &pp, const AttnParams &p) {
    pp.item_counter = p.item_counter;
    if (p.chunk_max <= 1) return;
    pp.chunk_max = p.chunk_max;
    // With layer 0's log-sum-exps given, its groups have no prefix: one item each.
    pp.single_groups = (p.lse0 && p.n_layers == 2) ? p.Hkv * p.MT : 0;
    pp.per_req = p.n_layers * p.Hkv * p.MT - pp.single_groups;
    pp.n_groups = p.n_layers * p.R * p.Hkv * p.MT;
    pp.item_base = const_cast<int32_t *>(p.item_base);
    pp.chunk_cnt = p.chunk_cnt;
}

focus_status_t check_attn_inputs(const focus_dims_t &d, const void *q, const void *k_prefix,
                                 const int32_t *cu_prefix, long long total_prefix,
                                 const void *k_block) {
    FOCUS_TRY(check_ptr(q, 16));
    FOCUS_TRY(check_ptr(k_block, 16));
    FOCUS_TRY(check_ptr(cu_prefix, 4));
    if (total_prefix < 0 || total_prefix > 0x7fffffffll) return FOCUS_ERR_INVALID_ARGUMENT;
    if (total_prefix > 0) FOCUS_TRY(check_ptr(k_prefix, 16));
    return FOCUS_OK;
}

}  // namespace

extern "C" {

size_t focus_workspace_size(const focus_dims_t *dims) {
    if (check_dims(dims) != FOCUS_OK) return 0;
    return ws_layout(*dims).total;
}

focus_status_t focus_plan_capacity(const focus_dims_t *dims, const uint8_t *decoded_host,
                                   const int32_t *budget_host, int dynamic,
                                   int64_t *capacity_out) {
    FOCUS_TRY(check_dims(dims));
    if (!decoded_host || !capacity_out || (!dynamic && !budget_host))
        return FOCUS_ERR_INVALID_ARGUMENT;
    const focus_dims_t &d = *dims;
    int64_t rows = 0;
    for (int r = 0; r < d.R; ++r) {
        const uint8_t *dec = decoded_host + static_cast<size_t>(r) * d.B;
        int64_t masked = 0;
        for (int j = 0; j < d.B; ++j) masked += dec[j] == 0;
        // a dynamic budget is at most the masked count; a given one is clamped to it
        const int64_t want = dynamic ? masked : (budget_host[r] > 0 ? budget_host[r] : 0);
        const int64_t k = want < masked ? want : masked;
        if (d.constraints == 0)
            rows += k;
        else if (k > 0)
            rows += masked + k < d.B ? masked + k : d.B;
    }
    *capacity_out = rows;
    return FOCUS_OK;
}

focus_status_t focus_clear_device_status(void *workspace, size_t workspace_bytes, void *stream) {
    if (!workspace || !aligned(workspace, kAlign) || workspace_bytes < kAlign)
        return FOCUS_ERR_WORKSPACE;
    // The status word and the exchange's block counter (both in the first 256 bytes).
    FOCUS_CUDA(cudaMemsetAsync(workspace, 0, kAlign, static_cast<cudaStream_t>(stream)));
    return FOCUS_OK;
}

focus_status_t focus_read_device_status(const void *workspace, void *stream, int timeout_ms) {
    if (!workspace || !aligned(workspace, kAlign)) return FOCUS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev;
    FOCUS_CUDA(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    if (cudaEventRecord(ev, s) != cudaSuccess) {
        cudaEventDestroy(ev);
        return FOCUS_ERR_CUDA;
    }
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t q = cudaEventQuery(ev);
        if (q == cudaSuccess) break;
        if (q != cudaErrorNotReady) {
            cudaEventDestroy(ev);
            return FOCUS_ERR_CUDA;
        }
        if (timeout_ms >= 0 &&
            std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms)) {
            cudaEventDestroy(ev);
            return FOCUS_ERR_TIMEOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    cudaEventDestroy(ev);
    uint32_t word = 0;
    FOCUS_CUDA(cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost));
    if (word & focus::FOCUS_DEV_TIMEOUT) return FOCUS_ERR_TIMEOUT;
    if (word & focus::FOCUS_DEV_BAD_INPUT) return FOCUS_ERR_DEVICE_CHECK;
    if (word & focus::FOCUS_DEV_CAPACITY) return FOCUS_ERR_CAPACITY;
    return FOCUS_OK;
}

focus_status_t focus_attn_stats(const focus_dims_t *dims, const void *q, const void *k_prefix,
                                const int32_t *cu_prefix, int64_t total_prefix,
                                const void *k_block, float *importance, void *workspace,
                                size_t workspace_bytes, void *stream) {
    NvtxRange nvtx_range("focus_attn_stats");
    FOCUS_TRY(check_dims(dims));
    const focus_dims_t &d = *dims;
    FOCUS_TRY(check_attn_inputs(d, q, k_prefix, cu_prefix, total_prefix, k_block));
    FOCUS_TRY(check_ptr(importance, 4));
    FOCUS_TRY(check_ws(d, workspace, workspace_bytes));
    FOCUS_TRY(get_encoder());
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    AttnParams p;
    FOCUS_TRY(setup_attention(p, d, 1, LayerIn{}, LayerIn{q, k_prefix, k_block}, cu_prefix,
                              total_prefix, ws));

    focus::PlanParams pp;
    memset(&pp, 0, sizeof pp);
    pp.cu_prefix = cu_prefix;
    pp.order = const_cast<int32_t *>(p.order);
    pp.status = p.status;
    pp.R = d.R;
    pp.B = d.B;
    plan_attention(pp, p);
    FOCUS_CUDA(focus::launch_plan(pp, s));
    FOCUS_CUDA(launch_attn_traced(p, d.head_dim, s));
    focus::ReduceParams rp{p.partial, importance, d.R, d.B, d.Hkv, p.MT, 1};
    FOCUS_CUDA(focus::launch_reduce(rp, s));
    return FOCUS_OK;
}

focus_status_t focus_importance_delta(const focus_dims_t *dims, const float *i0, const float *i1,
                                      const uint8_t *decoded, float *delta, float *raw_delta,
                                      void *stream) {
    NvtxRange nvtx_range("focus_importance_delta");
    FOCUS_TRY(check_dims(dims));
    FOCUS_TRY(check_ptr(i0, 4));
    FOCUS_TRY(check_ptr(i1, 4));
    FOCUS_TRY(check_ptr(decoded, 1));
    FOCUS_TRY(check_ptr(delta, 4));
    if (raw_delta) FOCUS_TRY(check_ptr(raw_delta, 4));
    focus::DeltaParams p{i0, i1, decoded, delta, raw_delta, dims->R, dims->B, dims->pool_window};
    FOCUS_CUDA(focus::launch_delta(p, static_cast<cudaStream_t>(stream)));
    return FOCUS_OK;
}

focus_status_t focus_topk_select(const focus_dims_t *dims, const float *delta,
                                 const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx,
                                 int32_t *cu_seqlens, int64_t capacity, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    NvtxRange nvtx_range("focus_topk_select");
    FOCUS_TRY(check_dims(dims));
    const focus_dims_t &d = *dims;
    FOCUS_TRY(check_ptr(delta, 4));
    FOCUS_TRY(check_ptr(decoded, 1));
    FOCUS_TRY(check_ptr(budget, 4));
    FOCUS_TRY(check_ptr(cu_seqlens, 4));
    if (capacity < 0) return FOCUS_ERR_INVALID_ARGUMENT;
    if (capacity > 0) FOCUS_TRY(check_ptr(kept_idx, 4));
    FOCUS_TRY(check_ws(d, workspace, workspace_bytes));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + ws_layout(d).status);

    const WsLayout w = ws_layout(d);
    focus::SelectParams sp;
    memset(&sp, 0, sizeof sp);
    sp.delta_in = delta;
    sp.decoded = decoded;
    sp.cu_seqlens = cu_seqlens;
    sp.kept_idx = kept_idx;
    sp.status = status;
    sp.capacity = capacity;
    sp.R = d.R;
    sp.B = d.B;
    sp.pool_window = d.pool_window;
    if (d.constraints) {
        // Retained lists per request, then cu_seqlens, then kept_idx from the lists.
        sp.constraints = d.constraints;
        sp.budget = budget;
        sp.lists = reinterpret_cast<int32_t *>(ws + w.lists);
        sp.counts = reinterpret_cast<int32_t *>(ws + w.counts);
        FOCUS_CUDA(focus::launch_select_compact(sp, s));
        focus::ScanParams sc{sp.counts, cu_seqlens, status, capacity, d.R};
        FOCUS_CUDA(focus::launch_scan(sc, s, /*pdl=*/true));
        focus::CompactParams cp{nullptr, nullptr, cu_seqlens, nullptr, status, capacity,
                                d.R, d.B, d.hidden, sp.lists, kept_idx};
        FOCUS_CUDA(focus::launch_compact(cp, s, /*pdl=*/true));
        return FOCUS_OK;
    }

    focus::PlanParams pp;
    memset(&pp, 0, sizeof pp);
    pp.decoded = decoded;
    pp.budget = budget;
    pp.cu_seqlens = cu_seqlens;
    pp.status = status;
    pp.capacity = capacity;
    pp.R = d.R;
    pp.B = d.B;
    FOCUS_CUDA(focus::launch_plan(pp, s));
    FOCUS_CUDA(focus::launch_select_compact(sp, s));
    return FOCUS_OK;
}

focus_status_t focus_compact(const focus_dims_t *dims, const void *hidden, const int32_t *kept_idx,
                             const int32_t *cu_seqlens, void *packed, int64_t capacity,
                             void *workspace, size_t workspace_bytes, void *stream) {
    NvtxRange nvtx_range("focus_compact");
    FOCUS_TRY(check_dims(dims));
    const focus_dims_t &d = *dims;
    FOCUS_TRY(check_ptr(hidden, 16));
    FOCUS_TRY(check_ptr(cu_seqlens, 4));
    if (capacity < 0) return FOCUS_ERR_INVALID_ARGUMENT;
    if (capacity > 0) {
        FOCUS_TRY(check_ptr(kept_idx, 4));
        FOCUS_TRY(check_ptr(packed, 16));
    }
    FOCUS_TRY(check_ws(d, workspace, workspace_bytes));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    focus::CompactParams p{static_cast<const uint16_t *>(hidden), kept_idx, cu_seqlens,
                           static_cast<uint16_t *>(packed),
                           reinterpret_cast<uint32_t *>(ws + ws_layout(d).status), capacity,
                           d.R, d.B, d.hidden, nullptr, nullptr};
    FOCUS_CUDA(focus::launch_compact(p, static_cast<cudaStream_t>(stream)));
    return FOCUS_OK;
}

}  // extern "C"

namespace {

// The fused step; `lse0` (nullable) supplies layer 0's row log-sum-exps, in which
// case layer 0 reads only Q0 and its block keys (k0_prefix is not used).
// Paged prefix keys: k*_prefix point at page pools [num_pages, page_size, Hkv, d].
struct Paging {
    const int32_t *page_table;  // [R, max_pages]
    const int32_t *prefix_len;  // [R]
    int max_pages, num_pages, page_size;
};

focus_status_t check_paging(const Paging &pg) {
    FOCUS_TRY(check_ptr(pg.page_table, 4));
    FOCUS_TRY(check_ptr(pg.prefix_len, 4));
    if (pg.max_pages < 1 || pg.num_pages < 1) return FOCUS_ERR_INVALID_ARGUMENT;
    if (pg.page_size < 8 || pg.page_size > (1 << 16) || (pg.page_size & (pg.page_size - 1)))
        return FOCUS_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(pg.num_pages) * pg.page_size > 0x7fffffffll)
        return FOCUS_ERR_UNSUPPORTED_SHAPE;
    return FOCUS_OK;
}

// The selection half of the step, behind the kernel that produced the column
// sums: selection per request, then the row copy spread over the whole GPU, each
// launched with programmatic dependent launch.  With constraints or a dynamic
// budget the kept counts depend on the data, so the selection writes per-request
// lists, cu_seqlens is scanned afterwards and the copy reads the lists; otherwise
// the planner has already written cu_seqlens.
struct Tail {
    const float *partial;  // [layers][R][groups][B] column sums
    int groups;            // summed per request: Hkv x row tiles, or 1 for a given importance
    int layers;            // 2: rank by I1 - I0; 1: by I1 alone
    uint32_t *status;
    const void *hidden;
    const uint8_t *decoded;
    const int32_t *budget;
    const float *decode_avg;
    float budget_alpha;
    int32_t *budget_out;
    int32_t *kept_idx;
    int32_t *cu_seqlens;
    void *packed;
    int64_t capacity;
    float *delta_out, *i0_out, *i1_out;
    const uint32_t *ex_flags;  // peer exchange: wait for these flags to show ex_epoch
    uint32_t ex_epoch;
};

bool tail_uses_lists(const focus_dims_t &d, const Tail &t) {
    return d.constraints != 0 || t.decode_avg != nullptr;
}

focus_status_t launch_tail(const focus_dims_t &d, const Tail &t, uint8_t *ws, cudaStream_t s) {
    focus::SelectParams sp;
    memset(&sp, 0, sizeof sp);
    sp.partial = t.partial;
    sp.decoded = t.decoded;
    sp.cu_seqlens = t.cu_seqlens;
    sp.kept_idx = t.kept_idx;
    sp.delta_out = t.delta_out;
    sp.i0_out = t.i0_out;
    sp.i1_out = t.i1_out;
    sp.status = t.status;
    sp.capacity = t.capacity;
    sp.R = d.R;
    sp.B = d.B;
    sp.Hkv = t.groups;
    sp.MT = 1;
    sp.H = d.hidden;
    sp.pool_window = d.pool_window;
    sp.layers = t.layers;
    sp.ex_flags = t.ex_flags;
    sp.ex_epoch = t.ex_epoch;
    if (tail_uses_lists(d, t)) {
        const WsLayout w = ws_layout(d);
        sp.constraints = d.constraints;
        sp.budget = t.budget;
        sp.decode_avg = t.decode_avg;
        sp.budget_alpha = t.budget_alpha;
        sp.budget_out = t.budget_out;
        sp.lists = reinterpret_cast<int32_t *>(ws + w.lists);
        sp.counts = reinterpret_cast<int32_t *>(ws + w.counts);
        FOCUS_CUDA(focus::launch_select_compact(sp, s, /*pdl=*/true));
        focus::ScanParams sc{sp.counts, t.cu_seqlens, t.status, t.capacity, d.R};
        FOCUS_CUDA(focus::launch_scan(sc, s, /*pdl=*/true));
        focus::CompactParams cp{static_cast<const uint16_t *>(t.hidden), nullptr, t.cu_seqlens,
                                static_cast<uint16_t *>(t.packed), t.status, t.capacity, d.R, d.B,
                                d.hidden, sp.lists, t.kept_idx};
        FOCUS_CUDA(focus::launch_compact(cp, s, /*pdl=*/true));
        return FOCUS_OK;
    }
    FOCUS_CUDA(focus::launch_select_compact(sp, s, /*pdl=*/true));
    focus::CompactParams cp{static_cast<const uint16_t *>(t.hidden), t.kept_idx, t.cu_seqlens,
                            static_cast<uint16_t *>(t.packed), t.status, t.capacity, d.R, d.B,
                            d.hidden, nullptr, nullptr};
    FOCUS_CUDA(focus::launch_compact(cp, s, /*pdl=*/true));
    return FOCUS_OK;
}

// What the host validation of a fused call derives from its arguments.
struct EvictInputs {
    const int32_t *cu_prefix;  // packed offsets, or the paged prefix lengths
    long long total_prefix;    // rows of the prefix buffers (or page-pool rows)
    int prefix_box;            // rows per prefix TMA box
    Paging pg;
    bool paged;
};

// Every host-side check of the fused step, in order; nothing is enqueued.
focus_status_t check_evict(const focus_dims_t *dims, const focus_evict_args_t &x, EvictInputs *in) {
    FOCUS_TRY(check_dims(dims));
    const focus_dims_t &d = *dims;
    const bool layer1_only = d.score == FOCUS_SCORE_LAYER1;
    const bool dynamic = x.decode_avg != nullptr;
    in->cu_prefix = x.cu_prefix;
    in->total_prefix = x.total_prefix;
    in->prefix_box = focus::kTileKeys;
    in->pg = Paging{x.page_table, x.prefix_len, x.max_pages, x.num_pages, x.page_size};
    in->paged = x.page_table != nullptr;
    if (in->paged) {  // the page pools stand in for the packed prefix buffers
        FOCUS_TRY(check_paging(in->pg));
        in->total_prefix = static_cast<long long>(in->pg.num_pages) * in->pg.page_size;
        in->prefix_box = in->pg.page_size < focus::kTileKeys ? in->pg.page_size : focus::kTileKeys;
        in->cu_prefix = in->pg.prefix_len;  // only checked for presence below; lengths come from here
    }
    if (x.lse0) {
        if (layer1_only) return FOCUS_ERR_INVALID_ARGUMENT;
        FOCUS_TRY(check_ptr(x.lse0, 4));
        FOCUS_TRY(check_attn_inputs(d, x.q0, nullptr, in->cu_prefix, 0, x.k0_block));
    } else if (!layer1_only) {
        FOCUS_TRY(check_attn_inputs(d, x.q0, x.k0_prefix, in->cu_prefix, in->total_prefix,
                                    x.k0_block));
    }
    FOCUS_TRY(check_attn_inputs(d, x.q1, x.k1_prefix, in->cu_prefix, in->total_prefix, x.k1_block));
    FOCUS_TRY(check_ptr(x.hidden, 16));
    FOCUS_TRY(check_ptr(x.decoded, 1));
    if (dynamic) {
        FOCUS_TRY(check_ptr(x.decode_avg, 4));
        if (!isfinite(x.budget_alpha) || x.budget_alpha < 0.f) return FOCUS_ERR_INVALID_ARGUMENT;
        if (x.budget_out) FOCUS_TRY(check_ptr(x.budget_out, 4));
    } else {
        FOCUS_TRY(check_ptr(x.budget, 4));
    }
    FOCUS_TRY(check_ptr(x.cu_seqlens, 4));
    if (x.capacity < 0) return FOCUS_ERR_INVALID_ARGUMENT;
    if (x.capacity > 0) {
        FOCUS_TRY(check_ptr(x.kept_idx, 4));
        FOCUS_TRY(check_ptr(x.packed, 16));
    }
    if (x.delta_out) FOCUS_TRY(check_ptr(x.delta_out, 4));
    if (x.i0_out) FOCUS_TRY(check_ptr(x.i0_out, 4));
    if (x.i1_out) FOCUS_TRY(check_ptr(x.i1_out, 4));
    FOCUS_TRY(check_ws(d, x.workspace, x.workspace_bytes));
    return get_encoder();
}

focus_status_t evict_impl(const focus_dims_t *dims, const focus_evict_args_t &x) {
    NvtxRange nvtx_range("focus_evict");
    EvictInputs in;
    FOCUS_TRY(check_evict(dims, x, &in));
    const focus_dims_t &d = *dims;
    const bool layer1_only = d.score == FOCUS_SCORE_LAYER1;
    const bool dynamic = x.decode_avg != nullptr;
    const int32_t *cu_prefix = in.cu_prefix;
    const long long total_prefix = in.total_prefix;
    const int prefix_box = in.prefix_box;
    const Paging *paging = in.paged ? &in.pg : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(x.stream);
    uint8_t *ws = static_cast<uint8_t *>(x.workspace);

    // With the layer-1 score (the Figure 13 ablation) layer 0 is not touched.
    AttnParams p;
    FOCUS_TRY(setup_attention(p, d, layer1_only ? 1 : 2, LayerIn{x.q0, x.k0_prefix, x.k0_block},
                              LayerIn{x.q1, x.k1_prefix, x.k1_block}, cu_prefix, total_prefix, ws,
                              prefix_box, layer1_only ? nullptr : x.lse0));
    if (paging) {
        p.cu_prefix = nullptr;
        p.page_table = paging->page_table;
        p.prefix_len = paging->prefix_len;
        p.page_size = paging->page_size;
        p.max_pages = paging->max_pages;
        p.num_pages = paging->num_pages;
        p.page_rows = prefix_box;
    }
    // With constraints or a dynamic budget the kept counts depend on the data, so the
    // selection writes per-request lists and cu_seqlens is scanned afterwards.
    const bool lists = d.constraints != 0 || dynamic;

    focus::PlanParams pp;
    memset(&pp, 0, sizeof pp);
    pp.cu_prefix = paging ? nullptr : cu_prefix;
    pp.prefix_len = paging ? paging->prefix_len : nullptr;
    pp.decoded = x.decoded;
    pp.budget = x.budget;
    pp.order = const_cast<int32_t *>(p.order);
    pp.cu_seqlens = lists ? nullptr : x.cu_seqlens;
    pp.status = p.status;
    pp.capacity = x.capacity;
    pp.R = d.R;
    pp.B = d.B;
    plan_attention(pp, p);
    FOCUS_CUDA(focus::launch_plan(pp, s));
    FOCUS_CUDA(launch_attn_traced(p, d.head_dim, s, /*pdl=*/true));

    Tail t{p.partial, d.Hkv * p.MT, layer1_only ? 1 : 2, p.status, x.hidden, x.decoded,
           x.budget, x.decode_avg, x.budget_alpha, x.budget_out, x.kept_idx, x.cu_seqlens,
           x.packed, x.capacity, x.delta_out, x.i0_out, x.i1_out, nullptr, 0};
    return launch_tail(d, t, ws, s);
}

// Both layers' importance over dims' heads: planner, attention, reduction into
// `importance` [2, R, B] or, with `ex`, into every rank's exchange buffer.
focus_status_t partial_importance_impl(const focus_dims_t *dims, const void *q0,
                                       const void *k0_prefix, const void *k0_block,
                                       const void *q1, const void *k1_prefix,
                                       const void *k1_block, const int32_t *cu_prefix,
                                       int64_t total_prefix, float *importance,
                                       const focus_exchange_t *ex, void *workspace,
                                       size_t workspace_bytes, void *stream) {
    NvtxRange nvtx_range("focus_partial_importance");
    FOCUS_TRY(check_dims(dims));
    const focus_dims_t &d = *dims;
    const bool layer1_only = d.score == FOCUS_SCORE_LAYER1;
    if (!layer1_only)
        FOCUS_TRY(check_attn_inputs(d, q0, k0_prefix, cu_prefix, total_prefix, k0_block));
    FOCUS_TRY(check_attn_inputs(d, q1, k1_prefix, cu_prefix, total_prefix, k1_block));
    FOCUS_TRY(check_ws(d, workspace, workspace_bytes));
    FOCUS_TRY(get_encoder());
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    const int layers = layer1_only ? 1 : 2;
    AttnParams p;
    FOCUS_TRY(setup_attention(p, d, layers, LayerIn{q0, k0_prefix, k0_block},
                              LayerIn{q1, k1_prefix, k1_block}, cu_prefix, total_prefix, ws));
    focus::PlanParams pp;
    memset(&pp, 0, sizeof pp);
    pp.cu_prefix = cu_prefix;
    pp.order = const_cast<int32_t *>(p.order);
    pp.status = p.status;
    pp.R = d.R;
    pp.B = d.B;
    plan_attention(pp, p);
    FOCUS_CUDA(focus::launch_plan(pp, s));
    FOCUS_CUDA(launch_attn_traced(p, d.head_dim, s, /*pdl=*/true));
    focus::ReduceParams rp;
    memset(&rp, 0, sizeof rp);
    rp.partial = p.partial;
    rp.R = d.R;
    rp.B = d.B;
    rp.Hkv = d.Hkv;
    rp.MT = p.MT;
    rp.layers = layers;
    if (ex) {
        rp.ex_bufs = ex->peer_buffers;
        rp.ex_rank = ex->rank;
        rp.ex_world = ex->world;
        rp.ex_epoch = ex->epoch;
        rp.ex_counter = reinterpret_cast<unsigned int *>(ws + ws_layout(d).status + 64);
    } else {
        // With the layer-1 score the single layer goes to importance[1].
        rp.importance = layer1_only ? importance + static_cast<size_t>(d.R) * d.B : importance;
    }
    FOCUS_CUDA(focus::launch_reduce(rp, s, /*pdl=*/true));
    return FOCUS_OK;
}

// Planner, selection and compaction from per-request sums `sums` ([layers][R][groups][B],
// summed over groups in order); with `ex_flags`, after those flags show `ex_epoch`.
focus_status_t evict_from_sums(const focus_dims_t *dims, const float *sums, int groups,
                               const uint32_t *ex_flags, uint32_t ex_epoch, const void *hidden,
                               const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx,
                               int32_t *cu_seqlens, void *packed, int64_t capacity,
                               float *delta_out, void *workspace, size_t workspace_bytes,
                               void *stream) {
    NvtxRange nvtx_range("focus_evict_from_importance");
    const focus_dims_t &d = *dims;
    FOCUS_TRY(check_ptr(hidden, 16));
    FOCUS_TRY(check_ptr(decoded, 1));
    FOCUS_TRY(check_ptr(budget, 4));
    FOCUS_TRY(check_ptr(cu_seqlens, 4));
    if (capacity < 0) return FOCUS_ERR_INVALID_ARGUMENT;
    if (capacity > 0) {
        FOCUS_TRY(check_ptr(kept_idx, 4));
        FOCUS_TRY(check_ptr(packed, 16));
    }
    if (delta_out) FOCUS_TRY(check_ptr(delta_out, 4));
    FOCUS_TRY(check_ws(d, workspace, workspace_bytes));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + ws_layout(d).status);

    const bool layer1_only = d.score == FOCUS_SCORE_LAYER1;
    Tail t{sums, groups, layer1_only ? 1 : 2, status, hidden, decoded, budget, nullptr, 0.f,
           nullptr, kept_idx, cu_seqlens, packed, capacity, delta_out, nullptr, nullptr,
           ex_flags, ex_epoch};
    focus::PlanParams pp;
    memset(&pp, 0, sizeof pp);
    pp.decoded = decoded;
    pp.budget = budget;
    pp.cu_seqlens = tail_uses_lists(d, t) ? nullptr : cu_seqlens;
    pp.status = status;
    pp.capacity = capacity;
    pp.R = d.R;
    pp.B = d.B;
    FOCUS_CUDA(focus::launch_plan(pp, s));
    return launch_tail(d, t, ws, s);
}

}  // namespace

namespace focus {

focus_status_t evict_check(const focus_dims_t *dims, const focus_evict_args_t *args) {
    if (!args) return FOCUS_ERR_INVALID_ARGUMENT;
    EvictInputs in;
    return check_evict(dims, *args, &in);
}

}  // namespace focus

extern "C" {

focus_status_t focus_evict_ex(const focus_dims_t *dims, const focus_evict_args_t *args) {
    if (!args) return FOCUS_ERR_INVALID_ARGUMENT;
    return evict_impl(dims, *args);
}

focus_status_t focus_evict(const focus_dims_t *dims, const void *q0, const void *k0_prefix,
                           const void *k0_block, const void *q1, const void *k1_prefix,
                           const void *k1_block, const int32_t *cu_prefix, int64_t total_prefix,
                           const void *hidden, const uint8_t *decoded, const int32_t *budget,
                           int32_t *kept_idx, int32_t *cu_seqlens, void *packed, int64_t capacity,
                           float *delta_out, float *i0_out, float *i1_out, void *workspace,
                           size_t workspace_bytes, void *stream) {
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
    x.workspace = workspace;
    x.workspace_bytes = workspace_bytes;
    x.stream = stream;
    return evict_impl(dims, x);
}

focus_status_t focus_evict_with_lse0(const focus_dims_t *dims, const float *lse0, const void *q0,
                                     const void *k0_block, const void *q1, const void *k1_prefix,
                                     const void *k1_block, const int32_t *cu_prefix,
                                     int64_t total_prefix, const void *hidden,
                                     const uint8_t *decoded, const int32_t *budget,
                                     int32_t *kept_idx, int32_t *cu_seqlens, void *packed,
                                     int64_t capacity, float *delta_out, float *i0_out,
                                     float *i1_out, void *workspace, size_t workspace_bytes,
                                     void *stream) {
    if (!lse0) return FOCUS_ERR_INVALID_ARGUMENT;
    focus_evict_args_t x;
    memset(&x, 0, sizeof x);
    x.q0 = q0;
    x.k0_block = k0_block;
    x.lse0 = lse0;
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
    x.workspace = workspace;
    x.workspace_bytes = workspace_bytes;
    x.stream = stream;
    return evict_impl(dims, x);
}

focus_status_t focus_evict_paged(const focus_dims_t *dims, const void *q0, const void *k0_pages,
                                 const void *k0_block, const void *q1, const void *k1_pages,
                                 const void *k1_block, const int32_t *page_table, int32_t max_pages,
                                 const int32_t *prefix_len, int32_t num_pages, int32_t page_size,
                                 const void *hidden, const uint8_t *decoded,
                                 const int32_t *budget, int32_t *kept_idx, int32_t *cu_seqlens,
                                 void *packed, int64_t capacity, float *delta_out, float *i0_out,
                                 float *i1_out, void *workspace, size_t workspace_bytes,
                                 void *stream) {
    if (!page_table) return FOCUS_ERR_INVALID_ARGUMENT;
    focus_evict_args_t x;
    memset(&x, 0, sizeof x);
    x.q0 = q0;
    x.k0_prefix = k0_pages;
    x.k0_block = k0_block;
    x.q1 = q1;
    x.k1_prefix = k1_pages;
    x.k1_block = k1_block;
    x.page_table = page_table;
    x.prefix_len = prefix_len;
    x.max_pages = max_pages;
    x.num_pages = num_pages;
    x.page_size = page_size;
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
    x.workspace = workspace;
    x.workspace_bytes = workspace_bytes;
    x.stream = stream;
    return evict_impl(dims, x);
}

focus_status_t focus_partial_importance(const focus_dims_t *dims, const void *q0,
                                        const void *k0_prefix, const void *k0_block,
                                        const void *q1, const void *k1_prefix,
                                        const void *k1_block, const int32_t *cu_prefix,
                                        int64_t total_prefix, float *importance, void *workspace,
                                        size_t workspace_bytes, void *stream) {
    FOCUS_TRY(check_ptr(importance, 4));
    return partial_importance_impl(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block,
                                   cu_prefix, total_prefix, importance, nullptr, workspace,
                                   workspace_bytes, stream);
}

size_t focus_exchange_buffer_size(const focus_dims_t *dims, int32_t world) {
    if (check_dims(dims) != FOCUS_OK || world < 1 || world > focus::kMaxExchangeWorld) return 0;
    return focus::ex_layout(dims->R, dims->B, world).total;
}

focus_status_t focus_partial_importance_push(const focus_dims_t *dims, const void *q0,
                                             const void *k0_prefix, const void *k0_block,
                                             const void *q1, const void *k1_prefix,
                                             const void *k1_block, const int32_t *cu_prefix,
                                             int64_t total_prefix, const focus_exchange_t *exchange,
                                             void *workspace, size_t workspace_bytes,
                                             void *stream) {
    if (!exchange) return FOCUS_ERR_INVALID_ARGUMENT;
    const focus_exchange_t &x = *exchange;
    FOCUS_TRY(check_ptr(x.peer_buffers, 8));
    if (x.world < 1 || x.world > focus::kMaxExchangeWorld || x.rank < 0 || x.rank >= x.world ||
        x.epoch == 0)
        return FOCUS_ERR_INVALID_ARGUMENT;
    return partial_importance_impl(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block,
                                   cu_prefix, total_prefix, nullptr, &x, workspace,
                                   workspace_bytes, stream);
}

focus_status_t focus_evict_from_exchange(const focus_dims_t *dims, const void *exchange_buffer,
                                         int32_t world, uint32_t epoch, const void *hidden,
                                         const uint8_t *decoded, const int32_t *budget,
                                         int32_t *kept_idx, int32_t *cu_seqlens, void *packed,
                                         int64_t capacity, float *delta_out, void *workspace,
                                         size_t workspace_bytes, void *stream) {
    FOCUS_TRY(check_dims(dims));
    FOCUS_TRY(check_ptr(exchange_buffer, kAlign));
    if (world < 1 || world > focus::kMaxExchangeWorld || epoch == 0)
        return FOCUS_ERR_INVALID_ARGUMENT;
    const focus_dims_t &d = *dims;
    const focus::ExLayout el = focus::ex_layout(d.R, d.B, world);
    const uint8_t *buf = static_cast<const uint8_t *>(exchange_buffer);
    const float *slots = reinterpret_cast<const float *>(buf) +
                         static_cast<size_t>(epoch & 1u) * 2 * d.R * world * d.B;
    const uint32_t *flags = reinterpret_cast<const uint32_t *>(buf + el.flags);
    return evict_from_sums(dims, slots, world, flags, epoch, hidden, decoded, budget, kept_idx,
                           cu_seqlens, packed, capacity, delta_out, workspace, workspace_bytes,
                           stream);
}

focus_status_t focus_evict_from_importance(const focus_dims_t *dims, const float *importance,
                                           const void *hidden, const uint8_t *decoded,
                                           const int32_t *budget, int32_t *kept_idx,
                                           int32_t *cu_seqlens, void *packed, int64_t capacity,
                                           float *delta_out, void *workspace,
                                           size_t workspace_bytes, void *stream) {
    FOCUS_TRY(check_dims(dims));
    FOCUS_TRY(check_ptr(importance, 4));
    // With the layer-1 score only importance[1] is read.
    const float *sums = dims->score == FOCUS_SCORE_LAYER1
                            ? importance + static_cast<size_t>(dims->R) * dims->B
                            : importance;
    return evict_from_sums(dims, sums, 1, nullptr, 0, hidden, decoded, budget, kept_idx,
                           cu_seqlens, packed, capacity, delta_out, workspace, workspace_bytes,
                           stream);
}

const char *focus_status_string(focus_status_t st) {
    switch (st) {
        case FOCUS_OK: return "FOCUS_OK";
        case FOCUS_ERR_INVALID_ARGUMENT: return "FOCUS_ERR_INVALID_ARGUMENT";
        case FOCUS_ERR_UNSUPPORTED_SHAPE: return "FOCUS_ERR_UNSUPPORTED_SHAPE";
        case FOCUS_ERR_CAPACITY: return "FOCUS_ERR_CAPACITY";
        case FOCUS_ERR_WORKSPACE: return "FOCUS_ERR_WORKSPACE";
        case FOCUS_ERR_CUDA: return "FOCUS_ERR_CUDA";
        case FOCUS_ERR_DEVICE_CHECK: return "FOCUS_ERR_DEVICE_CHECK";
        case FOCUS_ERR_TIMEOUT: return "FOCUS_ERR_TIMEOUT";
    }
    return "FOCUS_ERR_UNKNOWN";
}

int focus_abi_version(void) { return FOCUS_ABI_VERSION; }

void focus_set_trace_events(void *start_event, void *stop_event) {
    g_trace_start.store(static_cast<cudaEvent_t>(start_event));
    g_trace_stop.store(static_cast<cudaEvent_t>(stop_event));
}

}  // extern "C"
