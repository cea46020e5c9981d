/*
 * focus.h -- C ABI of libfocus: FOCUS importance-delta token eviction on B200 (sm_100a).
 *
 * The method ("FOCUS: DLLMs Know How to Tame Their Compute Bound", pith.science
 * review page, section "What carries the argument"): for every request's block
 * of B tokens, I_j is the column sum, over the block's queries and over the
 * query heads, of the row-wise softmax attention weights token j receives (the
 * softmax of a query row runs over the request's prefix keys followed by the B
 * block keys; Referee Report, minor comment on Eq. (2), reads the softmax as
 * row-wise).  I is taken at layer 0 and from the layer-1 Q/K projections
 * (Figure 5 caption: eviction happens right after the layer-1 QKProj).  The
 * importance delta dI = I(layer 1) - I(layer 0) (Eq. 3) is smoothed with
 * MaxPool1D (window 3, stride 1, same padding; Free-Parameter Ledger, Eq. 15),
 * already-decoded positions are masked, the top-K still-masked tokens under a
 * per-request budget K are kept (ties to the lower position), and the kept
 * tokens' hidden rows are packed into a varlen batch with cu_seqlens
 * ("The pith": the remaining layers run only on the retained candidates).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller, row-major,
 *    contiguous.  bf16 tensors are passed as `const void*` holding IEEE bfloat16
 *    and must be 16-byte aligned; int32/float32 arrays 4-byte aligned; the
 *    workspace 256-byte aligned.  The library allocates nothing and
 *    keeps no state between calls; it is thread-safe as long as concurrent
 *    calls use different workspaces.
 *  - `stream` is a cudaStream_t (passed as void*; NULL = legacy default stream).
 *    Every call only enqueues work on `stream` and returns without
 *    synchronising.  The return value reports host-side validation and launch
 *    errors.  Problems that only the device can see (budget rows beyond
 *    `capacity`, malformed cu_prefix, a kernel wait that timed out) are OR-ed
 *    into a status word inside the workspace; read it with
 *    focus_read_device_status().
 *  - Shapes: 1 <= B <= 128; head_dim in {64, 128}; Hq % Hkv == 0 and
 *    G = Hq / Hkv divides 128; hidden % 8 == 0; pool_window odd and >= 1;
 *    R >= 1; constraints in 0..3 and score in 0..1 (else FOCUS_ERR_INVALID_ARGUMENT).  Other shapes
 *    return FOCUS_ERR_UNSUPPORTED_SHAPE, as do R * B > 2^30 and more than 2^30 attention
 *    work items (R x 2 layers x Hkv x ceil(G * B / 128) row tiles).
 *  - Per-request budgets are clamped to [0, masked_r] on the device, so
 *    k_r = min(max(budget[r], 0), masked_r).  Without structural constraints
 *    (dims.constraints == 0) k_r depends only on `decoded` and `budget`, never on
 *    the attention data, so the host scheduler that owns both can size
 *    `capacity` = sum_r k_r exactly.
 *  - Kept positions are written in ascending order per request; requests are
 *    packed in order: request r owns rows cu_seqlens[r] .. cu_seqlens[r+1]-1.
 *  - CUDA graphs: every call that takes the caller's workspace and enqueues
 *    kernels may be captured into a graph (it only launches kernels, with
 *    programmatic dependent launch between them, and never synchronises); this
 *    note does not cover focus_evict_static_scratch.  Make one uncaptured call
 *    per process first (it looks up the driver's tensor-map encoder).  Tensor
 *    maps hold the pointers given at capture, so a replay reads and writes the
 *    same buffers: copy new inputs into them before each replay.
 *    focus_read_device_status synchronises and cannot be captured.
 */
#ifndef FOCUS_H_
#define FOCUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FOCUS_ABI_VERSION 5

#if defined(__GNUC__)
#define FOCUS_API __attribute__((visibility("default")))
#else
#define FOCUS_API
#endif

typedef enum {
    FOCUS_OK = 0,
    FOCUS_ERR_INVALID_ARGUMENT = 1,  /* null/misaligned pointer, negative size, bad scale   */
    FOCUS_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the supported set above              */
    FOCUS_ERR_CAPACITY = 3,          /* device: sum k_r > capacity (extra rows not written) */
    FOCUS_ERR_WORKSPACE = 4,         /* workspace null, misaligned or too small            */
    FOCUS_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed                  */
    FOCUS_ERR_DEVICE_CHECK = 6,      /* device: malformed cu_prefix, page or kept index, or
                                        non-finite inputs (seen as non-finite importance) */
    FOCUS_ERR_TIMEOUT = 7            /* device wait gave up, or status read timed out      */
} focus_status_t;

/* Problem dimensions, shared by all entry points. */
typedef struct {
    int32_t R;             /* requests (blocks) in the batch                          */
    int32_t B;             /* block size                                              */
    int32_t Hq;            /* query heads                                             */
    int32_t Hkv;           /* key/value heads (GQA: query head h reads kv head h/(Hq/Hkv)) */
    int32_t head_dim;      /* d                                                       */
    int32_t hidden;        /* hidden size H of the rows that are compacted            */
    float softmax_scale;   /* logit = softmax_scale * q.k (usually 1/sqrt(d)); finite, >= 0 */
    int32_t pool_window;   /* MaxPool1D window (odd; the method uses 3)               */
    int32_t constraints;   /* structural constraints on the retained set, bit mask:
                              FOCUS_KEEP_PREDECESSOR | FOCUS_KEEP_MASKED_BEFORE_RIGHTMOST;
                              0 keeps exactly the top-K candidates                   */
    int32_t score;         /* what is pooled and ranked: FOCUS_SCORE_DELTA (I1 - I0, the
                              method) or FOCUS_SCORE_LAYER1 (I1 alone, the Figure 13
                              ablation: layer 0 is not computed and may be NULL)     */
} focus_dims_t;

#define FOCUS_SCORE_DELTA 0
#define FOCUS_SCORE_LAYER1 1

/*
 * Structural constraints ("What carries the argument": after the top-K candidates
 * are chosen, each candidate's immediate predecessor and all masked tokens before
 * the rightmost candidate are retained as well).  With either bit set:
 *   retained_r = candidates_r
 *              U {j - 1 : j a candidate, j >= 1}            (FOCUS_KEEP_PREDECESSOR;
 *                                                          masked or decoded)
 *              U {masked j : j < rightmost candidate}    (FOCUS_KEEP_MASKED_BEFORE_RIGHTMOST)
 * in ascending order.  The retained count then depends on the attention data,
 * so `capacity` must be an upper bound (sum over requests of
 * min(B, masked_r + k_r) is one) and cu_seqlens is computed on the device.
 */
#define FOCUS_KEEP_PREDECESSOR 1
#define FOCUS_KEEP_MASKED_BEFORE_RIGHTMOST 2

/* Bytes of workspace every entry point below needs for `dims` (256-byte aligned). */
FOCUS_API size_t focus_workspace_size(const focus_dims_t *dims);

/*
 * Rows of the packed batch (the `capacity` to allocate), computed on the host from
 * HOST copies of the scheduler's own arrays; nothing touches the GPU.
 * "What carries the argument" (pith.science review page): each block keeps its
 * top-K still-masked tokens under its budget, so request r keeps
 *   k_r = min(max(budget_host[r], 0), masked_r),  masked_r = #{j : decoded_host[r*B + j] == 0}
 * rows, and without structural constraints (dims->constraints == 0) the batch has
 * exactly sum_r k_r rows -- the value cu_seqlens[R] will hold.  With `dynamic`
 * (the budget is computed on the device from the delta, focus_evict_ex with
 * decode_avg) k_r is bounded by masked_r and budget_host is not read (may be
 * NULL).  With constraints the retained count depends on the attention data and
 * the result is the upper bound sum over requests with k_r > 0 of
 * min(B, masked_r + k_r) (candidates, their predecessors, the other masked tokens).
 *   decoded_host [R, B] uint8 (host), budget_host [R] int32 (host), *capacity_out
 *   (host) receives the row count.
 * Returns FOCUS_ERR_INVALID_ARGUMENT for a null pointer (budget_host only when
 * dynamic is 0) and the check_dims errors of the other entry points for bad dims.
 */
FOCUS_API focus_status_t focus_plan_capacity(const focus_dims_t *dims, const uint8_t *decoded_host,
                                             const int32_t *budget_host, int dynamic,
                                             int64_t *capacity_out);

/* Zero the workspace's status region (enqueued on `stream`): the device status
 * word, the peer exchange's block counter and the attention kernel's item counter
 * (which every call that runs the attention kernel also resets first).  Call once
 * before the first use of a workspace and whenever the status should restart. */
FOCUS_API focus_status_t focus_clear_device_status(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Wait (up to timeout_ms; < 0 waits forever) for the work enqueued so far on
 * `stream` and return the workspace's device status: FOCUS_OK, or the first of
 * FOCUS_ERR_TIMEOUT (a kernel wait gave up), FOCUS_ERR_DEVICE_CHECK,
 * FOCUS_ERR_CAPACITY that is set.  Returns FOCUS_ERR_TIMEOUT without reading
 * when the stream has not finished in time.  This is the only call that
 * synchronises.
 */
FOCUS_API focus_status_t focus_read_device_status(const void *workspace, void *stream, int timeout_ms);

/*
 * Attention importance of ONE layer (method step "Delta Calculation", first half):
 *   I[r][j] = sum over query heads h and block queries i of
 *             softmax_i( softmax_scale * q[r,i,h,:] . key[:] )[prefix_len_r + j]
 * where the keys of request r are its prefix rows k_prefix[cu_prefix[r] ..
 * cu_prefix[r+1]-1, h/G, :] followed by its block rows k_block[r, 0..B-1, h/G, :].
 *
 *   q            [R, B, Hq, d]        bf16
 *   k_prefix     [total_prefix, Hkv, d] bf16 (may be NULL when total_prefix == 0)
 *   cu_prefix    [R + 1] int32        cu_prefix[0] = 0, non-decreasing, cu_prefix[R] <= total_prefix
 *   total_prefix rows of k_prefix
 *   k_block      [R, B, Hkv, d]       bf16
 *   importance   [R, B] float32       output
 * A malformed cu_prefix entry sets FOCUS_ERR_DEVICE_CHECK in the device status
 * and that request is computed with no prefix.
 */
FOCUS_API focus_status_t focus_attn_stats(const focus_dims_t *dims, const void *q, const void *k_prefix,
                                const int32_t *cu_prefix, int64_t total_prefix,
                                const void *k_block, float *importance, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Importance delta, smoothing and mask (method steps Eq. 3, MaxPool1D, mask):
 *   delta[r][j] = max_{|t-j| <= pool_window/2, 0 <= t < B} (i1[r][t] - i0[r][t])
 *   delta[r][j] = -inf where decoded[r][j] != 0
 *   i0, i1 [R, B] float32; decoded [R, B] uint8 (nonzero = decoded); delta [R, B] float32 out.
 * raw_delta (nullable) receives i1 - i0 before pooling.
 */
FOCUS_API focus_status_t focus_importance_delta(const focus_dims_t *dims, const float *i0, const float *i1,
                                      const uint8_t *decoded, float *delta, float *raw_delta,
                                      void *stream);

/*
 * Top-K candidate selection (method step "Token Eviction", selection half):
 *   k_r = min(max(budget[r], 0), #{j : decoded[r][j] == 0})
 *   kept_idx[cu_seqlens[r] ..] = the k_r positions ranked first by
 *                                (delta desc, position asc), in ascending position order
 *                                (plus the structural constraints of dims.constraints)
 *   cu_seqlens[0] = 0, cu_seqlens[r+1] = cu_seqlens[r] + (rows kept for request r)
 *   delta [R, B] float32 (as produced by focus_importance_delta); budget [R] int32;
 *   kept_idx [capacity] int32 out; cu_seqlens [R + 1] int32 out.
 * Rows beyond `capacity` are not written and FOCUS_ERR_CAPACITY is set in the
 * device status (cu_seqlens is still complete).  A non-finite delta at a still-masked
 * position is out of contract and sets FOCUS_ERR_DEVICE_CHECK.
 */
FOCUS_API focus_status_t focus_topk_select(const focus_dims_t *dims, const float *delta,
                                 const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx,
                                 int32_t *cu_seqlens, int64_t capacity, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * Compaction (method step "Token Eviction", eviction half): bit copy
 *   packed[cu_seqlens[r] + t][:] = hidden[r][kept_idx[cu_seqlens[r] + t]][:]
 *   hidden [R, B, H] bf16; kept_idx, cu_seqlens as above; packed [capacity, H] bf16 out.
 * Rows at or beyond `capacity` are skipped (FOCUS_ERR_CAPACITY in the device
 * status); a kept index outside [0, B) skips its row (FOCUS_ERR_DEVICE_CHECK).
 */
FOCUS_API focus_status_t focus_compact(const focus_dims_t *dims, const void *hidden, const int32_t *kept_idx,
                             const int32_t *cu_seqlens, void *packed, int64_t capacity,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * The whole eviction step, fused, on one stream: layer-0 and layer-1
 * importance, delta, MaxPool1D, mask, top-K, compaction.  Arguments as in the
 * calls above; q0/k0_* are layer 0, q1/k1_* the layer-1 Q/K projections, both
 * layers share cu_prefix/total_prefix.  delta_out (pooled and masked), i0_out
 * and i1_out ([R, B] float32) are optional (NULL skips them).  With
 * dims.score == FOCUS_SCORE_LAYER1 the layer-0 arguments may be NULL, I0 is not
 * computed (i0_out is left untouched) and delta_out holds the pooled, masked I1.
 * Non-finite Q or K values are out of contract: they make the importance of their
 * request non-finite, which sets FOCUS_ERR_DEVICE_CHECK; every access stays in
 * bounds and the other requests are unaffected.
 */
FOCUS_API focus_status_t focus_evict(const focus_dims_t *dims, const void *q0, const void *k0_prefix,
                           const void *k0_block, const void *q1, const void *k1_prefix,
                           const void *k1_block, const int32_t *cu_prefix, int64_t total_prefix,
                           const void *hidden, const uint8_t *decoded, const int32_t *budget,
                           int32_t *kept_idx, int32_t *cu_seqlens, void *packed, int64_t capacity,
                           float *delta_out, float *i0_out, float *i1_out, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * Tracing hook: when `start_event` and `stop_event` (cudaEvent_t, passed as void*)
 * are non-NULL, every later focus_evict / focus_attn_stats call records
 * start_event on its stream right before its attention-statistics kernel and
 * stop_event right after it, so the caller can time that kernel alone with
 * cudaEventElapsedTime.  NULL, NULL turns the hook off.  The setting is
 * process-wide; set it from the thread that issues the calls.
 */
FOCUS_API void focus_set_trace_events(void *start_event, void *stop_event);

/*
 * All arguments of the fused step, for focus_evict_ex.  Optional features are
 * switched on by their pointers:
 *  - lse0 != NULL: layer 0's row log-sum-exps are given (see focus_evict_with_lse0);
 *    k0_prefix is then not read.
 *  - page_table != NULL: the prefix keys are in page pools (see focus_evict_paged);
 *    cu_prefix/total_prefix are then not used.
 *  - decode_avg != NULL: dynamic retention budget (below); `budget` is then not read.
 *
 * Dynamic budget.  Eq. 4 is not printed on the FOCUS pages; the Referee Report
 * summary says the budget comes "from historical decoding yield and within-block
 * delta statistics", the Free-Parameter Ledger gives the expansion factor
 * alpha = 1.5 of Eq. 4, and Figure 14 marks the "+Std" sigma threshold used for
 * it.  This library's reading, per request r, over its masked positions M_r and
 * the pooled, masked delta D:
 *   mu_r = mean D_j, sigma_r = population std of D_j (j in M_r),
 *   n_r  = #{j in M_r : D_j > mu_r + sigma_r},
 *   K_r  = min(max(ceil(budget_alpha * max(decode_avg[r], 0)), n_r, 1), |M_r|)  (0 if M_r is empty)
 * decode_avg [R] float32 is the request's historical mean number of tokens
 * decoded per step.  budget_out [R] int32 (nullable) receives K_r.  The retained
 * counts then depend on the data: `capacity` must be an upper bound (the number
 * of masked positions, or min(B, 2 x masked) with structural constraints) and
 * cu_seqlens is computed on the device.
 */
typedef struct {
    const void *q0, *k0_prefix, *k0_block;  /* layer 0 */
    const float *lse0;                      /* optional [R, B, Hq] */
    const void *q1, *k1_prefix, *k1_block;  /* layer 1 */
    const int32_t *cu_prefix;               /* packed prefix layout */
    int64_t total_prefix;
    const int32_t *page_table;              /* paged prefix layout (optional) */
    const int32_t *prefix_len;
    int32_t max_pages, num_pages, page_size;
    const void *hidden;                     /* [R, B, H] bf16 */
    const uint8_t *decoded;                 /* [R, B] */
    const int32_t *budget;                  /* [R]; unused with decode_avg */
    const float *decode_avg;                /* optional [R]: dynamic budget */
    float budget_alpha;                     /* Eq. 4 expansion factor (1.5) */
    int32_t *budget_out;                    /* optional [R] */
    int32_t *kept_idx;                      /* outputs */
    int32_t *cu_seqlens;
    void *packed;
    int64_t capacity;
    float *delta_out, *i0_out, *i1_out;     /* optional [R, B] */
    void *workspace;
    size_t workspace_bytes;
    void *stream;
} focus_evict_args_t;

/* The fused step with every option (focus_evict and its variants call this). */
FOCUS_API focus_status_t focus_evict_ex(const focus_dims_t *dims, const focus_evict_args_t *args);

/*
 * The fused step with the prefix keys in a paged KV cache (pages of page_size
 * tokens, each request owning an ordered list of pages, the same list for both
 * layers), read in place:
 *   k0_pages, k1_pages [num_pages, page_size, Hkv, d] bf16 (16-byte aligned)
 *   page_table [R, max_pages] int32: request r's prefix key t is row
 *              t % page_size of page page_table[r][t / page_size]
 *   prefix_len [R] int32: prefix length of each request (0 <= L_r <= max_pages * page_size)
 *   page_size: a power of two, 8 .. 65536.  Pages shorter than 128 tokens are
 *              gathered several per 128-key tile.
 * Everything else is focus_evict's.  A page index outside [0, num_pages) sets
 * FOCUS_ERR_DEVICE_CHECK in the device status (page 0 is read instead).
 */
FOCUS_API focus_status_t focus_evict_paged(
    const focus_dims_t *dims, const void *q0, const void *k0_pages, const void *k0_block,
    const void *q1, const void *k1_pages, const void *k1_block, const int32_t *page_table,
    int32_t max_pages, const int32_t *prefix_len, int32_t num_pages, int32_t page_size,
    const void *hidden, const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx,
    int32_t *cu_seqlens, void *packed, int64_t capacity, float *delta_out, float *i0_out,
    float *i1_out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The fused step when the engine already ran layer 0's attention (as FOCUS does:
 * layer 0 runs on the whole block) and kept its row log-sum-exps:
 *   lse0 [R, B, Hq] float32, lse0[r][i][h] = ln sum_j exp(softmax_scale * q0[r,i,h,:] . k0_j)
 *        over request r's prefix keys and its B block keys (what an attention
 *        forward returns alongside its output).
 * I0[r][j] = sum over h, i of exp(softmax_scale * q0[r,i,h,:] . k0_block[r,j,h/G,:] - lse0[r][i][h]),
 * so layer 0 reads only Q0 and its block keys: no layer-0 prefix K argument.
 * Everything else is focus_evict's (layer 1 is computed in full).  dims.score
 * must be FOCUS_SCORE_DELTA.
 */
FOCUS_API focus_status_t focus_evict_with_lse0(
    const focus_dims_t *dims, const float *lse0, const void *q0, const void *k0_block,
    const void *q1, const void *k1_prefix, const void *k1_block, const int32_t *cu_prefix,
    int64_t total_prefix, const void *hidden, const uint8_t *decoded, const int32_t *budget,
    int32_t *kept_idx, int32_t *cu_seqlens, void *packed, int64_t capacity, float *delta_out,
    float *i0_out, float *i1_out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The two halves of the fused step, for tensor-parallel engines whose ranks each
 * hold a slice of the heads.  I_j is a sum over query heads ("What carries the
 * argument"), so each rank computes the importance of its own heads with
 * focus_partial_importance, the ranks sum the [2, R, B] results (one all-reduce),
 * and every rank runs focus_evict_from_importance on the same sums, so all ranks
 * keep the same tokens.  (The pages run on one GPU; this split is a deployment
 * variant of focus_evict.)
 *
 * focus_partial_importance: both layers' importance over the heads in `dims`
 * (dims.Hq / dims.Hkv = this rank's head counts, the same G = Hq/Hkv as the
 * model), with the layouts of focus_evict restricted to those heads:
 *   importance [2, R, B] float32 out: importance[0] = I0, importance[1] = I1.
 * With dims.score == FOCUS_SCORE_LAYER1 the layer-0 arguments may be NULL and
 * importance[0] is left untouched.  dims.hidden is not used (any multiple of 8).
 * The per-(request, kv head, row tile) column sums are reduced in a fixed
 * order, so the result is deterministic and equals what focus_attn_stats gives
 * for each layer.
 */
FOCUS_API focus_status_t focus_partial_importance(
    const focus_dims_t *dims, const void *q0, const void *k0_prefix, const void *k0_block,
    const void *q1, const void *k1_prefix, const void *k1_block, const int32_t *cu_prefix,
    int64_t total_prefix, float *importance, void *workspace, size_t workspace_bytes,
    void *stream);

/*
 * focus_evict_from_importance: delta (I1 - I0, or I1 alone with
 * dims.score == FOCUS_SCORE_LAYER1), MaxPool1D, mask, top-K (with
 * dims.constraints applied) and compaction from a given importance
 * [2, R, B] float32 (importance[0] is not read for the layer-1 score).
 * Outputs and their rules as in focus_evict; delta_out (nullable) receives the
 * pooled, masked delta.  Given the importance focus_partial_importance computes
 * over all heads, the outputs are bit-identical to focus_evict's.
 */
FOCUS_API focus_status_t focus_evict_from_importance(
    const focus_dims_t *dims, const float *importance, const void *hidden,
    const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx, int32_t *cu_seqlens,
    void *packed, int64_t capacity, float *delta_out, void *workspace, size_t workspace_bytes,
    void *stream);

/*
 * Peer exchange of the partial importance: the head-sharded step without a
 * separate all-reduce.  Each rank exposes one exchange buffer of
 * focus_exchange_buffer_size(dims, world) bytes to its peers (device memory that
 * every rank can address: CUDA IPC or symmetric-memory mappings over NVLink).
 * focus_partial_importance_push computes the rank's [2, R, B] sums like
 * focus_partial_importance and stores them, from the reducing kernel itself,
 * into slot `rank` of every rank's buffer, then raises the rank's flag there;
 * focus_evict_from_exchange waits for every rank's flag in the local buffer,
 * sums the slots in rank order (so every rank holds bit-identical sums) and
 * selects and compacts as focus_evict_from_importance.  (The pages run on one
 * GPU; this is a deployment variant.)
 *
 * Protocol, per rank and step: push(epoch), then evict_from_exchange(epoch), on
 * one stream, with epoch = 1, 2, 3, ... the same on every rank.  Zero every
 * buffer once (all bytes) and synchronise the ranks on the host before the
 * first push.  Two slot parities make it safe for a rank to run one step ahead.
 * A flag that does not arrive within 2 s sets FOCUS_ERR_TIMEOUT in the device
 * status (read with focus_read_device_status); the sums are then not valid.
 * The workspace must not be shared with another stream while a push runs.  The
 * push counts its finished blocks in the workspace's status region;
 * focus_clear_device_status resets that count too, so after an error clear the
 * status of every rank's workspaces, zero the buffers and restart at epoch 1.
 */
typedef struct {
    void *const *peer_buffers; /* DEVICE array [world] of device pointers: rank q's exchange
                                  buffer as this process addresses it (entry `rank` = own) */
    int32_t rank;              /* 0 <= rank < world */
    int32_t world;             /* 1 <= world <= 8 */
    uint32_t epoch;            /* >= 1 */
} focus_exchange_t;

/* Bytes of one rank's exchange buffer for dims.R, dims.B (0 for invalid dims or world). */
FOCUS_API size_t focus_exchange_buffer_size(const focus_dims_t *dims, int32_t world);

/* focus_partial_importance whose sums go to the peers' exchange buffers. */
FOCUS_API focus_status_t focus_partial_importance_push(
    const focus_dims_t *dims, const void *q0, const void *k0_prefix, const void *k0_block,
    const void *q1, const void *k1_prefix, const void *k1_block, const int32_t *cu_prefix,
    int64_t total_prefix, const focus_exchange_t *exchange, void *workspace,
    size_t workspace_bytes, void *stream);

/* focus_evict_from_importance on the sum over ranks of the exchange buffer's
 * slots of `epoch` (exchange_buffer: this rank's own buffer, 256-byte aligned). */
FOCUS_API focus_status_t focus_evict_from_exchange(
    const focus_dims_t *dims, const void *exchange_buffer, int32_t world, uint32_t epoch,
    const void *hidden, const uint8_t *decoded, const int32_t *budget, int32_t *kept_idx,
    int32_t *cu_seqlens, void *packed, int64_t capacity, float *delta_out, void *workspace,
    size_t workspace_bytes, void *stream);

/*
 * Self-test of the exchange protocol with `world` emulated ranks on ONE GPU, in one
 * cooperative launch (all blocks resident, so blocks may wait on one another):
 * block group q pushes partials[q] ([world][2][R][B] float32) into every buffer
 * with the device routines the push uses, raises its flags, waits for all flags
 * of its own buffer as the selection does, and writes the rank-ordered sum of
 * its slots to out[q] ([world][2][R][B]).  buffers: DEVICE array [world] of
 * exchange buffers (zeroed); scratch: DEVICE, >= 1 + world uint32, zeroed;
 * scratch[0] receives the device status bits.  R * 2 * world <= 1024.
 * (No counterpart on the pages: a test of this library.)
 */
FOCUS_API focus_status_t focus_selftest_exchange(const float *partials, void *const *buffers,
                                                 float *out, uint32_t *scratch, int32_t R,
                                                 int32_t B, int32_t world, uint32_t epoch,
                                                 void *stream);

/*
 * The fused step for callers that cannot allocate device memory.  (The FOCUS
 * pages have no counterpart: this is a deployment variant of focus_evict.)
 *
 * focus_evict needs a caller-allocated workspace.  A caller that cannot make
 * allocations -- e.g. a serving engine that has reserved nearly all HBM for its
 * KV cache and must not request more while it decodes, or a plug-in that only
 * sees this C ABI and has no access to its host framework's memory pool -- can
 * call this instead: the scratch lives in a device array of
 * FOCUS_STATIC_SCRATCH_BYTES (8 MiB) that the library owns, and that every GPU
 * which loads the library keeps until the process exits.  The call allocates
 * nothing (no cudaMalloc/cudaFree, no allocating library routine); the caller
 * still passes every input and output, as for focus_evict.
 *
 *  - Arguments and results are those of focus_evict, minus the workspace.
 *  - device_status (nullable, device pointer, 4-byte aligned) receives the
 *    call's raw device status bits: 1 = rows beyond `capacity`, 2 = malformed
 *    cu_prefix, page or kept index, or non-finite inputs, 4 = a kernel wait
 *    gave up; 0 = fine.  It is written on `stream` after the kernels.
 *  - Returns FOCUS_ERR_WORKSPACE when focus_workspace_size(dims) exceeds
 *    FOCUS_STATIC_SCRATCH_BYTES (shapes that large need focus_evict), otherwise
 *    the same codes as focus_evict.  The largest batch is set by the workspace
 *    formula: 256 B + the request order (4 R) + the column sums (8 R Hkv MT B,
 *    MT = ceil(Hq B / (128 Hkv))) + the retained lists (4 R B) + the counts (4 R),
 *    each rounded up to 256 B, plus the split-prefix regions of batches with at
 *    most 148 attention item groups: 3,840 requests at Hq 32 / Hkv 8 / B 32,
 *    251 at B 128, 991 at Hkv 4 / B 64.
 *  - Every argument is checked before anything is enqueued, so a refused call
 *    leaves the array (and a status word another call is about to report)
 *    untouched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current; `stream` must belong to
 *    the current device) and keeps it for the life of the process.  A cudaDeviceReset (or anything else
 *    that destroys and recreates the device's primary context) may move the
 *    array: do not use this entry point on a device after such a reset.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents: each call clears the status word and rewrites the rest before
 *    reading it.  Calls whose kernels overlap on the GPU (different streams, or
 *    threads without ordering) race on the array; serialise them.
 */
#define FOCUS_STATIC_SCRATCH_BYTES (8u << 20)
FOCUS_API focus_status_t focus_evict_static_scratch(
    const focus_dims_t *dims, const void *q0, const void *k0_prefix, const void *k0_block,
    const void *q1, const void *k1_prefix, const void *k1_block, const int32_t *cu_prefix,
    int64_t total_prefix, const void *hidden, const uint8_t *decoded, const int32_t *budget,
    int32_t *kept_idx, int32_t *cu_seqlens, void *packed, int64_t capacity, float *delta_out,
    float *i0_out, float *i1_out, uint32_t *device_status, void *stream);

/*
 * Self-test of the failure-detection path (no FOCUS counterpart; a test hook).
 * Launches one warp that waits, with the same bounded mbarrier wait the eviction
 * kernels use, on a barrier that never completes.  After `limit_ns`
 * (1 .. 2e9 nanoseconds) the wait gives up: FOCUS_DEV_TIMEOUT (4) is OR-ed into
 * the device word *status, and *elapsed_ns (device) receives how long it waited.
 * Nothing faults, traps or hangs; the context stays usable.
 */
FOCUS_API focus_status_t focus_selftest_wait_timeout(uint32_t *status, uint64_t limit_ns,
                                                     unsigned long long *elapsed_ns,
                                                     void *stream);

/* Human-readable name of a status code (static string). */
FOCUS_API const char *focus_status_string(focus_status_t status);

/* FOCUS_ABI_VERSION of the loaded library. */
FOCUS_API int focus_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FOCUS_H_ */
