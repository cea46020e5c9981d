/*
 * focus_oracle.c -- float64 CPU oracle for FOCUS importance-delta token eviction.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker that the
 * CUDA path is compared against.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library, and the library never calls it.
 *
 * Source of the method: "FOCUS: DLLMs Know How to Tame Their Compute Bound"
 * (pith.science review page), section "What carries the argument": the
 * importance of block token j is the column sum of the softmax attention
 * weights it receives from all query tokens of the block; the importance delta
 * is the layer-1 importance minus the layer-0 importance, smoothed by MaxPool1D;
 * the top-K candidates under a budget are kept.  The same page's Figure 5
 * caption places the eviction after the layer-1 Q/K projections, its Referee
 * Report (minor comment on Eq. (2)) reads the softmax as row (query) wise, and
 * its Free-Parameter Ledger fixes the MaxPool1D kernel size at k = 3 (Eq. 15).
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes):
 *   - the softmax of query row i runs over the request's prefix keys followed
 *     by all B block keys, with no causal mask inside the block;
 *   - every one of the B block queries contributes, decoded or not;
 *   - I_j sums over all query heads; query head h reads kv head h / (Hq/Hkv);
 *   - logits are softmax_scale * q.k on the given (post-RoPE) Q and K;
 *   - MaxPool1D smooths the delta (not I), stride 1, same padding, padded
 *     positions ignored (-inf padding);
 *   - decoded positions get -inf after pooling and are never selected;
 *   - k_r = min(max(K_r, 0), number of masked positions);
 *   - ties in the pooled delta go to the lower position; the kept positions
 *     are written in ascending order; requests are packed in order.
 *
 * Arithmetic is float64 throughout.  bf16 inputs are widened exactly.  Each
 * function is a direct transcription of its definition: no blocking, fusion or
 * reordering beyond what the definition states.  OpenMP (when compiled with
 * -fopenmp) only splits the outer loop over independent (request, kv head)
 * pairs; their contributions to I are added afterwards in kv-head order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARGUMENT 1
#define ORACLE_NO_MEMORY 2
#define ORACLE_CAPACITY 3

/* Exact widening of a bf16 bit pattern (upper half of an IEEE binary32). */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int focus_oracle_num_threads(void)
{
#ifdef _OPENMP
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
#else
    return 1;
#endif
}

/* Threads the following calls use (n >= 1); returns the count now in effect.  Only
 * the timing of the CPU baseline changes it (single-thread and all-core runs). */
int focus_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
    return focus_oracle_num_threads();
}

/*
 * Attention importance of one layer (the "column-wise sum of softmax attention
 * weights received by token j from all query tokens in the block").
 *
 *   q        [R, B, Hq, d]      bf16 bits, the block's queries
 *   k_prefix [sum L_r, Hkv, d]  bf16 bits, request r owns rows cu_prefix[r] .. cu_prefix[r+1]-1
 *   k_block  [R, B, Hkv, d]     bf16 bits, the block's keys
 *   out      [R, B]             float64, I[r][j] for block column j
 *
 * For each request r, query head h, block query i:
 *   s_j = scale * sum_c q[r,i,h,c] * key_j[c]   over keys j = prefix 0..L-1, then block 0..B-1
 *   m   = max_j s_j ;  Z = sum_j exp(s_j - m)
 *   out[r][j] += exp(s_{L+j} - m) / Z            for block columns j = 0..B-1
 */
int focus_oracle_importance(int R, int B, int Hq, int Hkv, int d, double scale,
                            const uint16_t *q, const uint16_t *k_prefix,
                            const int32_t *cu_prefix, const uint16_t *k_block,
                            double *out)
{
    if (R < 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0)
        return ORACLE_BAD_ARGUMENT;
    if (R == 0)
        return ORACLE_OK;
    for (int r = 0; r < R; ++r)
        if (cu_prefix[r + 1] < cu_prefix[r])
            return ORACLE_BAD_ARGUMENT;
    const int G = Hq / Hkv;
    /* part[r][g][j]: the contribution of the G query heads that read kv head g. */
    double *part = (double *)calloc((size_t)R * Hkv * B, sizeof(double));
    if (!part)
        return ORACLE_NO_MEMORY;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long long task = 0; task < (long long)R * Hkv; ++task) {
        const int r = (int)(task / Hkv);
        const int g = (int)(task % Hkv);
        const int L = cu_prefix[r + 1] - cu_prefix[r];
        const int N = L + B;
        double *acc = part + ((size_t)r * Hkv + g) * B;
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        double *keys = (double *)malloc(sizeof(double) * (size_t)N * (size_t)d);
        if (!s || !qrow || !keys) {
            free(s); free(qrow); free(keys);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* Key list of kv head g: prefix keys, then block keys. */
        for (int j = 0; j < N; ++j) {
            const uint16_t *src;
            if (j < L)
                src = k_prefix + (((size_t)cu_prefix[r] + j) * Hkv + g) * d;
            else
                src = k_block + (((size_t)r * B + (j - L)) * Hkv + g) * d;
            for (int c = 0; c < d; ++c)
                keys[(size_t)j * d + c] = bf16_bits_to_double(src[c]);
        }
        for (int h = g * G; h < (g + 1) * G; ++h) {
            for (int i = 0; i < B; ++i) {
                const uint16_t *qs = q + (((size_t)r * B + i) * Hq + h) * d;
                for (int c = 0; c < d; ++c)
                    qrow[c] = bf16_bits_to_double(qs[c]);
                double m = -INFINITY;
                for (int j = 0; j < N; ++j) {
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c)
                        dot += qrow[c] * keys[(size_t)j * d + c];
                    s[j] = scale * dot;
                    if (s[j] > m)
                        m = s[j];
                }
                double Z = 0.0;
                for (int j = 0; j < N; ++j)
                    Z += exp(s[j] - m);
                for (int j = 0; j < B; ++j)
                    acc[j] += exp(s[L + j] - m) / Z;
            }
        }
        free(s);
        free(qrow);
        free(keys);
    }
    /* I[r][j] = sum over kv heads g (in order) of the group contributions. */
    for (int r = 0; r < R; ++r)
        for (int j = 0; j < B; ++j) {
            double sum = 0.0;
            for (int g = 0; g < Hkv; ++g)
                sum += part[((size_t)r * Hkv + g) * B + j];
            out[(size_t)r * B + j] = sum;
        }
    free(part);
    return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/*
 * Attention importance with the prefix keys in a paged pool (a KV cache laid out
 * as pages of page_size tokens, each request owning an ordered list of pages):
 *
 *   prefix key t of request r = k_pages[page_table[r][t / page_size]][t % page_size][g][:]
 *   k_pages    [num_pages, page_size, Hkv, d] bf16 bits
 *   page_table [R, max_pages] int32;  prefix_len [R] int32
 *
 * Otherwise exactly focus_oracle_importance (prefix keys, then block keys).
 */
int focus_oracle_importance_paged(int R, int B, int Hq, int Hkv, int d, double scale,
                                  const uint16_t *q, const uint16_t *k_pages,
                                  const int32_t *page_table, int max_pages,
                                  const int32_t *prefix_len, int page_size, int num_pages,
                                  const uint16_t *k_block, double *out)
{
    if (R < 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || page_size <= 0)
        return ORACLE_BAD_ARGUMENT;
    for (int r = 0; r < R; ++r) {
        if (prefix_len[r] < 0 || (prefix_len[r] + page_size - 1) / page_size > max_pages)
            return ORACLE_BAD_ARGUMENT;
        for (int t = 0; t < (prefix_len[r] + page_size - 1) / page_size; ++t) {
            const int pg = page_table[(size_t)r * max_pages + t];
            if (pg < 0 || pg >= num_pages)
                return ORACLE_BAD_ARGUMENT;
        }
    }
    const int G = Hq / Hkv;
    double *part = (double *)calloc((size_t)R * Hkv * B, sizeof(double));
    if (!part)
        return ORACLE_NO_MEMORY;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long long task = 0; task < (long long)R * Hkv; ++task) {
        const int r = (int)(task / Hkv);
        const int g = (int)(task % Hkv);
        const int L = prefix_len[r];
        const int N = L + B;
        double *acc = part + ((size_t)r * Hkv + g) * B;
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        double *keys = (double *)malloc(sizeof(double) * (size_t)N * (size_t)d);
        if (!s || !qrow || !keys) {
            free(s); free(qrow); free(keys);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        for (int j = 0; j < N; ++j) {
            const uint16_t *src;
            if (j < L) {
                const size_t page = (size_t)page_table[(size_t)r * max_pages + j / page_size];
                src = k_pages + ((page * page_size + (size_t)(j % page_size)) * Hkv + g) * d;
            } else {
                src = k_block + (((size_t)r * B + (j - L)) * Hkv + g) * d;
            }
            for (int c = 0; c < d; ++c)
                keys[(size_t)j * d + c] = bf16_bits_to_double(src[c]);
        }
        for (int h = g * G; h < (g + 1) * G; ++h) {
            for (int i = 0; i < B; ++i) {
                const uint16_t *qs = q + ((((size_t)r * B) + i) * Hq + h) * d;
                for (int c = 0; c < d; ++c)
                    qrow[c] = bf16_bits_to_double(qs[c]);
                double m = -INFINITY;
                for (int j = 0; j < N; ++j) {
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c)
                        dot += qrow[c] * keys[(size_t)j * d + c];
                    s[j] = scale * dot;
                    if (s[j] > m)
                        m = s[j];
                }
                double Z = 0.0;
                for (int j = 0; j < N; ++j)
                    Z += exp(s[j] - m);
                for (int j = 0; j < B; ++j)
                    acc[j] += exp(s[L + j] - m) / Z;
            }
        }
        free(s);
        free(qrow);
        free(keys);
    }
    for (int r = 0; r < R; ++r)
        for (int j = 0; j < B; ++j) {
            double sum = 0.0;
            for (int g = 0; g < Hkv; ++g)
                sum += part[((size_t)r * Hkv + g) * B + j];
            out[(size_t)r * B + j] = sum;
        }
    free(part);
    return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/*
 * Attention importance from a given row normaliser (the log-sum-exp an
 * attention forward already produced for the same rows):
 *
 *   out[r][j] = sum over h, i of exp(scale * q[r,i,h,:] . k_block[r,j,h/G,:] - lse[r][i][h])
 *
 *   lse [R, B, Hq] float64, lse[r][i][h] = ln sum_j exp(s_j) over the row's keys.
 * With the true log-sum-exp this equals focus_oracle_importance; only the B block
 * keys are read.
 */
int focus_oracle_importance_lse(int R, int B, int Hq, int Hkv, int d, double scale,
                                const uint16_t *q, const uint16_t *k_block, const double *lse,
                                double *out)
{
    if (R < 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0)
        return ORACLE_BAD_ARGUMENT;
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r) {
        for (int j = 0; j < B; ++j) {
            double acc = 0.0;
            for (int h = 0; h < Hq; ++h) {
                const int g = h / G;
                const uint16_t *kj = k_block + (((size_t)r * B + j) * Hkv + g) * d;
                for (int i = 0; i < B; ++i) {
                    const size_t row = ((size_t)r * B + i) * Hq + h;  /* query (r, i, h) */
                    const uint16_t *qi = q + row * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c)
                        dot += bf16_bits_to_double(qi[c]) * bf16_bits_to_double(kj[c]);
                    acc += exp(scale * dot - lse[row]);
                }
            }
            out[(size_t)r * B + j] = acc;
        }
    }
    return ORACLE_OK;
}

/*
 * Importance delta, MaxPool1D smoothing and decoded mask.
 *
 *   delta[r][j]  = i1[r][j] - i0[r][j]                          (Eq. 3)
 *   pooled[r][j] = max over j' in [j - w/2, j + w/2], 0 <= j' < B, of delta[r][j']
 *                  (window w odd, stride 1, same padding; padded cells ignored)
 *   pooled[r][j] = -inf where decoded[r][j] != 0
 *
 * delta_out may be NULL.
 */
int focus_oracle_delta(int R, int B, int window, const double *i0, const double *i1,
                       const uint8_t *decoded, double *delta_out, double *pooled)
{
    if (R < 0 || B <= 0 || window <= 0 || window % 2 == 0)
        return ORACLE_BAD_ARGUMENT;
    const int half = window / 2;
    double *delta = (double *)malloc(sizeof(double) * (size_t)B);
    if (!delta)
        return ORACLE_NO_MEMORY;
    for (int r = 0; r < R; ++r) {
        for (int j = 0; j < B; ++j) {
            delta[j] = i1[(size_t)r * B + j] - i0[(size_t)r * B + j];
            if (delta_out)
                delta_out[(size_t)r * B + j] = delta[j];
        }
        for (int j = 0; j < B; ++j) {
            double best = -INFINITY;
            for (int t = j - half; t <= j + half; ++t)
                if (t >= 0 && t < B && delta[t] > best)
                    best = delta[t];
            pooled[(size_t)r * B + j] = decoded[(size_t)r * B + j] ? -INFINITY : best;
        }
    }
    free(delta);
    return ORACLE_OK;
}

/* (a ranks before b) iff value greater, or value equal and position lower. */
static int ranks_before(double va, int a, double vb, int b)
{
    if (va > vb)
        return 1;
    if (va < vb)
        return 0;
    return a < b;
}

/*
 * Top-K candidate selection and packing offsets.
 *
 *   masked_r = number of j with decoded[r][j] == 0
 *   k_r      = min(max(budget[r], 0), masked_r)
 *   kept     = the k_r positions ranked first by (pooled desc, position asc),
 *              written in ascending position order at kept[cu[r] .. cu[r+1]-1]
 *   cu[0] = 0, cu[r+1] = cu[r] + k_r
 *
 * Returns ORACLE_CAPACITY (after writing cu_seqlens in full and as many kept
 * positions as fit) when sum k_r exceeds capacity.
 */
int focus_oracle_select(int R, int B, const double *pooled, const uint8_t *decoded,
                        const int32_t *budget, int32_t *kept, int32_t *cu_seqlens,
                        int64_t capacity)
{
    if (R < 0 || B <= 0 || capacity < 0)
        return ORACLE_BAD_ARGUMENT;
    int *order = (int *)malloc(sizeof(int) * (size_t)B);
    int *chosen = (int *)malloc(sizeof(int) * (size_t)B);
    if (!order || !chosen) {
        free(order); free(chosen);
        return ORACLE_NO_MEMORY;
    }
    int status = ORACLE_OK;
    cu_seqlens[0] = 0;
    for (int r = 0; r < R; ++r) {
        const double *v = pooled + (size_t)r * B;
        int masked = 0;
        for (int j = 0; j < B; ++j)
            masked += decoded[(size_t)r * B + j] == 0;
        int k = budget[r] < 0 ? 0 : budget[r];
        if (k > masked)
            k = masked;

        /* Insertion sort of positions by rank; stable by construction. */
        for (int j = 0; j < B; ++j) {
            int t = j;
            while (t > 0 && ranks_before(v[j], j, v[order[t - 1]], order[t - 1])) {
                order[t] = order[t - 1];
                --t;
            }
            order[t] = j;
        }
        /* The first k ranked positions, re-sorted into ascending position. */
        for (int t = 0; t < k; ++t)
            chosen[t] = order[t];
        for (int a = 1; a < k; ++a) {
            int x = chosen[a], t = a;
            while (t > 0 && chosen[t - 1] > x) {
                chosen[t] = chosen[t - 1];
                --t;
            }
            chosen[t] = x;
        }
        const int64_t base = cu_seqlens[r];
        for (int t = 0; t < k; ++t) {
            if (base + t < capacity)
                kept[base + t] = chosen[t];
            else
                status = ORACLE_CAPACITY;
        }
        cu_seqlens[r + 1] = (int32_t)(base + k);
    }
    free(order);
    free(chosen);
    return status;
}

/*
 * Structural constraints on the retained set ("What carries the argument": after
 * the top-K candidates are chosen, each candidate's immediate predecessor and all
 * masked tokens before the rightmost candidate are retained as well).
 *
 *   S_r        = the top-k_r candidates of request r (focus_oracle_select's rule)
 *   retained_r = S_r
 *              U {j - 1 : j in S_r, j >= 1}                     (constraints & 1)
 *              U {j : j < max S_r, decoded[r][j] == 0}          (constraints & 2)
 *   written in ascending position order; cu[r+1] = cu[r] + |retained_r|.
 *
 * A predecessor is retained whether it is masked or decoded; the second rule adds
 * masked positions only.  Returns ORACLE_CAPACITY (cu complete) past capacity.
 */
int focus_oracle_select_structured(int R, int B, const double *pooled, const uint8_t *decoded,
                                   const int32_t *budget, int constraints, int32_t *kept,
                                   int32_t *cu_seqlens, int64_t capacity)
{
    if (R < 0 || B <= 0 || capacity < 0 || constraints < 0 || constraints > 3)
        return ORACLE_BAD_ARGUMENT;
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    int32_t cand_cu[2];
    unsigned char *keep = (unsigned char *)malloc((size_t)B);
    if (!cand || !keep) {
        free(cand); free(keep);
        return ORACLE_NO_MEMORY;
    }
    int status = ORACLE_OK;
    cu_seqlens[0] = 0;
    for (int r = 0; r < R; ++r) {
        /* The candidates: the plain top-k selection of this one request. */
        int st = focus_oracle_select(1, B, pooled + (size_t)r * B, decoded + (size_t)r * B,
                                     budget + r, cand, cand_cu, B);
        if (st != ORACLE_OK) {
            free(cand); free(keep);
            return st;
        }
        const int k = cand_cu[1];
        for (int j = 0; j < B; ++j)
            keep[j] = 0;
        int rightmost = -1;
        for (int t = 0; t < k; ++t) {
            keep[cand[t]] = 1;
            if (cand[t] > rightmost)
                rightmost = cand[t];
        }
        if (constraints & 1)
            for (int t = 0; t < k; ++t)
                if (cand[t] >= 1)
                    keep[cand[t] - 1] = 1;
        if (constraints & 2)
            for (int j = 0; j < rightmost; ++j)
                if (decoded[(size_t)r * B + j] == 0)
                    keep[j] = 1;
        int64_t row = cu_seqlens[r];
        for (int j = 0; j < B; ++j) {
            if (!keep[j])
                continue;
            if (row < capacity)
                kept[row] = j;
            else
                status = ORACLE_CAPACITY;
            ++row;
        }
        cu_seqlens[r + 1] = (int32_t)row;
    }
    free(cand);
    free(keep);
    return status;
}

/*
 * Dynamic retention budget (a reading of Eq. 4, which the pages do not print:
 * "Dynamic Budgeting" sets K from the request's historical decoding yield scaled
 * by the expansion factor alpha (default 1.5, Free-Parameter Ledger) and from the
 * within-block delta statistics -- the "+Std" sigma threshold of Figure 14):
 *
 *   over the masked positions M_r of block r (D = pooled, masked delta):
 *     mu_r = mean_{j in M_r} D_j,  sigma_r = sqrt(mean_{j in M_r} (D_j - mu_r)^2)
 *     n_r  = #{j in M_r : D_j > mu_r + sigma_r}
 *   K_r = min(max(ceil(alpha * decode_avg[r]), n_r, 1), |M_r|);  K_r = 0 when M_r is empty.
 */
int focus_oracle_dynamic_budget(int R, int B, const double *pooled, const uint8_t *decoded,
                                const double *decode_avg, double alpha, int32_t *budget_out)
{
    if (R < 0 || B <= 0 || !(alpha >= 0.0))
        return ORACLE_BAD_ARGUMENT;
    for (int r = 0; r < R; ++r) {
        const double *D = pooled + (size_t)r * B;
        const uint8_t *dec = decoded + (size_t)r * B;
        int m = 0;
        double sum = 0.0;
        for (int j = 0; j < B; ++j)
            if (!dec[j]) {
                ++m;
                sum += D[j];
            }
        if (m == 0) {
            budget_out[r] = 0;
            continue;
        }
        const double mu = sum / m;
        double ss = 0.0;
        for (int j = 0; j < B; ++j)
            if (!dec[j])
                ss += (D[j] - mu) * (D[j] - mu);
        const double sigma = sqrt(ss / m);
        int n = 0;
        for (int j = 0; j < B; ++j)
            if (!dec[j] && D[j] > mu + sigma)
                ++n;
        double want = ceil(alpha * (decode_avg[r] > 0.0 ? decode_avg[r] : 0.0));
        if (want < n)
            want = n;
        if (want < 1)
            want = 1;
        if (want > m)
            want = m;
        budget_out[r] = (int32_t)want;
    }
    return ORACLE_OK;
}

/*
 * Compaction of the retained tokens' hidden rows into a packed varlen batch:
 *   packed[cu[r] + t][:] = hidden[r][kept[cu[r] + t]][:]   (bit copy)
 */
int focus_oracle_compact(int R, int B, int H, const uint16_t *hidden, const int32_t *kept,
                         const int32_t *cu_seqlens, uint16_t *packed, int64_t capacity)
{
    if (R < 0 || B <= 0 || H <= 0)
        return ORACLE_BAD_ARGUMENT;
    for (int r = 0; r < R; ++r) {
        for (int64_t row = cu_seqlens[r]; row < cu_seqlens[r + 1]; ++row) {
            if (row >= capacity)
                return ORACLE_CAPACITY;
            const int j = kept[row];
            if (j < 0 || j >= B)
                return ORACLE_BAD_ARGUMENT;
            memcpy(packed + (size_t)row * H, hidden + ((size_t)r * B + j) * H,
                   sizeof(uint16_t) * (size_t)H);
        }
    }
    return ORACLE_OK;
}

/*
 * The whole eviction step in the order the method states it: layer-0
 * importance, layer-1 importance (from the layer-1 Q/K projections), delta,
 * MaxPool1D, decoded mask, top-K, compaction.  i0/i1/pooled are outputs of
 * size R*B; delta_out may be NULL.
 */
int focus_oracle_evict(int R, int B, int Hq, int Hkv, int d, int H, double scale, int window,
                       const uint16_t *q0, const uint16_t *k0_prefix, const uint16_t *k0_block,
                       const uint16_t *q1, const uint16_t *k1_prefix, const uint16_t *k1_block,
                       const int32_t *cu_prefix, const uint16_t *hidden, const uint8_t *decoded,
                       const int32_t *budget, int32_t *kept, int32_t *cu_seqlens,
                       uint16_t *packed, int64_t capacity, double *i0, double *i1,
                       double *delta_out, double *pooled)
{
    int st = focus_oracle_importance(R, B, Hq, Hkv, d, scale, q0, k0_prefix, cu_prefix, k0_block, i0);
    if (st != ORACLE_OK)
        return st;
    st = focus_oracle_importance(R, B, Hq, Hkv, d, scale, q1, k1_prefix, cu_prefix, k1_block, i1);
    if (st != ORACLE_OK)
        return st;
    st = focus_oracle_delta(R, B, window, i0, i1, decoded, delta_out, pooled);
    if (st != ORACLE_OK)
        return st;
    st = focus_oracle_select(R, B, pooled, decoded, budget, kept, cu_seqlens, capacity);
    if (st != ORACLE_OK)
        return st;
    return focus_oracle_compact(R, B, H, hidden, kept, cu_seqlens, packed, capacity);
}
