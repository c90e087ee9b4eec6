/*
 * attn_oracle.c -- plain, slow, fp64 CPU reference for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  The product
 * path (the CUDA library) neither links nor calls it, and it shares no code,
 * header, table or helper with the CUDA sources.
 *
 * What it computes is the textbook definition of attention, which fused
 * attention reproduces exactly up to rounding order:
 *   "FlashAttention" (ozercemkelahmet.com/tools/flashattention), section
 *   "What it is": the three steps -- scores Q.K^T, softmax of each row, and the
 *   weighted sum of values -- written out one after the other, and section
 *   "Checking correctness": scores scaled by d^-1/2 in higher precision, future
 *   keys masked to -inf, softmax, then multiply by V.
 *
 * For every query row i of one sequence, query head h (key/value head g):
 *   s_j   = scale * sum_t q[i,h,t] * k[j,g,t]        for each visible key j
 *   M     = max_j s_j
 *   Z     = sum_j exp(s_j - M)
 *   P_ij  = exp(s_j - M) / Z
 *   O[i,h,:] = sum_j P_ij * v[j,g,:]
 *   LSE   = M + ln Z          (the "log of the softmax normalizer" kept for the
 *                              backward pass: same page, How it works, Step 5)
 * The score row is materialised in fp64 (one row at a time, never N x N).
 *
 * Masks ("Flash Attention" skill page (skillmd.com), Workflow 2, the
 * window_size=(left, right) argument, -1 meaning no limit; the explainer page,
 * How it works, Step 6, causal = each position sees itself and earlier ones):
 *   key j is visible to query i of the same sequence iff
 *       (left  < 0 || j >= i - left) && (right < 0 || j <= i + right)
 *   and causal forces right = 0.  Window bounds are inclusive.
 * Grouped-query attention (explainer page, Glossary and "Variants you may
 * meet"): query head h reads key/value head g = h / (Hq / Hkv), i.e. consecutive
 * query heads share one key/value head.
 * Packed variable-length batches ("Flash Attention 2 in HuggingFace"
 * (cloudcodetree.com), section "Stack it with sequence packing"): cu_seqlens
 * holds cumulative boundaries and attention never crosses them.
 * A row with no visible key (unreachable with valid arguments) is defined as
 * O = 0, LSE = -inf, the log of an empty sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_NOMEM (-2)

/* bf16 is the upper half of an IEEE binary32; widening to double is exact. */
static double widen_bf16(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int key_visible(int64_t i, int64_t j, int64_t left, int64_t right) {
    if (left >= 0 && j < i - left) return 0;
    if (right >= 0 && j > i + right) return 0;
    return 1;
}

/*
 * One query row.  q/k/v point at the start of the packed token arrays; the row
 * belongs to the sequence whose tokens are [start, start + L).
 */
static void attend_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t start, int64_t L, int64_t i, int h, int g,
                       int Hq, int Hkv, int d, double scale,
                       int64_t left, int64_t right, double *s_row,
                       double *o_row, double *lse_out, int64_t *nvis_out) {
    const uint16_t *qi = q + ((start + i) * (int64_t)Hq + h) * d;
    double M = -INFINITY;
    int64_t nvis = 0;

    /* Step 1: scaled scores of this row (masked keys get -inf). */
    for (int64_t j = 0; j < L; ++j) {
        if (!key_visible(i, j, left, right)) {
            s_row[j] = -INFINITY;
            continue;
        }
        const uint16_t *kj = k + ((start + j) * (int64_t)Hkv + g) * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += widen_bf16(qi[t]) * widen_bf16(kj[t]);
        s_row[j] = scale * dot;
        if (s_row[j] > M) M = s_row[j];
        ++nvis;
    }
    if (nvis_out) *nvis_out = nvis;
    if (nvis == 0) {
        for (int c = 0; c < d; ++c) o_row[c] = 0.0;
        *lse_out = -INFINITY;
        return;
    }

    /* Step 2: softmax normaliser of the row. */
    double Z = 0.0;
    for (int64_t j = 0; j < L; ++j)
        if (s_row[j] != -INFINITY) Z += exp(s_row[j] - M);

    /* Step 3: weights times values. */
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        if (s_row[j] == -INFINITY) continue;
        double p = exp(s_row[j] - M) / Z;
        const uint16_t *vj = v + ((start + j) * (int64_t)Hkv + g) * d;
        for (int c = 0; c < d; ++c) o_row[c] += p * widen_bf16(vj[c]);
    }
    *lse_out = M + log(Z);
}

/*
 * oracle_attn_fwd
 *   q  [tokens, Hq, d]  bf16 bits      (dense: tokens = B*N, batch-major)
 *   k,v[tokens, Hkv, d] bf16 bits
 *   cu_seqlens: NULL (dense, B sequences of length N) or int32[B+1]
 *               (packed; N is then the total token count).
 *   rows: NULL -> every row is computed and written in full layout:
 *           o   [tokens, Hq, d] fp64
 *           lse dense [B, Hq, N] / packed [Hq, tokens] fp64
 *           nvis same layout as lse (may be NULL)
 *         else nrows triples (sequence b, head h, row i within the sequence);
 *           outputs are compact: o[r*d + c], lse[r], nvis[r].
 *   nthreads <= 0 uses the OpenMP default.
 * Returns 0 or a negative error code.
 */
int oracle_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    double *o, double *lse, int64_t *nvis,
                    int B, int Hq, int Hkv, int N, int d, double scale,
                    int causal, int window_left, int window_right,
                    const int32_t *cu_seqlens, const int64_t *rows,
                    int64_t nrows, int nthreads) {
    if (!q || !k || !v || !o || !lse) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0) return ORACLE_ERR_ARG;
    if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window_left < -1 || window_right < -1) return ORACLE_ERR_ARG;
    const int group = Hq / Hkv;
    const int64_t left = window_left;
    const int64_t right = causal ? 0 : window_right;
    const int64_t tokens = cu_seqlens ? (int64_t)cu_seqlens[B] : (int64_t)B * N;
    int64_t maxL = 0;
    for (int b = 0; b < B; ++b) {
        int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
        if (L < 0) return ORACLE_ERR_ARG;
        if (L > maxL) maxL = L;
    }
#ifdef _OPENMP
    const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
#endif
    int failed = 0;

    if (rows == NULL) {
        /* every (sequence, head, row), in chunks of ROW_CHUNK rows */
        enum { ROW_CHUNK = 32 };
        const int64_t chunks_per_seq = (maxL + ROW_CHUNK - 1) / ROW_CHUNK;
        const int64_t units = (int64_t)B * Hq * chunks_per_seq;
#pragma omp parallel num_threads(nt)
        {
            double *s_row = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
            if (!s_row) {
#pragma omp atomic write
                failed = 1;
            }
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < units; ++u) {
                if (!s_row) continue;
                const int64_t chunk = u % chunks_per_seq;
                const int64_t bh = u / chunks_per_seq;
                const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / group;
                const int64_t start = cu_seqlens ? cu_seqlens[b] : (int64_t)b * N;
                const int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
                const int64_t i_end = (chunk + 1) * ROW_CHUNK < L ? (chunk + 1) * ROW_CHUNK : L;
                for (int64_t i = chunk * ROW_CHUNK; i < i_end; ++i) {
                    const int64_t lse_idx = cu_seqlens ? (int64_t)h * tokens + start + i
                                                       : ((int64_t)b * Hq + h) * N + i;
                    double *o_row = o + ((start + i) * Hq + h) * (int64_t)d;
                    attend_row(q, k, v, start, L, i, h, g, Hq, Hkv, d, scale, left, right,
                               s_row, o_row, &lse[lse_idx], nvis ? &nvis[lse_idx] : NULL);
                }
            }
            free(s_row);
        }
    } else {
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0) return ORACLE_ERR_ARG;
            const int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
            if (i >= L) return ORACLE_ERR_ARG;
        }
#pragma omp parallel num_threads(nt)
        {
            double *s_row = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
            if (!s_row) {
#pragma omp atomic write
                failed = 1;
            }
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r) {
                if (!s_row) continue;
                const int b = (int)rows[3 * r], h = (int)rows[3 * r + 1];
                const int64_t i = rows[3 * r + 2];
                const int64_t start = cu_seqlens ? cu_seqlens[b] : (int64_t)b * N;
                const int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
                attend_row(q, k, v, start, L, i, h, h / group, Hq, Hkv, d, scale, left, right,
                           s_row, o + r * (int64_t)d, &lse[r], nvis ? &nvis[r] : NULL);
            }
            free(s_row);
        }
    }
    (void)tokens;
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * oracle_attn_kvcache -- attention of the newest tokens against a key/value
 * cache ("FlashAttention" explainer page, How it works, Step 9: decoding with a
 * cache of past keys and values, one or a few new tokens at a time).
 *
 * Sequence b holds L_b = cache_seqlens[b] keys (the new tokens included); its
 * Nq query rows are the newest positions pos_i = L_b - Nq + i (so causal
 * masking is aligned to the end of the cache).  Key j is visible to query i iff
 *     (left < 0 || j >= pos_i - left) && (right < 0 || j <= pos_i + right),
 * causal forcing right = 0, j < L_b.
 *   q        [B, Nq, Hq, d]  bf16 bits
 *   k/v cache, pages of page_size rows: [num_pages, page_size, Hkv, d] bf16;
 *            logical key j of sequence b lives in page block_table[b * pages_per_seq
 *            + j / page_size] at row j % page_size; block_table == NULL means page
 *            b * pages_per_seq + j / page_size (a contiguous [B, pages_per_seq *
 *            page_size, Hkv, d] cache).
 *   o        [B, Nq, Hq, d] fp64,   lse [B, Hq, Nq] fp64,   nvis like lse (or NULL)
 * Requires L_b >= Nq for every sequence.
 */
int oracle_attn_kvcache(const uint16_t *q, const uint16_t *kc, const uint16_t *vc,
                        double *o, double *lse, int64_t *nvis,
                        const int32_t *cache_seqlens, const int32_t *block_table,
                        int B, int Hq, int Hkv, int Nq, int d, int page_size,
                        int pages_per_seq, double scale, int causal, int window_left,
                        int window_right, int nthreads) {
    if (!q || !kc || !vc || !o || !lse || !cache_seqlens) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || page_size <= 0 ||
        pages_per_seq <= 0)
        return ORACLE_ERR_ARG;
    if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
    const int group = Hq / Hkv;
    const int64_t left = window_left;
    const int64_t right = causal ? 0 : window_right;
    int64_t maxL = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t L = cache_seqlens[b];
        if (L < Nq || L > (int64_t)page_size * pages_per_seq) return ORACLE_ERR_ARG;
        if (L > maxL) maxL = L;
    }
#ifdef _OPENMP
    const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel num_threads(nt)
    {
        double *s_row = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        if (!s_row) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int b = 0; b < B; ++b) {
            for (int h = 0; h < Hq; ++h) {
                if (!s_row) continue;
                const int g = h / group;
                const int64_t L = cache_seqlens[b];
                for (int i = 0; i < Nq; ++i) {
                    const int64_t pos = L - Nq + i;
                    const uint16_t *qi = q + (((int64_t)b * Nq + i) * Hq + h) * d;
                    double *o_row = o + (((int64_t)b * Nq + i) * Hq + h) * d;
                    double M = -INFINITY;
                    int64_t n = 0;
                    for (int64_t j = 0; j < L; ++j) {
                        if (!key_visible(pos, j, left, right)) {
                            s_row[j] = -INFINITY;
                            continue;
                        }
                        const int64_t page = block_table
                                                 ? block_table[(int64_t)b * pages_per_seq + j / page_size]
                                                 : (int64_t)b * pages_per_seq + j / page_size;
                        const int64_t row = page * page_size + j % page_size;
                        const uint16_t *kj = kc + (row * Hkv + g) * d;
                        double dot = 0.0;
                        for (int t = 0; t < d; ++t) dot += widen_bf16(qi[t]) * widen_bf16(kj[t]);
                        s_row[j] = scale * dot;
                        if (s_row[j] > M) M = s_row[j];
                        ++n;
                    }
                    const int64_t li = ((int64_t)b * Hq + h) * Nq + i;
                    if (nvis) nvis[li] = n;
                    if (n == 0) {
                        for (int c = 0; c < d; ++c) o_row[c] = 0.0;
                        lse[li] = -INFINITY;
                        continue;
                    }
                    double Z = 0.0;
                    for (int64_t j = 0; j < L; ++j)
                        if (s_row[j] != -INFINITY) Z += exp(s_row[j] - M);
                    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
                    for (int64_t j = 0; j < L; ++j) {
                        if (s_row[j] == -INFINITY) continue;
                        const double p = exp(s_row[j] - M) / Z;
                        const int64_t page = block_table
                                                 ? block_table[(int64_t)b * pages_per_seq + j / page_size]
                                                 : (int64_t)b * pages_per_seq + j / page_size;
                        const int64_t row = page * page_size + j % page_size;
                        const uint16_t *vj = vc + (row * Hkv + g) * d;
                        for (int c = 0; c < d; ++c) o_row[c] += p * widen_bf16(vj[c]);
                    }
                    lse[li] = M + log(Z);
                }
            }
        }
        free(s_row);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * oracle_attn_bwd -- gradients of attention with respect to q, k and v.
 *
 * The pages ("FlashAttention" explainer page, How it works, Step 5, and
 * "Backward pass in a bit more detail") say what the backward pass needs
 * (queries, keys, values, the output gradient and each row's log-sum-exp; the
 * weights are rebuilt, key/value gradients accumulate over query rows and
 * query gradients over keys) but print no formulas.  This is the plain
 * chain rule for L = sum(dO * O) with O the forward above:
 *   P_ij  = exp(s_ij - LSE_i)              (the forward's weights)
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)             (softmax Jacobian)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i        summed over the query heads of the group
 *   dV_j  = sum_i P_ij dO_i                summed over the query heads of the group
 * with the forward's masks, head groups and sequences.  Phase 1 walks query
 * rows (scores, LSE, D and dQ); phase 2 walks keys and rebuilds the weights of
 * every row that sees the key from the row's LSE and D.
 *   q, dout [tokens, Hq, d] bf16 bits;  k, v [tokens, Hkv, d] bf16 bits
 *   dq [tokens, Hq, d] fp64;  dk, dv [tokens, Hkv, d] fp64
 * A row with no visible key contributes nothing.
 */
static double dot_bf16(const uint16_t *a, const uint16_t *b, int d) {
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += widen_bf16(a[t]) * widen_bf16(b[t]);
    return s;
}

int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    const uint16_t *dout, double *dq, double *dk, double *dv,
                    int B, int Hq, int Hkv, int N, int d, double scale,
                    int causal, int window_left, int window_right,
                    const int32_t *cu_seqlens, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0) return ORACLE_ERR_ARG;
    if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window_left < -1 || window_right < -1) return ORACLE_ERR_ARG;
    const int group = Hq / Hkv;
    const int64_t left = window_left;
    const int64_t right = causal ? 0 : window_right;
    const int64_t tokens = cu_seqlens ? (int64_t)cu_seqlens[B] : (int64_t)B * N;
    int64_t maxL = 0;
    for (int b = 0; b < B; ++b) {
        int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
        if (L < 0) return ORACLE_ERR_ARG;
        if (L > maxL) maxL = L;
    }
#ifdef _OPENMP
    const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
#endif
    double *lse = (double *)malloc(sizeof(double) * (size_t)(tokens * Hq > 0 ? tokens * Hq : 1));
    double *D = (double *)malloc(sizeof(double) * (size_t)(tokens * Hq > 0 ? tokens * Hq : 1));
    if (!lse || !D) {
        free(lse);
        free(D);
        return ORACLE_ERR_NOMEM;
    }
    int failed = 0;

    /* Phase 1: one query row at a time -- LSE_i, D_i and dQ_i. */
#pragma omp parallel num_threads(nt)
    {
        double *s_row = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        double *dp_row = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        if (!s_row || !dp_row) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t u = 0; u < tokens * Hq; ++u) {
            if (!s_row || !dp_row) continue;
            const int64_t t = u / Hq;
            const int h = (int)(u % Hq), g = h / group;
            int b = 0;
            if (cu_seqlens) {
                while (b + 1 < B && cu_seqlens[b + 1] <= t) ++b;
            } else {
                b = (int)(t / (N > 0 ? N : 1));
            }
            const int64_t start = cu_seqlens ? cu_seqlens[b] : (int64_t)b * N;
            const int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
            const int64_t i = t - start;
            const uint16_t *qi = q + (t * Hq + h) * (int64_t)d;
            const uint16_t *doi = dout + (t * Hq + h) * (int64_t)d;
            double *dqi = dq + (t * Hq + h) * (int64_t)d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            double M = -INFINITY;
            int64_t nvis = 0;
            for (int64_t j = 0; j < L; ++j) {
                if (!key_visible(i, j, left, right)) {
                    s_row[j] = -INFINITY;
                    continue;
                }
                const int64_t kj = ((start + j) * Hkv + g) * (int64_t)d;
                s_row[j] = scale * dot_bf16(qi, k + kj, d);
                dp_row[j] = dot_bf16(doi, v + kj, d);
                if (s_row[j] > M) M = s_row[j];
                ++nvis;
            }
            if (nvis == 0) {
                lse[u] = -INFINITY;
                D[u] = 0.0;
                continue;
            }
            double Z = 0.0;
            for (int64_t j = 0; j < L; ++j)
                if (s_row[j] != -INFINITY) Z += exp(s_row[j] - M);
            const double lse_i = M + log(Z);
            double Di = 0.0;
            for (int64_t j = 0; j < L; ++j)
                if (s_row[j] != -INFINITY) Di += exp(s_row[j] - lse_i) * dp_row[j];
            lse[u] = lse_i;
            D[u] = Di;
            for (int64_t j = 0; j < L; ++j) {
                if (s_row[j] == -INFINITY) continue;
                const double ds = exp(s_row[j] - lse_i) * (dp_row[j] - Di);
                const uint16_t *kj = k + ((start + j) * Hkv + g) * (int64_t)d;
                for (int c = 0; c < d; ++c) dqi[c] += scale * ds * widen_bf16(kj[c]);
            }
        }
        free(s_row);
        free(dp_row);
    }

    /* Phase 2: one key at a time -- dK_j and dV_j over every row that sees it. */
    if (!failed) {
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
        for (int64_t u = 0; u < tokens * Hkv; ++u) {
            const int64_t t = u / Hkv;
            const int g = (int)(u % Hkv);
            int b = 0;
            if (cu_seqlens) {
                while (b + 1 < B && cu_seqlens[b + 1] <= t) ++b;
            } else {
                b = (int)(t / (N > 0 ? N : 1));
            }
            const int64_t start = cu_seqlens ? cu_seqlens[b] : (int64_t)b * N;
            const int64_t L = cu_seqlens ? (int64_t)cu_seqlens[b + 1] - cu_seqlens[b] : N;
            const int64_t j = t - start;
            const uint16_t *kj = k + (t * Hkv + g) * (int64_t)d;
            const uint16_t *vj = v + (t * Hkv + g) * (int64_t)d;
            double *dkj = dk + (t * Hkv + g) * (int64_t)d;
            double *dvj = dv + (t * Hkv + g) * (int64_t)d;
            for (int c = 0; c < d; ++c) dkj[c] = dvj[c] = 0.0;
            for (int hh = 0; hh < group; ++hh) {
                const int h = g * group + hh;
                for (int64_t i = 0; i < L; ++i) {
                    if (!key_visible(i, j, left, right)) continue;
                    const int64_t r = (start + i) * Hq + h;
                    const uint16_t *qi = q + r * (int64_t)d;
                    const uint16_t *doi = dout + r * (int64_t)d;
                    const double p = exp(scale * dot_bf16(qi, kj, d) - lse[r]);
                    const double ds = p * (dot_bf16(doi, vj, d) - D[r]);
                    for (int c = 0; c < d; ++c) {
                        dkj[c] += scale * ds * widen_bf16(qi[c]);
                        dvj[c] += p * widen_bf16(doi[c]);
                    }
                }
            }
        }
    }
    free(lse);
    free(D);
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
