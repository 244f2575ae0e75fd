/*
 * qsa_oracle.c -- plain, slow, fp64 CPU oracle for Qwen Sparse Attention (QSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA library: inputs arrive as raw fp32 or bf16 bytes and are up-converted to
 * double exactly; every sum, product, exponential and comparison is in double.
 *
 * What it computes follows the Qwen4-Exp model documentation (Hugging Face
 * Transformers model doc "Qwen4-Exp"):
 *   - intro paragraph on QSA: several indexer query heads score compressed key
 *     blocks, the most relevant contiguous token blocks are selected, and the
 *     incomplete trailing block is kept uncompressed;
 *   - Qwen4ExpTextConfig parameters indexer_n_heads / indexer_kv_heads /
 *     indexer_head_dim / indexer_budget / indexer_compress_ratio: one indexer
 *     key head, the budget counts tokens taken from complete compressed blocks,
 *     a compressed block is the average of compress_ratio consecutive keys;
 *   - Qwen4ExpTextConfig parameter num_key_value_heads: grouped-query attention,
 *     query head h reads KV head h / (Hq / Hkv).
 * Readings of points the page leaves open (score formula, tie order, trailing
 * block at a block boundary, fewer candidates than k) are stated at each
 * function and are the same readings the CUDA path implements independently.
 *
 * Parity pins (the tests in tests/test_oracle_pins.py): closed forms for the
 * block mean and the score, brute-force subset enumeration for the selection,
 * equality with dense causal GQA attention (torch SDPA, fp64) when the budget
 * covers every block, causality, trailing-block, GQA-repeat, left-padding and
 * decode-equals-prefill invariants.  No function here is "parity unpinned".
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -o libqsa_oracle.so qsa_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Input element types: 0 = fp32, 1 = bf16 (raw 16-bit patterns). */
#define ORC_FP32 0
#define ORC_BF16 1

/* Exact up-conversion of one stored element to double. */
static double orc_load(const void *base, int dtype, size_t idx) {
    if (dtype == ORC_FP32) return (double)((const float *)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Block compression (Qwen4ExpTextConfig, indexer_compress_ratio: "consecutive
 * token keys averaged into one index block"; indexer_kv_heads: a single key
 * head).  ki is the indexer-key plane of one sequence, [n_keys][di], relative
 * position 0 first.  Only complete blocks exist: n_blocks = n_keys / B.
 * kbar[j][c] = (1/B) * sum_{u=jB}^{jB+B-1} ki[u][c].
 */
void qsa_oracle_compress(const void *ki, int dtype, int64_t n_keys, int di, int B,
                         double *kbar) {
    int64_t n_blocks = n_keys / B;
    for (int64_t j = 0; j < n_blocks; ++j) {
        for (int c = 0; c < di; ++c) {
            double acc = 0.0;
            for (int u = 0; u < B; ++u) acc += orc_load(ki, dtype, (size_t)(j * B + u) * di + c);
            kbar[j * di + c] = acc / (double)B;
        }
    }
}

/*
 * Multi-head block scores for one query position (intro: "multiple query
 * heads score compressed key blocks").  The page gives no formula; the reading
 * used is s_j = sum_{h < Hi} max(0, qi[h] . kbar[j]), no scale, no per-head
 * weights.  qi_row is [Hi][di] of one query; s receives n_c scores.
 */
void qsa_oracle_block_scores(const void *qi_row, int dtype, int Hi, int di,
                             const double *kbar, int64_t n_c, double *s) {
    for (int64_t j = 0; j < n_c; ++j) {
        double total = 0.0;
        for (int h = 0; h < Hi; ++h) {
            double dot = 0.0;
            for (int c = 0; c < di; ++c)
                dot += orc_load(qi_row, dtype, (size_t)h * di + c) * kbar[j * di + c];
            total += dot > 0.0 ? dot : 0.0;
        }
        s[j] = total;
    }
}

typedef struct {
    double score;
    int64_t idx;
} orc_pair;

/* Order: higher score first; equal scores -> lower block index first. */
static int orc_rank_cmp(const void *a, const void *b) {
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

static int orc_int_cmp(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Top-k block selection (intro: "selects the most relevant contiguous token
 * blocks"; indexer_budget: tokens taken from complete compressed blocks).
 * Candidates are the n_c complete blocks visible to the query.  If n_c <= k all
 * are kept; otherwise the k best under the order (-score, index) are kept, so
 * ties go to the lower block index.  Output: k entries, ascending block index,
 * padded with -1.  Returns the number of blocks selected.
 */
int qsa_oracle_select(const double *s, int64_t n_c, int k, int32_t *sel) {
    orc_pair *p = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(n_c > 0 ? n_c : 1));
    for (int64_t j = 0; j < n_c; ++j) {
        p[j].score = s[j];
        p[j].idx = j;
    }
    qsort(p, (size_t)n_c, sizeof(orc_pair), orc_rank_cmp);
    int n_sel = (int)(n_c < k ? n_c : k);
    for (int i = 0; i < n_sel; ++i) sel[i] = (int32_t)p[i].idx;
    qsort(sel, (size_t)n_sel, sizeof(int32_t), orc_int_cmp);
    for (int i = n_sel; i < k; ++i) sel[i] = -1;
    free(p);
    return n_sel;
}

/*
 * The token set a query at relative position t attends (intro: selected
 * contiguous blocks plus the incomplete trailing block, kept uncompressed).
 * With L = t + 1 visible tokens, n_c = L / B complete blocks; the trailing
 * block is [n_c * B, t], empty exactly when L is a multiple of B (then the
 * block just completed is a compressed candidate like any other).  Writes the
 * ascending token list into toks and returns its length.
 */
int64_t qsa_oracle_token_set(int64_t t, int B, const int32_t *sel, int k, int64_t *toks) {
    int64_t n = 0;
    int64_t n_c = (t + 1) / B;
    for (int i = 0; i < k; ++i) {
        if (sel[i] < 0) continue;
        for (int u = 0; u < B; ++u) toks[n++] = (int64_t)sel[i] * B + u;
    }
    for (int64_t u = n_c * B; u <= t; ++u) toks[n++] = u;
    return n;
}

/*
 * Exact softmax attention of one query row over a token list (Usage tips:
 * sparse token selection with eager/SDPA attention, i.e. ordinary softmax
 * attention restricted to the selected tokens; num_key_value_heads: GQA).
 * q_row [Hq][d]; k, v are the sequence's planes [Hkv][kv_stride][d] starting at
 * relative position 0; o_row [Hq][d] receives the fp64 result.
 */
void qsa_oracle_attend(const void *q_row, const void *k, const void *v, int dtype,
                       int Hq, int Hkv, int d, int64_t kv_stride, double scale,
                       const int64_t *toks, int64_t n_toks, double *o_row) {
    int G = Hq / Hkv;
    double *logit = (double *)malloc(sizeof(double) * (size_t)(n_toks > 0 ? n_toks : 1));
    for (int h = 0; h < Hq; ++h) {
        int g = h / G;
        const size_t kv_base = (size_t)g * (size_t)kv_stride * (size_t)d;
        double mx = -INFINITY;
        for (int64_t i = 0; i < n_toks; ++i) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += orc_load(q_row, dtype, (size_t)h * d + c) *
                       orc_load(k, dtype, kv_base + (size_t)toks[i] * d + c);
            logit[i] = scale * dot;
            if (logit[i] > mx) mx = logit[i];
        }
        double denom = 0.0;
        for (int64_t i = 0; i < n_toks; ++i) {
            logit[i] = exp(logit[i] - mx);
            denom += logit[i];
        }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < n_toks; ++i)
                acc += logit[i] * orc_load(v, dtype, kv_base + (size_t)toks[i] * d + c);
            o_row[(size_t)h * d + c] = n_toks > 0 ? acc / denom : 0.0;
        }
    }
    free(logit);
}

/*
 * The whole path for a set of query rows of ONE sequence: compress the
 * sequence's complete blocks, then per row score, select, gather the token set
 * and attend.  Prefill and decode are the same computation; a decode step is
 * the row t = L - 1 of a sequence of L visible tokens.
 *
 *   q     [n_rows][Hq][d]      qi [n_rows][Hi][di]     t_pos [n_rows]
 *   k, v  [Hkv][kv_stride][d]  ki [n_keys][di]         (relative position 0 first)
 *   o     [n_rows][Hq][d] fp64 out;  sel [n_rows][k] out;  kbar [n_keys/B][di] out
 *         (kbar may be NULL).  Rows with t_pos < 0 or >= n_keys are padding:
 *         o = 0, sel = -1.
 * Rows are independent; OpenMP spreads them over n_threads host threads
 * (n_threads <= 0 keeps the runtime default).
 */
void qsa_oracle_sequence(const void *q, const void *qi, const int64_t *t_pos, int64_t n_rows,
                         const void *k, const void *v, const void *ki, int64_t n_keys,
                         int64_t kv_stride, int dtype, int Hq, int Hkv, int d, int Hi, int di,
                         int B, int topk, double scale, double *o, int32_t *sel, double *kbar_out,
                         int n_threads) {
    int64_t n_blocks = n_keys / B;
    double *kbar = (double *)malloc(sizeof(double) * (size_t)(n_blocks > 0 ? n_blocks : 1) * di);
    qsa_oracle_compress(ki, dtype, n_keys, di, B, kbar);
    if (kbar_out) memcpy(kbar_out, kbar, sizeof(double) * (size_t)n_blocks * di);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(n_blocks > 0 ? n_blocks : 1));
        int64_t *toks = (int64_t *)malloc(sizeof(int64_t) * (size_t)((int64_t)topk * B + B));
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t t = t_pos[r];
            double *o_row = o + (size_t)r * Hq * d;
            int32_t *sel_row = sel + (size_t)r * topk;
            if (t < 0 || t >= n_keys) {
                memset(o_row, 0, sizeof(double) * (size_t)Hq * d);
                for (int i = 0; i < topk; ++i) sel_row[i] = -1;
                continue;
            }
            int64_t n_c = (t + 1) / B;
            const char *qi_row = (const char *)qi + (size_t)r * Hi * di * (dtype == ORC_FP32 ? 4 : 2);
            const char *q_row = (const char *)q + (size_t)r * Hq * d * (dtype == ORC_FP32 ? 4 : 2);
            qsa_oracle_block_scores(qi_row, dtype, Hi, di, kbar, n_c, s);
            qsa_oracle_select(s, n_c, topk, sel_row);
            int64_t n_toks = qsa_oracle_token_set(t, B, sel_row, topk, toks);
            qsa_oracle_attend(q_row, k, v, dtype, Hq, Hkv, d, kv_stride, scale, toks, n_toks, o_row);
        }
        free(toks);
        free(s);
    }
    free(kbar);
}

/* Row-level scores of one sequence, for diagnostics of near-ties: s [n_rows][n_blocks],
 * entries j >= n_c(t) are set to -1 (not candidates). */
void qsa_oracle_sequence_scores(const void *qi, const int64_t *t_pos, int64_t n_rows,
                                const void *ki, int64_t n_keys, int dtype, int Hi, int di, int B,
                                double *s_out, int n_threads) {
    int64_t n_blocks = n_keys / B;
    double *kbar = (double *)malloc(sizeof(double) * (size_t)(n_blocks > 0 ? n_blocks : 1) * di);
    qsa_oracle_compress(ki, dtype, n_keys, di, B, kbar);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; ++r) {
        double *row = s_out + (size_t)r * n_blocks;
        for (int64_t j = 0; j < n_blocks; ++j) row[j] = -1.0;
        int64_t t = t_pos[r];
        if (t < 0 || t >= n_keys) continue;
        int64_t n_c = (t + 1) / B;
        const char *qi_row = (const char *)qi + (size_t)r * Hi * di * (dtype == ORC_FP32 ? 4 : 2);
        qsa_oracle_block_scores(qi_row, dtype, Hi, di, kbar, n_c, row);
    }
    free(kbar);
}

/*
 * Input projections and rotary position embedding, the steps before the path
 * (Qwen4ExpTextConfig: hidden_size, attention_bias = False so no bias terms,
 * rope_parameters with rope_theta; num_attention_heads / num_key_value_heads /
 * head_dim for q, k, v; indexer_n_heads / indexer_head_dim for the indexer query
 * heads and the single indexer key head).
 *
 * One rotary head of dimension hd at position pos, in place, rotate-half form
 * (readings: the page fixes neither the pairing nor the rotary fraction): the
 * first rd dims rotate (rd even, <= hd); for i < rd / 2, with
 * angle_i = pos * theta^(-2 i / rd), the pair (h[i], h[i + rd/2]) becomes
 * (h[i] cos - h[i + rd/2] sin, h[i + rd/2] cos + h[i] sin); dims >= rd are kept.
 */
void qsa_oracle_rope_head(double *h, int hd, int rd, double pos, double theta) {
    (void)hd;
    int half = rd / 2;
    for (int i = 0; i < half; ++i) {
        double ang = pos * pow(theta, -2.0 * (double)i / (double)rd);
        double c = cos(ang), sn = sin(ang);
        double a = h[i], b = h[i + half];
        h[i] = a * c - b * sn;
        h[i + half] = b * c + a * sn;
    }
}

/*
 * y[r][o] = sum_c x[r][c] w[o][c] for the stacked weight rows
 *   [W_q: Hq*d][W_k: Hkv*d][W_v: Hkv*d][W_qi: Hi*di][W_ki: di]   (n_out rows of D)
 * then RoPE at position pos[r] on every q and k head (rotary dims rd_attn) and on
 * every indexer query head and the indexer key head (rotary dims rd_idx; 0 = none);
 * v is never rotated.  x [n_rows][D] and w in fp32 or bf16 (dtype), y fp64.
 */
void qsa_oracle_project_rope(const void *x, const void *w, int dtype, int64_t n_rows, int D,
                             const int64_t *pos, double theta, int Hq, int Hkv, int d, int Hi,
                             int di, int rd_attn, int rd_idx, double *y, int n_threads) {
    int n_out = Hq * d + 2 * Hkv * d + Hi * di + di;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
        double *yr = y + (size_t)r * n_out;
        for (int o = 0; o < n_out; ++o) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c)
                acc += orc_load(x, dtype, (size_t)r * D + c) * orc_load(w, dtype, (size_t)o * D + c);
            yr[o] = acc;
        }
        double p = (double)pos[r];
        for (int h = 0; h < Hq + Hkv; ++h) qsa_oracle_rope_head(yr + (size_t)h * d, d, rd_attn, p, theta);
        double *yi = yr + (size_t)(Hq + 2 * Hkv) * d;
        if (rd_idx > 0)
            for (int h = 0; h < Hi + 1; ++h) qsa_oracle_rope_head(yi + (size_t)h * di, di, rd_idx, p, theta);
    }
}

int qsa_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
