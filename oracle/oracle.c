/*
 * oracle.c -- plain, slow, fp64 CPU oracle for single-token GQA decode with
 * output-aware token dropping (OAM), an INT8 KV cache and split-KV merging.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; it is compiled with plain
 * gcc (no fast-math) and every loop below is the textbook definition, with no
 * blocking, fusion or reordering.
 *
 * Sources (web pages; cited by title and section):
 *   [TD]  "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse
 *         attention), lzwjava.github.io: section 2 (attention output), section 3
 *         (OAM score pseudocode), section 5 (split-KV and the cross-chunk
 *         online-softmax reduction), section 6 (INT8 KV cache, schemes A and B).
 *   [AO]  "注意力优化（Attention Optimization）", learnagent.wiki: core principle
 *         (softmax(QK^T/sqrt(d_k))V), the GQA example (repeat_interleave mapping).
 *   [CD]  "共同设计 AI 模型注意力，实现快速的交互式长上下文推理" (Co-designing AI
 *         model attention for fast interactive long-context inference), NVIDIA
 *         developer blog: decode equations 5-7 (decode streams the KV cache).
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py
 * against closed forms, invariants, library routines or brute force; none is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Attention of the G query heads of one KV group over n cached tokens.      */
/*                                                                          */
/* [TD] section 2 and [AO] core principle: out = sum_t softmax_t(z_t) v_t,   */
/* z_t = q . k_t / sqrt(d).  The softmax is taken over exactly the n tokens  */
/* passed in (the kept set when tokens were dropped).  Also returns          */
/* lse = ln sum_t exp(z_t), the natural-log normaliser, computed as          */
/* m + ln(sum_t exp(z_t - m)) with m = max_t z_t.                            */
/*   q [G][D], k [n][D], v [n][D]  ->  out [G][D], lse [G]                   */
/* Returns 0, or -1 when n, D or G is not positive.                          */
/* ------------------------------------------------------------------------ */
int orc_attend(int D, int G, int64_t n, const double *q, const double *k,
               const double *v, double *out, double *lse)
{
    if (n < 1 || D < 1 || G < 1)
        return -1;
    double *z = (double *)malloc((size_t)n * sizeof(double));
    if (!z)
        return -2;
    const double sqrt_d = sqrt((double)D);
    for (int g = 0; g < G; ++g) {
        const double *qg = q + (size_t)g * D;
        double m = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += qg[d] * k[(size_t)t * D + d];
            z[t] = dot / sqrt_d;
            if (z[t] > m)
                m = z[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < n; ++t)
            l += exp(z[t] - m);
        double *og = out + (size_t)g * D;
        for (int d = 0; d < D; ++d)
            og[d] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const double w = exp(z[t] - m);
            for (int d = 0; d < D; ++d)
                og[d] += w * v[(size_t)t * D + d];
        }
        for (int d = 0; d < D; ++d)
            og[d] /= l;
        lse[g] = m + log(l);
    }
    free(z);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Exact merge of C split-KV partial results of one KV group.               */
/*                                                                          */
/* [TD] section 5: each chunk reports its own normalised output o_c and its  */
/* log-sum-exp lse_c; the combined result is                                 */
/*   lse = ln sum_c exp(lse_c)       (taken as M + ln sum_c exp(lse_c - M)) */
/*   out = sum_c exp(lse_c - lse) o_c                                        */
/* This is the page's running (m, exp_sum, out) recurrence written in        */
/* closed form, with the factor exp(m_chunk - m_new) on the chunk term that  */
/* the printed out-update omits (the exp_sum update on the same page has it).*/
/*   o_c [C][G][D], lse_c [C][G]  ->  out [G][D], lse [G]                    */
/* ------------------------------------------------------------------------ */
int orc_merge(int C, int G, int D, const double *o_c, const double *lse_c,
              double *out, double *lse)
{
    if (C < 1 || G < 1 || D < 1)
        return -1;
    for (int g = 0; g < G; ++g) {
        double M = -INFINITY;
        for (int c = 0; c < C; ++c)
            if (lse_c[(size_t)c * G + g] > M)
                M = lse_c[(size_t)c * G + g];
        double s = 0.0;
        for (int c = 0; c < C; ++c)
            s += exp(lse_c[(size_t)c * G + g] - M);
        const double L = M + log(s);
        lse[g] = L;
        for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int c = 0; c < C; ++c)
                acc += exp(lse_c[(size_t)c * G + g] - L) * o_c[((size_t)c * G + g) * D + d];
            out[(size_t)g * D + d] = acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* INT8 quantisation primitives.                                            */
/*                                                                          */
/* [TD] section 6: q_val = round(val / scale), val ~= q_val * scale, and     */
/* scale = max|x| / 127 over the group that shares the scale.  Readings used */
/* here: the scale is the float32 value nearest to amax/127; the quotient is */
/* the float32 value nearest to val/scale (computed in double and rounded    */
/* once, which equals the correctly rounded float32 quotient because         */
/* 53 >= 2*24 + 2); round() is round-half-to-even; codes are clamped to      */
/* [-127, 127]; a group whose scale is zero gets all-zero codes.             */
/* ------------------------------------------------------------------------ */
float orc_amax(const float *x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        const float a = fabsf(x[i]);
        if (a > m)
            m = a;
    }
    return m;
}

float orc_scale_from_amax(float amax)
{
    return (float)((double)amax / 127.0);
}

int8_t orc_code(float x, float scale)
{
    if (scale == 0.0f)
        return 0;
    const float quotient = (float)((double)x / (double)scale);
    double r = nearbyint((double)quotient); /* default rounding mode: half to even */
    if (r > 127.0)
        r = 127.0;
    if (r < -127.0)
        r = -127.0;
    return (int8_t)r;
}

void orc_quantize(const float *x, int64_t n, float scale, int8_t *codes)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = orc_code(x[i], scale);
}

/* Scheme A keys ([TD] section 6, "fine-grained QK"): one scale per partition of
 * `part` consecutive tokens, partitions counted from the first token of the
 * sequence; the last partition takes the remaining (< part) tokens.  The scale
 * covers every channel of every token in the partition.
 *   x [n_tok][D] -> scales [ceil(n_tok/part)], codes [n_tok][D]               */
void orc_quantize_partitions(const float *x, int64_t n_tok, int D, int part,
                             float *scales, int8_t *codes)
{
    const int64_t n_part = (n_tok + part - 1) / part;
    for (int64_t p = 0; p < n_part; ++p) {
        const int64_t t0 = p * part;
        const int64_t t1 = (t0 + part < n_tok) ? t0 + part : n_tok;
        const int64_t len = (t1 - t0) * D;
        const float s = orc_scale_from_amax(orc_amax(x + t0 * D, len));
        scales[p] = s;
        orc_quantize(x + t0 * D, len, s, codes + t0 * D);
    }
}

/* ------------------------------------------------------------------------ */
/* Output-aware token score (OAM) of n tokens for one KV group.             */
/*                                                                          */
/* [TD] section 3 pseudocode: score = q . k / sqrt(d_k) + beta * ln(|v| + eps)*/
/* with |v| the Euclidean norm of the value row and natural log.  Selection  */
/* is shared by the G query heads of the group (one index set per KV head);  */
/* the group's routing term is the largest of its G scaled logits.           */
/*   q [G][D], k [n][D], v [n][D] -> s [n]                                   */
/* ------------------------------------------------------------------------ */
int orc_oam_scores(int D, int G, int64_t n, const double *q, const double *k,
                   const double *v, double beta, double eps, double *s)
{
    if (D < 1 || G < 1 || n < 0)
        return -1;
    const double sqrt_d = sqrt((double)D);
    for (int64_t t = 0; t < n; ++t) {
        double best = -INFINITY;
        for (int g = 0; g < G; ++g) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += q[(size_t)g * D + d] * k[(size_t)t * D + d];
            const double z = dot / sqrt_d;
            if (z > best)
                best = z;
        }
        double sq = 0.0;
        for (int d = 0; d < D; ++d)
            sq += v[(size_t)t * D + d] * v[(size_t)t * D + d];
        s[t] = best + beta * log(sqrt(sq) + eps);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Top-K token selection ([TD] section 3: drop the tokens with the lowest    */
/* score, keep the K highest).  Ties are broken by the lower token index, so */
/* the order is the total order (score descending, index ascending); the     */
/* kept indices are returned in ascending order.                             */
/*   s [n], K in [1, n] -> idx [K]                                           */
/* ------------------------------------------------------------------------ */
static const double *g_sort_scores; /* single-threaded use only */

static int by_score_then_index(const void *a, const void *b)
{
    const int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    const double si = g_sort_scores[i], sj = g_sort_scores[j];
    if (si > sj)
        return -1;
    if (si < sj)
        return 1;
    return (i > j) - (i < j);
}

static int ascending(const void *a, const void *b)
{
    const int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    return (i > j) - (i < j);
}

int orc_topk(int64_t n, const double *s, int64_t K, int32_t *idx)
{
    if (n < 1 || K < 1 || K > n)
        return -1;
    int32_t *order = (int32_t *)malloc((size_t)n * sizeof(int32_t));
    if (!order)
        return -2;
    for (int64_t t = 0; t < n; ++t)
        order[t] = (int32_t)t;
    g_sort_scores = s;
    qsort(order, (size_t)n, sizeof(int32_t), by_score_then_index);
    memcpy(idx, order, (size_t)K * sizeof(int32_t));
    qsort(idx, (size_t)K, sizeof(int32_t), ascending);
    free(order);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Equal-work split-KV partition ([TD] section 5: cut the KV of each row into */
/* chunks handled by separate CTAs so that a 128K row and a 512 row do not   */
/* leave CTAs idle).  The rule, written out:                                 */
/*   - the rows (one per (KV head, sequence), in stream order) are laid end  */
/*     to end, each padded to a multiple of `granule` tokens and followed by */
/*     `row_cost` more positions (a fixed work charge per row: its segment   */
/*     setup and merge; 0 gives the plain token split);                      */
/*   - mode 0 (equal work): the padded stream of W tokens is cut into CTA    */
/*     ranges of S = max(min_chunk, round_up(ceil(W / n_req), granule))      */
/*     tokens, the last one shorter; mode 1: one CTA per row;                */
/*   - a segment is the intersection of one CTA range with the real (not     */
/*     padding) tokens of one row; segments are numbered in stream order,    */
/*     and each segment yields one partial result (slot).                    */
/* Writes up to max_segs segments (cta, row, row-local start, length) and    */
/* returns their number, the number of CTAs through *n_cta, or -1.           */
/* ------------------------------------------------------------------------ */
int64_t orc_plan(int R, const int64_t *len, int n_req, int granule, int min_chunk,
                 int mode, int row_cost, int64_t max_segs, int32_t *seg_cta, int32_t *seg_row,
                 int64_t *seg_start, int64_t *seg_len, int32_t *n_cta)
{
    if (R < 1 || granule < 1 || row_cost < 0 || (mode == 0 && n_req < 1))
        return -1;
    int64_t *pos = (int64_t *)malloc(((size_t)R + 1) * sizeof(int64_t));
    if (!pos)
        return -2;
    pos[0] = 0;
    for (int r = 0; r < R; ++r) {
        if (len[r] < 1) {
            free(pos);
            return -1;
        }
        pos[r + 1] = pos[r] + (len[r] + granule - 1) / granule * granule + row_cost;
    }
    const int64_t W = pos[R];
    int64_t count = 0;
    int ncta = 0;
    if (mode == 0) {
        int64_t S = (W + n_req - 1) / n_req;
        S = (S + granule - 1) / granule * granule;
        if (S < min_chunk)
            S = min_chunk;
        for (int64_t a = 0; a < W; a += S, ++ncta) {
            const int64_t b = (a + S < W) ? a + S : W;
            for (int r = 0; r < R; ++r) {
                const int64_t lo = (a > pos[r]) ? a : pos[r];
                const int64_t hi_pad = (b < pos[r + 1]) ? b : pos[r + 1];
                const int64_t hi = (hi_pad < pos[r] + len[r]) ? hi_pad : pos[r] + len[r];
                if (hi <= lo)
                    continue;
                if (count < max_segs) {
                    seg_cta[count] = ncta;
                    seg_row[count] = r;
                    seg_start[count] = lo - pos[r];
                    seg_len[count] = hi - lo;
                }
                ++count;
            }
        }
    } else {
        for (int r = 0; r < R; ++r, ++ncta) {
            if (count < max_segs) {
                seg_cta[count] = r;
                seg_row[count] = r;
                seg_start[count] = 0;
                seg_len[count] = len[r];
            }
            ++count;
        }
    }
    free(pos);
    *n_cta = ncta;
    return count;
}
