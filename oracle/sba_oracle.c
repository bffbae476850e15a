/*
 * Plain CPU oracle for group-shared block-sparse decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library: it reads the same raw buffers (bf16 bit patterns, int32 tables) and
 * computes everything itself, step by step, in double precision, in the order
 * the method is stated, with no blocking or fusion.
 *
 * Sources (page title, section):
 *  [ReSA]  "Rectified Sparse Attention for Efficient Long-Sequence Generation",
 *          Summary (Quest-style min/max block descriptors score memory blocks;
 *          all query heads of a GQA group share one block selection) and Key
 *          points (dynamic top-n that always keeps the recent local blocks and a
 *          minimum block count; sparsity p).  Its references list cites
 *          Quest (query-aware min/max bounds), Flash-Decoding (split-KV with a
 *          log-sum-exp merge) and PagedAttention (block tables).
 *  [SAS]   "SAS: Simple Attention Sparsification via End-to-End Optimization of
 *          Context Ranking", Method (current block B0 with unit gate; candidate
 *          historical blocks B1..BC; g = softmax(s); o_SAS = softmax(q K_S^T +
 *          log g_S) V_S, with the current block unbiased) and Limitations
 *          (pooling-based block summaries).
 *  [SeerR] "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning",
 *          abstract (plug-in gate that scores blocks from the decode query,
 *          no query pooling).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - Quest score of block j for one head: sum_c max(q_c*mn_jc, q_c*mx_jc),
 *    the tightest per-channel upper bound of q.k over the block's key box.
 *  - The group shares one selection by SUMMING per-head scores over the heads
 *    of the group (for the gate: summing per-head softmax probabilities).
 *  - Budget counts the local blocks; n_sel = min(N, max(L, n_min, budget)),
 *    budget = n_budget or ceil(N*keep_num/keep_den) for a sparsity ratio.
 *  - Local blocks are the last L logical blocks {N-L..N-1}; they are not
 *    ranked.  Ranking is by fp32 score descending, then block index
 *    ascending; -0 and +0 are equal.  Output indices ascend.
 *  - Gate: pooled = [max || min || avg] over the block's valid keys (3d),
 *    kg = Wk pooled, q' = Wq q, u_j = q'.kg_j / sqrt(dg); g = softmax over the
 *    C = N-1 historical blocks 0..N-2; block N-1 is B0 (gate 1, bias 0) and is
 *    always kept; log-gate bias = log g_j = u_j - logsumexp(u).
 *  - Logits: l_t = (q.k_t)*scale + bias_j(t); tokens t >= len are masked.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> double (exact: bf16 is the top half of a float). */
static double bf16_to_double(uint16_t x)
{
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const uint16_t *k;          /* [num_pages][H_kv][b][d] bf16 bits */
    const uint16_t *v;          /* same layout */
    const int32_t *block_table; /* [B][max_blocks] or NULL (contiguous) */
    const int32_t *seq_lens;    /* [B] */
    int32_t B, H_q, H_kv, d, b, max_blocks, num_pages;
} orc_cache;

/* Physical page of logical block j of sequence s (PagedAttention-style
 * block table; NULL table = page s*max_blocks + j). */
static int64_t page_of(const orc_cache *c, int s, int j)
{
    if (c->block_table)
        return c->block_table[(int64_t)s * c->max_blocks + j];
    return (int64_t)s * c->max_blocks + j;
}

static int num_blocks(const orc_cache *c, int s)
{
    int len = c->seq_lens[s];
    return len <= 0 ? 0 : (len + c->b - 1) / c->b;
}

/* Key element (token t of sequence s, kv head h, channel ch). */
static double key_at(const orc_cache *c, int s, int t, int h, int ch)
{
    int64_t p = page_of(c, s, t / c->b);
    int64_t off = (((p * c->H_kv + h) * c->b) + (t % c->b)) * c->d + ch;
    return bf16_to_double(c->k[off]);
}

static double val_at(const orc_cache *c, int s, int t, int h, int ch)
{
    int64_t p = page_of(c, s, t / c->b);
    int64_t off = (((p * c->H_kv + h) * c->b) + (t % c->b)) * c->d + ch;
    return bf16_to_double(c->v[off]);
}

/* ------------------------------------------------------------------------ */
/* Block descriptors                                                         */
/* ------------------------------------------------------------------------ */

/* Quest-style descriptor [ReSA Summary; Quest]: per channel, the min and the
 * max of the block's VALID keys (tokens j*b .. min((j+1)*b, len)-1).
 * Output indexed by LOGICAL block: mn, mx [B][max_blocks][H_kv][d]; blocks at
 * or past N are left untouched. */
void orc_quest_desc(const orc_cache *c, double *mn, double *mx)
{
    for (int s = 0; s < c->B; ++s) {
        int len = c->seq_lens[s];
        int N = num_blocks(c, s);
        for (int j = 0; j < N; ++j) {
            int t0 = j * c->b;
            int t1 = t0 + c->b < len ? t0 + c->b : len;
            for (int h = 0; h < c->H_kv; ++h) {
                for (int ch = 0; ch < c->d; ++ch) {
                    double lo = key_at(c, s, t0, h, ch), hi = lo;
                    for (int t = t0 + 1; t < t1; ++t) {
                        double x = key_at(c, s, t, h, ch);
                        if (x < lo) lo = x;
                        if (x > hi) hi = x;
                    }
                    int64_t o = (((int64_t)s * c->max_blocks + j) * c->H_kv + h) * c->d + ch;
                    mn[o] = lo;
                    mx[o] = hi;
                }
            }
        }
    }
}

/* Pooled block summary for the gate [SAS Limitations: pooling-based block
 * summaries]: pooled = [max || min || avg] over the valid keys, 3*d values.
 * kg = Wk . pooled with Wk [dg][3d] row-major (no bias).
 * pooled [B][max_blocks][H_kv][3d], kg [B][max_blocks][H_kv][dg]. */
void orc_gate_desc(const orc_cache *c, const float *Wk, int dg, double *pooled, double *kg)
{
    int d = c->d;
    double *p = (double *)malloc(sizeof(double) * 3 * d);
    for (int s = 0; s < c->B; ++s) {
        int len = c->seq_lens[s];
        int N = num_blocks(c, s);
        for (int j = 0; j < N; ++j) {
            int t0 = j * c->b;
            int t1 = t0 + c->b < len ? t0 + c->b : len;
            for (int h = 0; h < c->H_kv; ++h) {
                for (int ch = 0; ch < d; ++ch) {
                    double hi = key_at(c, s, t0, h, ch), lo = hi, sum = 0.0;
                    for (int t = t0; t < t1; ++t) {
                        double x = key_at(c, s, t, h, ch);
                        if (x > hi) hi = x;
                        if (x < lo) lo = x;
                        sum += x;
                    }
                    p[ch] = hi;
                    p[d + ch] = lo;
                    p[2 * d + ch] = sum / (double)(t1 - t0);
                }
                int64_t base = ((int64_t)s * c->max_blocks + j) * c->H_kv + h;
                for (int i = 0; i < 3 * d; ++i)
                    pooled[base * 3 * d + i] = p[i];
                for (int r = 0; r < dg; ++r) {
                    double acc = 0.0;
                    for (int i = 0; i < 3 * d; ++i)
                        acc += (double)Wk[(int64_t)r * 3 * d + i] * p[i];
                    kg[base * dg + r] = acc;
                }
            }
        }
    }
    free(p);
}

/* ------------------------------------------------------------------------ */
/* Block scores                                                              */
/* ------------------------------------------------------------------------ */

/* Quest group score [ReSA Summary]: for each sequence s, kv head g and block
 * j < N, score = sum over the query heads qh of group g of
 * sum_c max(q_c*mn_jc, q_c*mx_jc).  q: bf16 bits [B][H_q][d].
 * score [B][H_kv][max_blocks] (blocks >= N untouched). */
void orc_quest_scores(const orc_cache *c, const uint16_t *q, double *score)
{
    int64_t nd = (int64_t)c->B * c->max_blocks * c->H_kv * c->d;
    double *mn = (double *)malloc(sizeof(double) * nd);
    double *mx = (double *)malloc(sizeof(double) * nd);
    orc_quest_desc(c, mn, mx);
    int G = c->H_q / c->H_kv;
    for (int s = 0; s < c->B; ++s) {
        int N = num_blocks(c, s);
        for (int g = 0; g < c->H_kv; ++g) {
            for (int j = 0; j < N; ++j) {
                double total = 0.0;
                for (int hh = 0; hh < G; ++hh) {
                    int qh = g * G + hh;
                    for (int ch = 0; ch < c->d; ++ch) {
                        double qc = bf16_to_double(q[((int64_t)s * c->H_q + qh) * c->d + ch]);
                        int64_t o = (((int64_t)s * c->max_blocks + j) * c->H_kv + g) * c->d + ch;
                        double a = qc * mn[o], bb = qc * mx[o];
                        total += a > bb ? a : bb;
                    }
                }
                score[((int64_t)s * c->H_kv + g) * c->max_blocks + j] = total;
            }
        }
    }
    free(mn);
    free(mx);
}

/* Gate group score [SeerR abstract; SAS Method]: q' = Wq q (Wq [dg][d]),
 * u_j = q'.kg_j / sqrt(dg) for the historical blocks j = 0..N-2,
 * g_j = exp(u_j - LSE) with LSE = log sum_j exp(u_j), score_j = sum over the
 * group's heads of g_j.  logg [B][H_q][max_blocks] receives log g_j = u_j - LSE
 * for j < N-1 and 0 for the current block j = N-1 (unit gate).
 * score [B][H_kv][max_blocks]: entries j < N-1 written, j = N-1 set to 0. */
void orc_gate_scores(const orc_cache *c, const uint16_t *q, const float *Wq, const float *Wk,
                     int dg, double *score, double *logg)
{
    int d = c->d;
    int64_t nb = (int64_t)c->B * c->max_blocks * c->H_kv;
    double *pooled = (double *)malloc(sizeof(double) * nb * 3 * d);
    double *kg = (double *)malloc(sizeof(double) * nb * dg);
    orc_gate_desc(c, Wk, dg, pooled, kg);
    int G = c->H_q / c->H_kv;
    double *qp = (double *)malloc(sizeof(double) * dg);
    double *u = (double *)malloc(sizeof(double) * (c->max_blocks > 0 ? c->max_blocks : 1));
    for (int s = 0; s < c->B; ++s) {
        int N = num_blocks(c, s);
        for (int g = 0; g < c->H_kv; ++g) {
            for (int j = 0; j < N; ++j)
                score[((int64_t)s * c->H_kv + g) * c->max_blocks + j] = 0.0;
        }
        for (int qh = 0; qh < c->H_q; ++qh) {
            int g = qh / G;
            for (int r = 0; r < dg; ++r) {
                double acc = 0.0;
                for (int ch = 0; ch < d; ++ch)
                    acc += (double)Wq[(int64_t)r * d + ch] *
                           bf16_to_double(q[((int64_t)s * c->H_q + qh) * d + ch]);
                qp[r] = acc;
            }
            int C = N - 1; /* number of historical blocks */
            double m = -INFINITY;
            for (int j = 0; j < C; ++j) {
                double acc = 0.0;
                for (int r = 0; r < dg; ++r)
                    acc += qp[r] * kg[((((int64_t)s * c->max_blocks + j) * c->H_kv) + g) * dg + r];
                u[j] = acc / sqrt((double)dg);
                if (u[j] > m) m = u[j];
            }
            double z = 0.0;
            for (int j = 0; j < C; ++j)
                z += exp(u[j] - m);
            double lse = m + log(z);
            for (int j = 0; j < C; ++j) {
                double lg = u[j] - lse;
                logg[((int64_t)s * c->H_q + qh) * c->max_blocks + j] = lg;
                score[((int64_t)s * c->H_kv + g) * c->max_blocks + j] += exp(lg);
            }
            if (N >= 1)
                logg[((int64_t)s * c->H_q + qh) * c->max_blocks + (N - 1)] = 0.0;
        }
    }
    free(u);
    free(qp);
    free(kg);
    free(pooled);
}

/* ------------------------------------------------------------------------ */
/* Selection                                                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    float s;
    int j;
} orc_key;

/* Rank: larger score first; equal scores (+0 == -0) by smaller index. */
static int cmp_key(const void *pa, const void *pb)
{
    const orc_key *a = (const orc_key *)pa, *b = (const orc_key *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return a->j - b->j;
}

static int cmp_int(const void *pa, const void *pb)
{
    return *(const int *)pa - *(const int *)pb;
}

/* Number of blocks one (sequence, group) selects [ReSA Key points]. */
int orc_num_selected(int N, int n_budget, int n_local, int n_min, int keep_num, int keep_den)
{
    if (N <= 0) return 0;
    int budget = n_budget;
    if (keep_den > 0)
        budget = (int)(((int64_t)N * keep_num + keep_den - 1) / keep_den);
    int L = n_local < N ? n_local : N;
    int n = budget;
    if (n_min > n) n = n_min;
    if (L > n) n = L;
    return n < N ? n : N;
}

/* Dynamic top-n with forced local blocks [ReSA Key points, Summary].
 * score [B][H_kv][max_blocks] (double; rounded to fp32 here, the precision in
 * which the ranking decision is taken).  n_local counts the forced most-recent
 * blocks; for the gate scorer the caller passes max(n_local, 1) so that the
 * current block B0 is always kept [SAS Method].  Writes ascending logical
 * indices to sel_idx [B][H_kv][n_max] and counts to sel_cnt [B][H_kv].
 * Returns 0, or -1 if some count exceeds n_max. */
int orc_select(const double *score, const int32_t *seq_lens, int B, int H_kv, int b,
               int max_blocks, int n_budget, int n_local, int n_min, int keep_num,
               int keep_den, int n_max, int32_t *sel_idx, int32_t *sel_cnt)
{
    orc_key *keys = (orc_key *)malloc(sizeof(orc_key) * (max_blocks > 0 ? max_blocks : 1));
    int *chosen = (int *)malloc(sizeof(int) * (max_blocks > 0 ? max_blocks : 1));
    int rc = 0;
    for (int s = 0; s < B; ++s) {
        int len = seq_lens[s];
        int N = len <= 0 ? 0 : (len + b - 1) / b;
        int n = orc_num_selected(N, n_budget, n_local, n_min, keep_num, keep_den);
        int L = n_local < N ? n_local : N;
        for (int g = 0; g < H_kv; ++g) {
            int cnt = 0;
            int ncand = N - L;
            for (int j = 0; j < ncand; ++j) {
                /* rounded to fp32; cmp_key's comparisons treat -0 == +0 */
                keys[j].s = (float)score[((int64_t)s * H_kv + g) * max_blocks + j];
                keys[j].j = j;
            }
            qsort(keys, (size_t)ncand, sizeof(orc_key), cmp_key);
            for (int i = 0; i < n - L; ++i)
                chosen[cnt++] = keys[i].j;
            for (int j = N - L; j < N; ++j)
                chosen[cnt++] = j;
            qsort(chosen, (size_t)cnt, sizeof(int), cmp_int);
            if (cnt > n_max) {
                rc = -1;
                cnt = n_max;
            }
            sel_cnt[s * H_kv + g] = cnt;
            for (int i = 0; i < cnt; ++i)
                sel_idx[((int64_t)s * H_kv + g) * n_max + i] = chosen[i];
        }
    }
    free(chosen);
    free(keys);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Attention over the selected blocks                                        */
/* ------------------------------------------------------------------------ */

/* Exact softmax attention restricted to the selected blocks [ReSA Summary:
 * group block-sparse attention; SAS Method: o = softmax(q K_S^T + log g_S) V_S].
 * For query head qh of group g and every token t < len of every selected block
 * j: l_t = (q.k_t)*scale + bias[qh][j]; out = sum_t softmax(l)_t v_t;
 * lse = log sum_t exp(l_t).  bias [B][H_q][max_blocks] indexed by logical block
 * (NULL = no gate).  out [B][H_q][d], lse [B][H_q]; an empty selection gives
 * out = 0 and lse = -inf. */
void orc_attend(const orc_cache *c, const uint16_t *q, const int32_t *sel_idx,
                const int32_t *sel_cnt, int n_max, const double *bias, double scale,
                double *out, double *lse)
{
    int d = c->d;
    int G = c->H_q / c->H_kv;
    int64_t cap = (int64_t)n_max * c->b;
    double *l = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
    int *tok = (int *)malloc(sizeof(int) * (cap > 0 ? cap : 1));
    for (int s = 0; s < c->B; ++s) {
        int len = c->seq_lens[s];
        for (int qh = 0; qh < c->H_q; ++qh) {
            int g = qh / G;
            const uint16_t *qv = q + ((int64_t)s * c->H_q + qh) * d;
            int cnt = sel_cnt[s * c->H_kv + g];
            int nt = 0;
            for (int i = 0; i < cnt; ++i) {
                int j = sel_idx[((int64_t)s * c->H_kv + g) * n_max + i];
                double bj = bias ? bias[((int64_t)s * c->H_q + qh) * c->max_blocks + j] : 0.0;
                for (int t = j * c->b; t < (j + 1) * c->b && t < len; ++t) {
                    double dot = 0.0;
                    for (int ch = 0; ch < d; ++ch)
                        dot += bf16_to_double(qv[ch]) * key_at(c, s, t, g, ch);
                    l[nt] = dot * scale + bj;
                    tok[nt] = t;
                    ++nt;
                }
            }
            double *o = out + ((int64_t)s * c->H_q + qh) * d;
            for (int ch = 0; ch < d; ++ch)
                o[ch] = 0.0;
            if (nt == 0) {
                lse[(int64_t)s * c->H_q + qh] = -INFINITY;
                continue;
            }
            double m = l[0];
            for (int i = 1; i < nt; ++i)
                if (l[i] > m) m = l[i];
            double z = 0.0;
            for (int i = 0; i < nt; ++i)
                z += exp(l[i] - m);
            for (int i = 0; i < nt; ++i) {
                double w = exp(l[i] - m) / z;
                for (int ch = 0; ch < d; ++ch)
                    o[ch] += w * val_at(c, s, tok[i], g, ch);
            }
            lse[(int64_t)s * c->H_q + qh] = m + log(z);
        }
    }
    free(tok);
    free(l);
}

/* Split-KV merge [Flash-Decoding, cited by ReSA]: partial outputs o_part
 * [B][H_q][S][d] with their log-sum-exps lse_part [B][H_q][S] combine as
 * out = sum_s w_s o_s, w_s = exp(lse_s - LSE), LSE = log sum_s exp(lse_s).
 * Splits with lse = -inf carry no weight; all -inf gives out = 0, LSE = -inf. */
void orc_combine(const double *o_part, const double *lse_part, int B, int H_q, int S, int d,
                 double *out, double *lse)
{
    for (int64_t r = 0; r < (int64_t)B * H_q; ++r) {
        double m = -INFINITY;
        for (int sp = 0; sp < S; ++sp)
            if (lse_part[r * S + sp] > m) m = lse_part[r * S + sp];
        for (int ch = 0; ch < d; ++ch)
            out[r * d + ch] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double z = 0.0;
        for (int sp = 0; sp < S; ++sp)
            z += exp(lse_part[r * S + sp] - m);
        for (int sp = 0; sp < S; ++sp) {
            double w = exp(lse_part[r * S + sp] - m) / z;
            if (w == 0.0) continue;
            for (int ch = 0; ch < d; ++ch)
                out[r * d + ch] += w * o_part[(r * S + sp) * d + ch];
        }
        lse[r] = m + log(z);
    }
}
