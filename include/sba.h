/*
 * sba.h -- C ABI of libsba.so: group-shared block-sparse attention for
 * single-token decode over a long (optionally paged) KV cache, on NVIDIA B200
 * (sm_100a).
 *
 * The method (page title, section):
 *  - "Rectified Sparse Attention for Efficient Long-Sequence Generation",
 *    Summary: Quest-style min/max block descriptors score the memory blocks,
 *    every query head of a GQA group shares one block selection, and attention
 *    runs over the selected blocks only ("group block-sparse attention").
 *    Key points: the top-n rule always keeps the recent local blocks and a
 *    minimum block count; the sparsity ratio p; per-step memory ~ 1/b + p + 1/f.
 *    References: Flash-Decoding (split-KV with a log-sum-exp merge), Quest,
 *    PagedAttention (block tables).
 *  - "SAS: Simple Attention Sparsification via End-to-End Optimization of
 *    Context Ranking", Method: gates g = softmax(s) over the historical
 *    blocks, the current block B0 keeps a unit gate, and
 *    o = softmax(q K_S^T + log g_S) V_S (the log-gate sits inside the softmax).
 *    Limitations: pooling-based block summaries feed the selector.
 *  - "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning",
 *    abstract: a plug-in gate scores blocks from the decode query (no query
 *    pooling); sparse decode kernel.
 *
 * Conventions shared by every call:
 *  - Pointers marked "device" point to device memory owned by the caller; the
 *    library never frees, keeps or reallocates them.  Scalars and the structs
 *    themselves live in host memory and are read before the call returns.
 *  - Every compute call enqueues kernels on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and returns without synchronising.  The calls
 *    allocate nothing and keep no state between calls except what the caller's
 *    workspace holds (see sba_score_select).
 *  - Return value: SBA_OK, or an SBA_ERR_* code when the arguments are
 *    rejected on the host (nothing is enqueued then) or a launch fails.
 *    Faults of already-enqueued kernels surface at the caller's next
 *    synchronisation, as usual for CUDA.  No C++ exception crosses the ABI.
 *  - The library remembers, per device, the kernel attributes it has set
 *    (shared-memory limits, cluster sizes).  A cudaDeviceReset discards them
 *    on the device; a process that resets a device reloads the library before
 *    using it there again (calls otherwise fail with SBA_ERR_CUDA).
 *  - Every softmax_scale argument must be positive and finite
 *    (SBA_ERR_INVALID_ARG otherwise).
 *  - Data-dependent problems found on the device (a block-table entry outside
 *    [0, num_pages), a position outside the table, a selected index outside
 *    [0, N), a wait that timed out) never trap: the offending access is
 *    skipped and an SBA_DEV_* bit is OR-ed into cache->status when that
 *    pointer is non-NULL.
 *
 * Notation: B sequences; H_q query heads; H_kv KV heads; G = H_q / H_kv query
 * heads per group (query head qh reads KV head qh / G); d = 128 head width;
 * b in {64, 128} tokens per block; len_s = seq_lens[s];
 * N_s = ceil(len_s / b) blocks in sequence s.
 */
#ifndef SBA_H
#define SBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side status codes. */
#define SBA_OK 0
#define SBA_ERR_INVALID_ARG 1  /* NULL where required, misaligned, inconsistent sizes */
#define SBA_ERR_UNSUPPORTED 2  /* d != 128, b not in {64,128}, G > 16, too many blocks */
#define SBA_ERR_WORKSPACE 3    /* workspace missing or smaller than sba_workspace_size() */
#define SBA_ERR_CUDA 4         /* a CUDA runtime call or launch failed */

/* Device-side status bits OR-ed into cache->status. */
#define SBA_DEV_BAD_PAGE 1       /* block-table entry outside [0, num_pages) */
#define SBA_DEV_BAD_POSITION 2   /* append/update position outside [0, max_blocks*b) */
#define SBA_DEV_BAD_SELECTION 4  /* selected index outside [0, N_s) or count > n_max */
#define SBA_DEV_TIMEOUT 8        /* a bounded wait inside a kernel ran out */

#define SBA_SCORER_QUEST 0
#define SBA_SCORER_GATE 1

#define SBA_OUT_F32 0
#define SBA_OUT_BF16 1

/* Where the gate enters the attention ("SAS ...", Method: the gate may sit
 * inside the softmax or outside it, on the values). */
#define SBA_LOG_GATE_OFF 0    /* the gates select blocks only: o = softmax(l) V */
#define SBA_LOG_GATE_INNER 1  /* o = softmax(l + log g) V (log g per selected block) */
#define SBA_LOG_GATE_OUTER 2  /* o = softmax(l) (g . V): each token's value times its block's gate */

/* Gate activation phi, g = phi(u) on the historical blocks ("SAS ...", Method
 * and its ablations: softmax, sigmoid and unnormalised logit injection). */
#define SBA_GATE_SOFTMAX 0  /* g = softmax of u over the C = N-1 historical blocks */
#define SBA_GATE_SIGMOID 1  /* g = 1 / (1 + exp(-u)), each block on its own */
#define SBA_GATE_RAW 2      /* unnormalised: log g = u (g = exp(u)) */

/* The KV cache of ONE attention layer, and its block descriptors.
 *
 * k, v          device, bf16 [num_pages][H_kv][b][d]: token t of sequence s
 *               lives in page P(s, t/b) at row t % b.  One (page, head) tile is
 *               b*d*2 contiguous bytes.  16-byte aligned.
 * block_table   device int32 [B][max_blocks]: P(s, j) = block_table[s][j]
 *               (PagedAttention-style).  NULL means contiguous pages,
 *               P(s, j) = s*max_blocks + j.  Entries past N_s are never read.
 * seq_lens      device int32 [B], 0 <= len_s <= max_blocks*b.
 * max_len       host upper bound of every len_s (grid sizing only).
 * desc          Quest descriptors, device bf16 [num_pages][H_kv][2][d]: row 0
 *               the per-channel MIN, row 1 the per-channel MAX of the block's
 *               valid keys ("Rectified Sparse Attention ...", Summary).  Indexed
 *               by physical page, so a descriptor moves with its page.  NULL if
 *               the layer uses the gate scorer only.
 * kg            gate keys, device fp32 [num_pages][H_kv][d]: the pooled block
 *               summary [max || min || avg] projected by the gate weights and
 *               already multiplied into query space (see sba_update_descriptors).
 *               NULL if the layer uses the Quest scorer only.
 * status        optional device int32 word for SBA_DEV_* bits (may be NULL).
 */
typedef struct sba_cache {
    void *k;
    void *v;
    const int32_t *block_table;
    const int32_t *seq_lens;
    int32_t B, H_q, H_kv, d, b, max_blocks, num_pages, max_len;
    void *desc;
    float *kg;
    int32_t *status;
} sba_cache;

/* Gate weights of one layer ("SeerAttention-R ...", abstract: a light plug-in
 * gate; "SAS ...", Method/Limitations: scores from pooled block summaries).
 * Wk  device fp32 [dg][3d] (row-major, no bias): pooled key -> gate key;
 * Wq  device fp32 [dg][d]  (row-major, no bias): query -> gate query;
 * dg  gate width (1..256).  Gate logit of block j for query head qh:
 * u = (Wq q).(Wk pooled_j) / sqrt(dg). */
typedef struct sba_gate {
    const float *Wq;
    const float *Wk;
    int32_t dg;
} sba_gate;

/* Selection rule ("Rectified Sparse Attention ...", Key points): every
 * (sequence, KV group) keeps n_sel = min(N, max(L, n_min, budget)) blocks, where
 * budget = n_budget, or ceil(N*keep_num/keep_den) when keep_den > 0 (sparsity
 * p = 1 - keep_num/keep_den); the L = min(n_local, N) most recent blocks
 * {N-L .. N-1} are always kept and the rest are the top scores of blocks
 * 0 .. N-L-1 (fp32 score descending, then index ascending; -0 == +0).
 * With the gate scorer the current block B0 = N-1 is always kept, i.e. L >= 1
 * ("SAS ...", Method).
 * Gate scorer only (ignored by Quest, where they must be 0):
 *  - gate_act: phi of the gates g = phi(u) (SBA_GATE_*).  The group ranks the
 *    historical blocks by sum over its heads of g; the log-gate of a selected
 *    historical block is log g, and 0 for B0 (unit gate).  With
 *    SBA_GATE_RAW, exp(u) must stay finite in fp32 (u < 88).
 *  - log_gate: whether and where the gate enters the attention of
 *    sba_decode_step (SBA_LOG_GATE_*).  The split-KV calls take the choice
 *    through which decode call is made (see sba_sparse_decode). */
typedef struct sba_select_params {
    int32_t n_budget;
    int32_t n_local;
    int32_t n_min;
    int32_t keep_num;
    int32_t keep_den;
    int32_t scorer;   /* SBA_SCORER_QUEST or SBA_SCORER_GATE */
    int32_t log_gate; /* SBA_LOG_GATE_OFF, _INNER or _OUTER */
    int32_t gate_act; /* SBA_GATE_SOFTMAX, _SIGMOID or _RAW */
} sba_select_params;

/* Message for a status code (static string, never NULL). */
const char *sba_status_string(int status);

/* Text of the last CUDA error a call of this thread returned SBA_ERR_CUDA for
 * ("no error" if none); static string, never NULL. */
const char *sba_last_cuda_error(void);

/* Self-test of the bounded waits every kernel uses (failure detection without
 * a fault): one warp waits, with the library's own bounded mbarrier wait limited
 * to limit_ns, on a barrier that nothing arrives on; the wait runs out, ORs
 * SBA_DEV_TIMEOUT into *status (device int32) and the kernel returns, leaving
 * the context usable.  0 < limit_ns <= 10 s (SBA_ERR_INVALID_ARG otherwise, or
 * for a NULL status).  The kernels' own waits give up after about 2 s. */
int sba_selftest_wait_timeout(int32_t *status, uint64_t limit_ns, void *stream);

/* Host helper: blocks selected for a sequence of N blocks under `p` (the rule
 * above).  Returns -1 if p is NULL. */
int32_t sba_num_selected(int32_t N, const sba_select_params *p);

/* Host helper: ceil(N * keep_num / keep_den) in integer arithmetic (the
 * sparsity-ratio budget; p = 0.95 on 2048 blocks gives 103). */
int32_t sba_budget_from_sparsity(int32_t N, int32_t keep_num, int32_t keep_den);

/* Host helper: a split count for sba_sparse_decode that fills the GPU with one
 * wave of CTAs for this cache shape and selection size (n_max blocks per
 * group).  `num_sms` is the device's multiprocessor count. */
int32_t sba_default_num_splits(const sba_cache *c, int32_t n_max, int32_t num_sms);

/* Bytes of workspace sba_score_select needs for this cache and scorer. */
size_t sba_workspace_size(const sba_cache *c, const sba_select_params *p);

/* Append: write n_new tokens per sequence into the cache
 * ("Rectified Sparse Attention ...", Summary: KV entries are written as tokens
 * are generated and overwritten when a window is re-encoded).
 * k_new, v_new  device bf16 [B][n_new][H_kv][d];
 * pos_start     device int32 [B]: token i goes to position pos_start[s] + i.
 * Overwriting existing positions is allowed.  Does not change seq_lens: the
 * caller advances it, then calls sba_update_descriptors. */
int sba_append_kv(const sba_cache *c, const void *k_new, const void *v_new,
                  const int32_t *pos_start, int32_t n_new, void *stream);

/* Descriptor update: for every sequence s, recompute the descriptors of every
 * block that overlaps positions [pos_start[s], pos_start[s] + n_new) and lies
 * below N_s, from ALL of that block's valid tokens (recomputing, not folding in
 * the new keys, keeps overwrites correct).
 *  - Quest (when c->desc != NULL): per channel min and max, exact in bf16.
 *  - Gate (when gate != NULL and c->kg != NULL): pooled = [max || min || avg]
 *    (3d, fp32), k' = Wk pooled (dg), and the stored gate key
 *    kg = Wq^T k' / sqrt(dg) (d), so that the gate logit of a query head is
 *    u = q . kg.  Folding Wq into the stored key is exact algebra
 *    ((Wq q).k' = q.(Wq^T k')) and removes the per-step query projection.
 * To fill a fresh cache call it once with pos_start = 0, n_new = max_len. */
int sba_update_descriptors(const sba_cache *c, const int32_t *pos_start, int32_t n_new,
                           const sba_gate *gate, void *stream);

/* Score every block and select the shared top-n set of each (sequence, KV group).
 *  - Quest ("Rectified Sparse Attention ...", Summary): score of block j for
 *    group g = sum over the group's query heads qh of
 *    sum_c max(q_qh,c * min_jc, q_qh,c * max_jc), an upper bound of
 *    max_t q.k_t over the block, in fp32.
 *  - Gate ("SAS ...", Method): u_qh,j = q_qh . kg_j over the historical blocks
 *    j < N-1, g = phi(u) with phi = p->gate_act (softmax over j by default),
 *    score = sum over the group of g.  When gate_bias != NULL it receives
 *    log g_qh,j (softmax: u_qh,j - logsumexp_j(u_qh); sigmoid: log sigmoid(u);
 *    raw: u) for every selected historical block and 0 for B0 = N-1.
 * q          device bf16 [B][H_q][d].
 * sel_idx    device int32 [B][H_kv][n_max]: selected logical block indices,
 *            ascending; entries past sel_cnt are left unchanged.
 * sel_cnt    device int32 [B][H_kv].
 * gate_bias  device fp32 [B][H_q][n_max] aligned with sel_idx, or NULL.
 * n_max      must be >= the largest n_sel any sequence can reach (host check
 *            against max_len).
 * ws         device workspace of at least sba_workspace_size() bytes, 16-byte
 *            aligned, ZERO-FILLED before its first use; every completed call
 *            leaves its counters at zero again, so the same workspace is reused
 *            as is.  Calls that share a workspace must not run concurrently. */
int sba_score_select(const sba_cache *c, const void *q, const sba_select_params *p,
                     int32_t *sel_idx, int32_t *sel_cnt, float *gate_bias, int32_t n_max,
                     void *ws, size_t ws_bytes, void *stream);

/* Split-KV sparse decode ("Rectified Sparse Attention ...", Summary: group
 * block-sparse attention; References: Flash-Decoding).  For every sequence s,
 * KV head h and split sp, over its share of the selected blocks
 * (sel_idx[s][h][i] for i in [cnt*sp/S, cnt*(sp+1)/S)) and for every query head
 * qh of the group: logits l_t = (q_qh . k_t) * softmax_scale + bias (bias =
 * gate_bias[s][qh][i] when gate_bias != NULL, "SAS ...", Method), tokens
 * t >= len_s masked; writes
 *   o_part[s][qh][sp][:] = sum_t softmax(l)_t v_t   (fp32, device [B][H_q][S][d])
 *   lse_part[s][qh][sp]  = log sum_t exp(l_t)       (fp32, device [B][H_q][S];
 *                                                    -inf for an empty split).
 * num_splits S >= 1 (sba_default_num_splits gives a good value). */
int sba_sparse_decode(const sba_cache *c, const void *q, const int32_t *sel_idx,
                      const int32_t *sel_cnt, const float *gate_bias, int32_t n_max,
                      float softmax_scale, int32_t num_splits, float *o_part, float *lse_part,
                      void *stream);

/* sba_sparse_decode with the gate OUTSIDE the softmax ("SAS ...", Method: the
 * gate may scale the values instead of entering the logits).  Same arguments;
 * gate_bias (log g, as sba_score_select writes it) is required.  Per split:
 *   o_part = sum_t softmax(l)_t g_j(t) v_t,  l_t = (q . k_t) * softmax_scale,
 *   lse_part = log sum_t exp(l_t)  (the ungated logits),
 * so sba_combine of the splits gives o = softmax(q K^T * scale) (g . V). */
int sba_sparse_decode_outer(const sba_cache *c, const void *q, const int32_t *sel_idx,
                            const int32_t *sel_cnt, const float *gate_bias, int32_t n_max,
                            float softmax_scale, int32_t num_splits, float *o_part,
                            float *lse_part, void *stream);

/* Log-sum-exp merge of the splits (Flash-Decoding, cited by "Rectified Sparse
 * Attention ...", References): out = sum_s w_s o_s with
 * w_s = exp(lse_s - LSE), LSE = log sum_s exp(lse_s).  All splits -inf gives
 * out = 0 and LSE = -inf.
 * o_part fp32 [B][H_q][S][d], lse_part fp32 [B][H_q][S] (device);
 * out device [B][H_q][d] in out_dtype (SBA_OUT_F32 or SBA_OUT_BF16);
 * lse_out device fp32 [B][H_q] or NULL. */
int sba_combine(const float *o_part, const float *lse_part, int32_t B, int32_t H_q,
                int32_t num_splits, int32_t d, void *out, int32_t out_dtype, float *lse_out,
                void *stream);

/* Several query tokens per sequence sharing one selection ("Rectified Sparse
 * Attention ...", Summary: the f tokens re-encoded together, every query head
 * of a GQA group sharing one block selection; Key points: the comparison with
 * self-speculative decoding, which checks several draft tokens at once).
 * The M query tokens of sequence s sit at its last M positions, len_s-M ..
 * len_s-1 (their keys and values already in the cache), and token i attends
 * causally to positions t <= len_s-M+i.  Quest scorer only.
 *
 * sba_score_select_multi: as sba_score_select, with the Quest score of a block
 * summed over the group's G heads AND the M tokens (the M*G query rows act as
 * one group); one selection per (sequence, KV group).
 * q  device bf16 [B][M][H_q][d].  Other arguments as sba_score_select. */
int sba_score_select_multi(const sba_cache *c, const void *q, int32_t M, const sba_select_params *p,
                           int32_t *sel_idx, int32_t *sel_cnt, int32_t n_max, void *ws, size_t ws_bytes,
                           void *stream);

/* sba_sparse_decode for M query tokens: every query row (token i, head qh)
 * attends over the group's selected blocks, masked causally (t <= len-M+i) and
 * at len.  Writes o_part fp32 [B][M][H_q][S][d] and lse_part [B][M][H_q][S]
 * (-inf for a row that saw no token), so sba_combine with H_q' = M*H_q merges
 * the splits into [B][M][H_q][d].  The M*G rows of a group run in row groups
 * of 128 (sba_multi_row_groups), each a CTA per split: choose num_splits so
 * that B*H_kv*row_groups*num_splits fills the GPU.  From M*G >= 64 rows the
 * call runs on the tcgen05 tensor cores (the rectification pipeline walking the
 * selection), below that on mma.sync; both give the same results within the
 * output tolerance. */
int sba_sparse_decode_multi(const sba_cache *c, const void *q, int32_t M, const int32_t *sel_idx,
                            const int32_t *sel_cnt, int32_t n_max, float softmax_scale,
                            int32_t num_splits, float *o_part, float *lse_part, void *stream);

/* Row groups (CTAs per split and KV head) of the multi-token calls: ceil(M*G/128). */
int32_t sba_multi_row_groups(const sba_cache *c, int32_t M);

/* The rectification pass ("Rectified Sparse Attention ...", Summary: every f
 * generated tokens are re-encoded in one parallel dense pass that rewrites
 * their KV entries, which bounds the error the sparse steps accumulate; Key
 * points: f in {16, 32, 64, 128}).  The caller has already advanced seq_lens
 * to include the f tokens, which sit at positions len_s-f .. len_s-1.  One
 * launch:
 *  1. writes k_new, v_new (device bf16 [B][f][H_kv][d]) at those positions
 *     through the block table, overwriting what the sparse steps stored;
 *  2. recomputes the Quest descriptors (c->desc, when non-NULL) of the blocks
 *     those positions touch, from all of each block's valid keys;
 *  3. dense causal attention of the f query tokens (q [B][f][H_q][d]) over
 *     every block [0, N): outputs as sba_sparse_decode_multi with M = f.
 * 1 <= f <= 128 and f <= len_s (a shorter sequence reports
 * SBA_DEV_BAD_POSITION).  Gate keys are not refreshed here (call
 * sba_update_descriptors for them). */
int sba_rectify(const sba_cache *c, const void *q, const void *k_new, const void *v_new, int32_t f,
                float softmax_scale, int32_t num_splits, float *o_part, float *lse_part, void *stream);

/* Size in bytes of the static scratch behind sba_score_select_static (8 MiB). */
size_t sba_static_scratch_bytes(void);

/* sba_score_select for callers that cannot allocate device memory when they
 * issue a step: an engine that records its step into a CUDA graph and forbids
 * cudaMalloc during capture, a serving-framework plugin whose enqueue callback
 * must not allocate, an embedded runtime with a device-memory budget fixed at
 * start-up.  No counterpart on the pages: it is a deployment convenience.
 * Same arguments, semantics and outputs as sba_score_select, without ws and
 * ws_bytes: the scratch is one static device array of
 * sba_static_scratch_bytes() bytes that the library reserves on every GPU that
 * loads it, until the process exits.
 *  - A problem needing more scratch than that (sba_workspace_size) returns
 *    SBA_ERR_WORKSPACE before anything is enqueued.
 *  - The first call on a device looks the array's address up for that device
 *    (and again when the device's context has changed, e.g. after
 *    cudaDeviceReset); make it before any stream capture.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents; each call first clears the completion counters on `stream`
 *    (cudaMemsetAsync).  Calls whose kernels can overlap on the GPU (streams
 *    with no ordering between them) race on the array.
 *  - Calls no allocating routine (cudaMalloc, cudaFree, library allocators). */
int sba_score_select_static(const sba_cache *c, const void *q, const sba_select_params *p, int32_t *sel_idx,
                            int32_t *sel_cnt, float *gate_bias, int32_t n_max, void *stream);

/* Fold the gate projection into query space once per layer:
 * A = Wq^T Wk / sqrt(dg), device fp32 [d][3d] (row-major), so that the stored
 * gate key of a block is kg = A pooled and its gate logit for a query head is
 * u = q . kg ("SAS ...", Method; "SeerAttention-R ...", abstract).  Used by
 * sba_decode_step. */
int sba_fold_gate(const sba_gate *gate, float *A, void *stream);

/* Cluster size (CTAs per sequence and KV group) that sba_decode_step uses on
 * the current device for this cache shape and rule: the largest C <= 16 with
 * B * H_kv * C <= the SM count whose clusters are all resident at once (one
 * CTA per SM), else the largest C the device can schedule.  Remembered per
 * device and shape.  Sets kernel attributes, launches nothing; 0 if the shape
 * is not supported by the fused step or no device is present. */
int32_t sba_decode_step_cluster(const sba_cache *c, const sba_select_params *p);

/* One whole decode step of one layer in ONE launch: rows a1-a6 fused.
 * 1. append n_new tokens per sequence at pos_start[s] (as sba_append_kv;
 *    n_new = 0 skips steps 1-2, pos_start may then be NULL);
 * 2. recompute the descriptors of the blocks those tokens touch (as
 *    sba_update_descriptors; the gate path uses the folded gate_A);
 * 3-4. score and select exactly as sba_score_select;
 * 5-6. attention over the selected blocks and the merge, as sba_sparse_decode
 *    followed by sba_combine, writing out [B][H_q][d] (SBA_OUT_F32 or
 *    SBA_OUT_BF16) and lse_out [B][H_q] (fp32, may be NULL).  With the gate
 *    scorer, p->log_gate places the gate: off (selection only), inside the
 *    softmax (as sba_sparse_decode with gate_bias) or on the values (as
 *    sba_sparse_decode_outer).
 * sel_idx/sel_cnt/gate_bias (layouts of sba_score_select, each may be NULL)
 * report the selection; n_max is their row length.
 * The caller advances seq_lens to include the appended tokens BEFORE the call.
 * Each (sequence, KV head) runs on one thread-block cluster of up to 16 CTAs
 * (one per SM); scores, the selection and the partial outputs stay in (shared
 * and distributed shared) memory, so the call needs no workspace.  A step whose
 * appended tokens touch a block it also scores (e.g. n_local = 0) refreshes
 * that block before scoring, at the cost of one extra cluster barrier. */
int sba_decode_step(const sba_cache *c, const void *q, const void *k_new, const void *v_new,
                    const int32_t *pos_start, int32_t n_new, const float *gate_A,
                    const sba_select_params *p, float softmax_scale, void *out, int32_t out_dtype,
                    float *lse_out, int32_t *sel_idx, int32_t *sel_cnt, float *gate_bias, int32_t n_max,
                    void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SBA_H */
