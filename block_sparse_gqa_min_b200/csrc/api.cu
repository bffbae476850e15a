// extern "C" entry points of libsba.so: argument validation on the host, then
// the kernel launches of the other files.  Nothing here allocates, keeps state
// or synchronises.
#include <stdint.h>

#include "common.cuh"
#include "launch.cuh"

using namespace sba;

namespace sba {
namespace {
thread_local cudaError_t g_last = cudaSuccess;
}
void note_cuda_error(cudaError_t e) { g_last = e; }
cudaError_t last_cuda_error() { return g_last; }
}  // namespace sba

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by every call that takes a cache.
int check_cache(const sba_cache* c) {
    if (!c || !c->k || !c->v || !c->seq_lens) return SBA_ERR_INVALID_ARG;
    if (!aligned16(c->k) || !aligned16(c->v)) return SBA_ERR_INVALID_ARG;
    if (c->B < 1 || c->H_kv < 1 || c->H_q < 1 || c->H_q % c->H_kv != 0) return SBA_ERR_INVALID_ARG;
    if (c->max_blocks < 1 || c->num_pages < 1 || c->max_len < 0) return SBA_ERR_INVALID_ARG;
    if (c->d != kHeadDim) return SBA_ERR_UNSUPPORTED;
    if (c->b != 64 && c->b != 128) return SBA_ERR_UNSUPPORTED;
    if (c->H_q / c->H_kv > kMaxGroup) return SBA_ERR_UNSUPPORTED;
    if (c->max_blocks > kMaxBlocksPerSeq) return SBA_ERR_UNSUPPORTED;
    if ((int64_t)c->max_len > (int64_t)c->max_blocks * c->b) return SBA_ERR_INVALID_ARG;
    if (!c->block_table && (int64_t)c->num_pages < (int64_t)c->B * c->max_blocks) return SBA_ERR_INVALID_ARG;
    // TMA row coordinates are signed 32-bit
    if ((int64_t)c->num_pages * c->H_kv * c->b >= (int64_t)1 << 31) return SBA_ERR_UNSUPPORTED;
    if (c->desc && !aligned16(c->desc)) return SBA_ERR_INVALID_ARG;
    if (c->kg && !aligned16(c->kg)) return SBA_ERR_INVALID_ARG;
    return SBA_OK;
}

int check_params(const sba_select_params* p) {
    if (!p) return SBA_ERR_INVALID_ARG;
    if (p->n_budget < 0 || p->n_local < 0 || p->n_min < 0) return SBA_ERR_INVALID_ARG;
    if (p->keep_den < 0 || p->keep_num < 0 || (p->keep_den > 0 && p->keep_num > p->keep_den))
        return SBA_ERR_INVALID_ARG;
    if (p->scorer != SBA_SCORER_QUEST && p->scorer != SBA_SCORER_GATE) return SBA_ERR_INVALID_ARG;
    if (p->log_gate < SBA_LOG_GATE_OFF || p->log_gate > SBA_LOG_GATE_OUTER) return SBA_ERR_INVALID_ARG;
    if (p->gate_act < SBA_GATE_SOFTMAX || p->gate_act > SBA_GATE_RAW) return SBA_ERR_INVALID_ARG;
    if (p->scorer == SBA_SCORER_QUEST && (p->log_gate != 0 || p->gate_act != 0)) return SBA_ERR_INVALID_ARG;
    return SBA_OK;
}

}  // namespace

namespace sba {
// Every host-side check of sba_score_select except the workspace (also used by the
// allocation-free variant, which must reject a call before it enqueues anything).
int check_score_select(const sba_cache* c, const void* q, const sba_select_params* p, const int32_t* sel_idx,
                       const int32_t* sel_cnt, int32_t n_max) {
    int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    rc = check_params(p);
    if (rc != SBA_OK) return rc;
    if (!q || !sel_idx || !sel_cnt || n_max < 1 || !aligned16(q)) return SBA_ERR_INVALID_ARG;
    if (p->scorer == SBA_SCORER_QUEST && !c->desc) return SBA_ERR_INVALID_ARG;
    if (p->scorer == SBA_SCORER_GATE && !c->kg) return SBA_ERR_INVALID_ARG;
    const int n_need = num_selected((c->max_len + c->b - 1) / c->b, *p);
    if (n_max < n_need) return SBA_ERR_INVALID_ARG;
    return SBA_OK;
}
}  // namespace sba

namespace {

int after_launch(int rc) {
    if (rc != SBA_OK) return rc;
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return SBA_OK;
    note_cuda_error(e);
    return SBA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* sba_status_string(int status) {
    switch (status) {
        case SBA_OK: return "ok";
        case SBA_ERR_INVALID_ARG: return "invalid argument (null, misaligned or inconsistent sizes)";
        case SBA_ERR_UNSUPPORTED: return "unsupported shape (d must be 128, b 64 or 128, G <= 16)";
        case SBA_ERR_WORKSPACE: return "workspace missing or too small";
        case SBA_ERR_CUDA: return "CUDA launch or runtime error";
        default: return "unknown status";
    }
}

const char* sba_last_cuda_error(void) {
    const cudaError_t e = last_cuda_error();
    return e == cudaSuccess ? "no error" : cudaGetErrorString(e);
}

int sba_selftest_wait_timeout(int32_t* status, uint64_t limit_ns, void* stream) {
    if (!status || limit_ns == 0 || limit_ns > 10000000000ull) return SBA_ERR_INVALID_ARG;
    return after_launch(launch_wait_timeout_selftest(status, limit_ns, static_cast<cudaStream_t>(stream)));
}

int32_t sba_num_selected(int32_t N, const sba_select_params* p) {
    if (!p) return -1;
    return num_selected(N, *p);
}

int32_t sba_budget_from_sparsity(int32_t N, int32_t keep_num, int32_t keep_den) {
    if (keep_den <= 0 || N <= 0 || keep_num < 0) return 0;
    return (int32_t)(((int64_t)N * keep_num + keep_den - 1) / keep_den);
}

int32_t sba_default_num_splits(const sba_cache* c, int32_t n_max, int32_t num_sms) {
    if (!c || c->B < 1 || c->H_kv < 1 || n_max < 1) return 1;
    if (num_sms < 1) num_sms = 148;
    const int64_t units = (int64_t)c->B * c->H_kv;
    int64_t s = num_sms / units;  // one wave of one-CTA-per-SM decode CTAs
    if (s < 1) s = 1;
    if (s > n_max) s = n_max;
    return (int32_t)s;
}

size_t sba_workspace_size(const sba_cache* c, const sba_select_params* p) {
    if (check_cache(c) != SBA_OK || check_params(p) != SBA_OK) return 0;
    return score_workspace_bytes(*c, *p);
}

int sba_append_kv(const sba_cache* c, const void* k_new, const void* v_new, const int32_t* pos_start, int32_t n_new,
                  void* stream) {
    int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    if (!k_new || !v_new || !pos_start || n_new < 0) return SBA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new)) return SBA_ERR_INVALID_ARG;
    if (n_new == 0) return SBA_OK;
    return after_launch(launch_append_kv(*c, k_new, v_new, pos_start, n_new, static_cast<cudaStream_t>(stream)));
}

int sba_update_descriptors(const sba_cache* c, const int32_t* pos_start, int32_t n_new, const sba_gate* gate,
                           void* stream) {
    int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    if (!pos_start || n_new < 0) return SBA_ERR_INVALID_ARG;
    if (gate && (!gate->Wq || !gate->Wk || gate->dg < 1 || gate->dg > 256 || !c->kg)) return SBA_ERR_INVALID_ARG;
    if (!c->desc && !gate) return SBA_ERR_INVALID_ARG;
    if (n_new == 0) return SBA_OK;
    return after_launch(launch_update_descriptors(*c, pos_start, n_new, gate, static_cast<cudaStream_t>(stream)));
}

int sba_score_select(const sba_cache* c, const void* q, const sba_select_params* p, int32_t* sel_idx,
                     int32_t* sel_cnt, float* gate_bias, int32_t n_max, void* ws, size_t ws_bytes, void* stream) {
    const int rc = check_score_select(c, q, p, sel_idx, sel_cnt, n_max);
    if (rc != SBA_OK) return rc;
    if (!ws || !aligned16(ws) || ws_bytes < score_workspace_bytes(*c, *p)) return SBA_ERR_WORKSPACE;
    return after_launch(launch_score_select(*c, q, 1, *p, sel_idx, sel_cnt, p->scorer == SBA_SCORER_GATE ? gate_bias : nullptr,
                                            n_max, ws, static_cast<cudaStream_t>(stream)));
}

// a softmax scale is positive and finite
static bool good_scale(float s) { return s > 0.f && s <= 3.4028234e38f; }

static int sparse_decode_any(const sba_cache* c, const void* q, const int32_t* sel_idx, const int32_t* sel_cnt,
                             const float* gate_bias, int32_t n_max, float softmax_scale, int32_t num_splits,
                             float* o_part, float* lse_part, bool outer, void* stream) {
    int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    if (!q || !sel_idx || !sel_cnt || !o_part || !lse_part || n_max < 1) return SBA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_part)) return SBA_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 65535) return SBA_ERR_INVALID_ARG;
    if (!good_scale(softmax_scale)) return SBA_ERR_INVALID_ARG;
    if (outer && !gate_bias) return SBA_ERR_INVALID_ARG;
    return after_launch(launch_sparse_decode(*c, q, sel_idx, sel_cnt, gate_bias, n_max, softmax_scale, num_splits,
                                             o_part, lse_part, outer, static_cast<cudaStream_t>(stream)));
}

int sba_sparse_decode(const sba_cache* c, const void* q, const int32_t* sel_idx, const int32_t* sel_cnt,
                      const float* gate_bias, int32_t n_max, float softmax_scale, int32_t num_splits, float* o_part,
                      float* lse_part, void* stream) {
    return sparse_decode_any(c, q, sel_idx, sel_cnt, gate_bias, n_max, softmax_scale, num_splits, o_part, lse_part,
                             false, stream);
}

int sba_sparse_decode_outer(const sba_cache* c, const void* q, const int32_t* sel_idx, const int32_t* sel_cnt,
                            const float* gate_bias, int32_t n_max, float softmax_scale, int32_t num_splits,
                            float* o_part, float* lse_part, void* stream) {
    return sparse_decode_any(c, q, sel_idx, sel_cnt, gate_bias, n_max, softmax_scale, num_splits, o_part, lse_part,
                             true, stream);
}

int sba_score_select_multi(const sba_cache* c, const void* q, int32_t M, const sba_select_params* p,
                           int32_t* sel_idx, int32_t* sel_cnt, int32_t n_max, void* ws, size_t ws_bytes,
                           void* stream) {
    const int rc = check_score_select(c, q, p, sel_idx, sel_cnt, n_max);
    if (rc != SBA_OK) return rc;
    if (M < 1 || M > kMaxQueryTokens) return SBA_ERR_INVALID_ARG;
    if (p->scorer != SBA_SCORER_QUEST) return SBA_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws) || ws_bytes < score_workspace_bytes(*c, *p)) return SBA_ERR_WORKSPACE;
    return after_launch(launch_score_select(*c, q, M, *p, sel_idx, sel_cnt, nullptr, n_max, ws,
                                            static_cast<cudaStream_t>(stream)));
}

static int check_multi(const sba_cache* c, const void* q, int32_t M, float softmax_scale, int32_t num_splits,
                       const float* o_part, const float* lse_part) {
    const int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    if (!q || !o_part || !lse_part || !aligned16(q)) return SBA_ERR_INVALID_ARG;
    if (M < 1 || M > kMaxQueryTokens) return SBA_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 65535) return SBA_ERR_INVALID_ARG;
    if (!good_scale(softmax_scale)) return SBA_ERR_INVALID_ARG;
    if ((int64_t)c->H_kv * mq_row_groups(*c, M) > 65535 || c->B > 65535) return SBA_ERR_UNSUPPORTED;
    return SBA_OK;
}

int32_t sba_multi_row_groups(const sba_cache* c, int32_t M) {
    if (check_cache(c) != SBA_OK || M < 1) return 0;
    return mq_row_groups(*c, M);
}

int sba_sparse_decode_multi(const sba_cache* c, const void* q, int32_t M, const int32_t* sel_idx,
                            const int32_t* sel_cnt, int32_t n_max, float softmax_scale, int32_t num_splits,
                            float* o_part, float* lse_part, void* stream) {
    const int rc = check_multi(c, q, M, softmax_scale, num_splits, o_part, lse_part);
    if (rc != SBA_OK) return rc;
    if (!sel_idx || !sel_cnt || n_max < 1) return SBA_ERR_INVALID_ARG;
    return after_launch(launch_multi_query(*c, q, M, sel_idx, sel_cnt, n_max, softmax_scale, num_splits, o_part, lse_part,
                                           static_cast<cudaStream_t>(stream)));
}

int sba_rectify(const sba_cache* c, const void* q, const void* k_new, const void* v_new, int32_t f,
                float softmax_scale, int32_t num_splits, float* o_part, float* lse_part, void* stream) {
    const int rc = check_multi(c, q, f, softmax_scale, num_splits, o_part, lse_part);
    if (rc != SBA_OK) return rc;
    if (f > kMaxRectifyTokens) return SBA_ERR_UNSUPPORTED;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SBA_ERR_INVALID_ARG;
    return after_launch(launch_rectify_tc(*c, q, f, k_new, v_new, softmax_scale, num_splits, o_part, lse_part,
                                          static_cast<cudaStream_t>(stream)));
}

int sba_combine(const float* o_part, const float* lse_part, int32_t B, int32_t H_q, int32_t num_splits, int32_t d,
                void* out, int32_t out_dtype, float* lse_out, void* stream) {
    if (!o_part || !lse_part || !out || B < 1 || H_q < 1 || num_splits < 1) return SBA_ERR_INVALID_ARG;
    if (d != kHeadDim) return SBA_ERR_UNSUPPORTED;
    if (out_dtype != SBA_OUT_F32 && out_dtype != SBA_OUT_BF16) return SBA_ERR_INVALID_ARG;
    if (B > 65535) return SBA_ERR_UNSUPPORTED;
    return after_launch(launch_combine(o_part, lse_part, B, H_q, num_splits, out, out_dtype, lse_out,
                                       static_cast<cudaStream_t>(stream)));
}

int sba_fold_gate(const sba_gate* g, float* A, void* stream) {
    if (!g || !g->Wq || !g->Wk || !A || g->dg < 1 || g->dg > 256) return SBA_ERR_INVALID_ARG;
    return after_launch(launch_fold_gate(g->Wq, g->Wk, g->dg, A, static_cast<cudaStream_t>(stream)));
}

int32_t sba_decode_step_cluster(const sba_cache* c, const sba_select_params* p) {
    if (check_cache(c) != SBA_OK || check_params(p) != SBA_OK) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return step_cluster_size(*c, *p, sms);
}

int sba_decode_step(const sba_cache* c, const void* q, const void* k_new, const void* v_new, const int32_t* pos_start,
                    int32_t n_new, const float* gate_A, const sba_select_params* p, float softmax_scale, void* out,
                    int32_t out_dtype, float* lse_out, int32_t* sel_idx, int32_t* sel_cnt, float* gate_bias,
                    int32_t n_max, void* stream) {
    int rc = check_cache(c);
    if (rc != SBA_OK) return rc;
    rc = check_params(p);
    if (rc != SBA_OK) return rc;
    if (!q || !out || !aligned16(q) || n_new < 0) return SBA_ERR_INVALID_ARG;
    if (out_dtype != SBA_OUT_F32 && out_dtype != SBA_OUT_BF16) return SBA_ERR_INVALID_ARG;
    if (!good_scale(softmax_scale)) return SBA_ERR_INVALID_ARG;
    if (n_new > 0 && (!k_new || !v_new || !pos_start || !aligned16(k_new) || !aligned16(v_new)))
        return SBA_ERR_INVALID_ARG;
    if (p->scorer == SBA_SCORER_QUEST && !c->desc) return SBA_ERR_INVALID_ARG;
    if (p->scorer == SBA_SCORER_GATE && (!c->kg || !gate_A)) return SBA_ERR_INVALID_ARG;
    const int n_need = num_selected((c->max_len + c->b - 1) / c->b, *p);
    if ((sel_idx || gate_bias) && n_max < n_need) return SBA_ERR_INVALID_ARG;
    if (c->B > 65535 || c->H_kv > 65535) return SBA_ERR_UNSUPPORTED;
    const int C = sba_decode_step_cluster(c, p);
    if (C < 1) return SBA_ERR_UNSUPPORTED;
    return after_launch(launch_decode_step(*c, q, k_new, v_new, pos_start, n_new, gate_A, *p, softmax_scale, out,
                                           out_dtype, lse_out, sel_idx, sel_cnt,
                                           p->scorer == SBA_SCORER_GATE ? gate_bias : nullptr, n_max, C,
                                           static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
