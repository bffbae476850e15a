// Kernel launch helper: every libsba kernel is launched with programmatic
// dependent launch enabled, so that it is scheduled while the previous kernel
// in the stream drains; each kernel calls griddepcontrol.wait before it reads
// anything a previous kernel may write.  SBA_PDL=0 in the environment turns
// the attribute off (plain stream order).
#pragma once

#include <cuda_runtime.h>
#include <stdlib.h>

#include "../../include/sba.h"

namespace sba {

inline bool pdl_enabled() {
    static const bool on = [] {
        const char* e = getenv("SBA_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

// Record the last CUDA error of a library call (for sba_last_cuda_error).
void note_cuda_error(cudaError_t e);

// Raise a kernel's dynamic shared-memory limit to `bytes` when the current
// limit is lower (not a stream operation, so it is safe during capture).
template <auto Kernel>
int allow_smem(int bytes) {
    static int allowed[64] = {};  // per device, per kernel instantiation
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    if (bytes <= 48 * 1024 || bytes <= allowed[dev]) return SBA_OK;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    allowed[dev] = bytes;
    return SBA_OK;
}

template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args&&... args) {
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return SBA_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    return SBA_OK;
}

// Host-side argument checks of sba_score_select, short of the workspace (api.cu).
int check_score_select(const sba_cache* c, const void* q, const sba_select_params* p, const int32_t* sel_idx,
                       const int32_t* sel_cnt, int32_t n_max);

// Host-side entry points of the kernel files (validated arguments only).
int launch_append_kv(const sba_cache& c, const void* k_new, const void* v_new, const int32_t* pos_start, int n_new,
                     cudaStream_t stream);
int launch_update_descriptors(const sba_cache& c, const int32_t* pos_start, int n_new, const sba_gate* gate,
                              cudaStream_t stream);
int score_chunk_blocks(const sba_cache& c);
size_t score_workspace_bytes(const sba_cache& c, const sba_select_params& p);
int launch_score_select(const sba_cache& c, const void* q, int M, const sba_select_params& p, int32_t* sel_idx,
                        int32_t* sel_cnt, float* gate_bias, int n_max, void* ws, cudaStream_t stream);
int launch_sparse_decode(const sba_cache& c, const void* q, const int32_t* sel_idx, const int32_t* sel_cnt,
                         const float* gate_bias, int n_max, float scale, int num_splits, float* o_part,
                         float* lse_part, bool outer, cudaStream_t stream);
int step_cluster_size(const sba_cache& c, const sba_select_params& p, int num_sms);
int launch_decode_step(const sba_cache& c, const void* q, const void* k_new, const void* v_new,
                       const int32_t* pos_start, int n_new, const float* gate_A, const sba_select_params& p,
                       float scale, void* out, int out_dtype, float* lse_out, int32_t* sel_idx, int32_t* sel_cnt,
                       float* gate_bias, int n_max, int cluster, cudaStream_t stream);
int mq_row_groups(const sba_cache& c, int M);
int launch_multi_query(const sba_cache& c, const void* q, int M, const int32_t* sel_idx, const int32_t* sel_cnt,
                       int n_max, float scale, int num_splits,
                       float* o_part, float* lse_part, cudaStream_t stream);
int launch_multi_query_tc(const sba_cache& c, const void* q, int M, const int32_t* sel_idx, const int32_t* sel_cnt,
                          int n_max, float scale, int num_splits, float* o_part, float* lse_part,
                          cudaStream_t stream);
int launch_rectify_tc(const sba_cache& c, const void* q, int f, const void* k_new, const void* v_new, float scale,
                      int num_splits, float* o_part, float* lse_part, cudaStream_t stream);
int launch_fold_gate(const float* Wq, const float* Wk, int dg, float* A, cudaStream_t stream);
int launch_wait_timeout_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t stream);
int launch_combine(const float* o_part, const float* lse_part, int B, int H_q, int S, void* out, int out_dtype,
                   float* lse_out, cudaStream_t stream);

}  // namespace sba
