// Split-KV sparse decode over the selected blocks, and the split merge.
// (kOuter: the SAS gate on the values instead of inside the softmax.)
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation",
// Summary: exact attention over the group's selected blocks only; its
// references cite Flash-Decoding (split the KV range, merge partial results by
// log-sum-exp) and PagedAttention (block tables).  "SAS: Simple Attention
// Sparsification ...", Method: o = softmax(q K_S^T + log g_S) V_S, the log-gate
// added to the logits of each selected historical block.
//
// One CTA per (split, KV head, sequence), 5 warps:
//  - warp 4 is the producer: it looks up the physical page of each of its
//    selected blocks and streams the block's K and V tiles (b x 128 bf16 each,
//    two 64-channel halves per tensor) into a ring of shared-memory stages with
//    2-D TMA loads (128-byte swizzle), signalling an mbarrier per stage;
//  - warps 0-3 are consumers: each owns b/4 tokens of every block and runs the
//    G query heads of the group (padded to the 16 rows of an MMA tile) through
//    QK^T and PV on the bf16 tensor cores (fp32 accumulate) with an online
//    softmax; P enters PV as bf16 hi + bf16 lo parts, which keeps ~16 mantissa
//    bits of the fp32 probabilities;
//  - at the end the four warps' (max, sum, O) are merged in shared memory and
//    the split's normalised O and log-sum-exp are written.
// Every K/V byte is read from HBM once per group: the G query heads share it.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "decode_tile.cuh"
#include "launch.cuh"

namespace sba {

namespace {

constexpr int kConsumerWarps = kDecodeConsumerWarps;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

struct DecodeArgs {
    const int32_t* seq_lens;
    const int32_t* block_table;
    int32_t* status;
    int H_q, H_kv, max_blocks, num_pages;
    const __nv_bfloat16* q;
    const int32_t* sel_idx;
    const int32_t* sel_cnt;
    const float* gate_bias;
    int n_max;
    float scale_log2;  // softmax_scale * log2(e)
    int num_splits;
    float* o_part;
    float* lse_part;
};

template <int kBlk>
struct Smem {
    static constexpr int kHalf = TileGeom<kBlk>::kHalf;
    static constexpr int kStage = TileGeom<kBlk>::kStage;
    static constexpr int kStages = kBlk == 64 ? 6 : 3;
    static constexpr int kMerge = kConsumerWarps * 16 * kHeadDim * 4 + kConsumerWarps * 16 * 2 * 4;
    static constexpr int kBars = 2 * kStages * 8 + kStages * (int)sizeof(StageInfo);
    static constexpr int kBytes = kStages * kStage + kMerge + kBars + 1024;  // + alignment slack
};

template <int kBlk, bool kOuter>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         DecodeArgs a) {
    using S = Smem<kBlk>;
    constexpr int kStages = S::kStages;
    extern __shared__ uint8_t dyn_raw[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    float* merge_o = reinterpret_cast<float*>(dyn + kStages * S::kStage);          // [4][16][128]
    float* merge_ml = merge_o + kConsumerWarps * 16 * kHeadDim;                   // [4][16][2]
    uint64_t* full = reinterpret_cast<uint64_t*>(dyn + kStages * S::kStage + S::kMerge);
    uint64_t* empty = full + kStages;
    StageInfo* info = reinterpret_cast<StageInfo*>(empty + kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int G = a.H_q / a.H_kv;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        fence_mbar_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    __syncthreads();

    pdl_wait();
    pdl_trigger();

    const int len = __ldg(a.seq_lens + s);
    const int N = min(blocks_of(len, kBlk), a.max_blocks);
    int cnt = __ldg(a.sel_cnt + s * a.H_kv + h);
    if (cnt > a.n_max || cnt < 0) {
        if (tid == 0 && sp == 0) report(a.status, SBA_DEV_BAD_SELECTION);
        cnt = cnt < 0 ? 0 : a.n_max;
    }
    const int i0 = (int)((int64_t)cnt * sp / a.num_splits);
    const int i1 = (int)((int64_t)cnt * (sp + 1) / a.num_splits);
    const int nb = i1 - i0;
    const int32_t* sel = a.sel_idx + ((int64_t)s * a.H_kv + h) * a.n_max + i0;

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ------------------------------
        bool alive = true;
        for (int g0 = 0; g0 < nb && alive; g0 += 32) {
            // look up 32 blocks' pages in parallel
            int my_j = -1, my_page = -1;
            if (g0 + lane < nb) {
                my_j = __ldg(sel + g0 + lane);
                if (my_j >= 0 && my_j < N) {
                    my_page = a.block_table ? __ldg(a.block_table + (int64_t)s * a.max_blocks + my_j)
                                            : s * a.max_blocks + my_j;
                    if (my_page < 0 || my_page >= a.num_pages) {
                        report(a.status, SBA_DEV_BAD_PAGE);
                        my_page = -1;
                    }
                } else {
                    report(a.status, SBA_DEV_BAD_SELECTION);
                }
            }
            const int n_here = min(32, nb - g0);
            for (int ii = 0; ii < n_here; ++ii) {
                const int j = __shfl_sync(0xffffffffu, my_j, ii);
                const int page = __shfl_sync(0xffffffffu, my_page, ii);
                if (lane == 0 && alive) {
                    const int i = g0 + ii;
                    const int st = i % kStages;
                    if (i >= kStages && !mbar_wait(&empty[st], ((i / kStages) - 1) & 1, a.status)) alive = false;
                    if (alive) {
                        StageInfo inf;
                        inf.j = j;
                        inf.valid = page >= 0 ? min(kBlk, len - j * kBlk) : 0;
                        inf.ok = page >= 0;
                        inf.pos = i;
                        info[st] = inf;
                        if (page >= 0) {
                            uint8_t* base = dyn + st * S::kStage;
                            const int y = (page * a.H_kv + h) * kBlk;
                            mbar_arrive_expect_tx(&full[st], S::kStage);
                            tma_load_2d(base, &tmK, &full[st], 0, y);
                            tma_load_2d(base + S::kHalf, &tmK, &full[st], 64, y);
                            tma_load_2d(base + 2 * S::kHalf, &tmV, &full[st], 0, y);
                            tma_load_2d(base + 3 * S::kHalf, &tmV, &full[st], 64, y);
                        } else {
                            mbar_arrive(&full[st]);
                        }
                    }
                }
                alive = __shfl_sync(0xffffffffu, alive, 0);
            }
        }
    } else {
        // ------------------------------ consumers -----------------------------
        const int r = lane >> 2;
        uint32_t qa[8][4];
        load_q_frags(qa, a.q + ((int64_t)s * a.H_q + h * G) * kHeadDim, G, lane);
        const float* bias_r = (a.gate_bias && r < G) ? a.gate_bias + ((int64_t)s * a.H_q + h * G + r) * a.n_max + i0 : nullptr;
        const float* bias_r8 =
            (a.gate_bias && r + 8 < G) ? a.gate_bias + ((int64_t)s * a.H_q + h * G + r + 8) * a.n_max + i0 : nullptr;
        DecodeState dst;
        decode_state_init(dst);
        for (int i = 0; i < nb; ++i) {
            const int st = i % kStages;
            if (!mbar_wait(&full[st], (i / kStages) & 1, a.status)) break;
            const StageInfo inf = info[st];
            if (inf.ok) {
                const float g0 = bias_r ? __ldg(bias_r + i) * kLog2e : 0.f;
                const float g1 = bias_r8 ? __ldg(bias_r8 + i) * kLog2e : 0.f;
                decode_block<kBlk, kOuter>(dst, qa, dyn + st * S::kStage, inf.valid, g0, g1, a.scale_log2, warp,
                                           lane);  // slot = warp
            }
            // release the stage (generic-proxy writes ordered before the next TMA write)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        decode_state_store(dst, merge_o, merge_ml, warp, lane);
    }
    __syncthreads();
    // ---- merge the four consumer warps; 128 threads = 128 channels ----
    if (tid < kHeadDim) {
        const int ch = tid;
        for (int row = 0; row < G; ++row) {
            float o, lse;
            merge_warps(merge_o, merge_ml, row, ch, o, lse);
            const int64_t orow = ((int64_t)s * a.H_q + h * G + row) * a.num_splits + sp;
            a.o_part[orow * kHeadDim + ch] = o;
            if (ch == 0) a.lse_part[orow] = lse;
        }
    }
}

// LSE merge of the splits: one CTA per (query head, sequence), one thread per channel.
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                                      int H_q, int S, void* out, int out_dtype, float* lse_out) {
    pdl_wait();
    pdl_trigger();
    const int qh = blockIdx.x, s = blockIdx.y, ch = threadIdx.x;
    const int64_t row = (int64_t)s * H_q + qh;
    const float* lp = lse_part + row * S;
    float M = -INFINITY;
    for (int i = 0; i < S; ++i) M = fmaxf(M, __ldg(lp + i));
    float acc = 0.f, z = 0.f;
    if (M > -INFINITY) {
        for (int i = 0; i < S; ++i) {
            const float l = __ldg(lp + i);
            if (l == -INFINITY) continue;
            const float w = expf(l - M);
            z += w;
            acc = fmaf(w, __ldg(o_part + (row * S + i) * kHeadDim + ch), acc);
        }
    }
    const float v = z > 0.f ? acc / z : 0.f;
    if (out_dtype == SBA_OUT_BF16)
        reinterpret_cast<__nv_bfloat16*>(out)[row * kHeadDim + ch] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(out)[row * kHeadDim + ch] = v;
    if (lse_out && ch == 0) lse_out[row] = z > 0.f ? M + logf(z) : -INFINITY;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

// 2-D view [rows = num_pages*H_kv*b][128] bf16 of a K or V cache; box = 64 channels x b rows.
bool make_kv_tmap(CUtensorMap* m, void* base, uint64_t rows, int blk) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)blk};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Descriptor rows (512 bytes per (page, KV head)) of a contiguous cache as a 4-D
// map of 4-byte words: 32 words x 4 quarter rows x H_kv x pages, one box = `rows`
// consecutive pages of one head, 128-byte swizzle (16-byte chunk c of quarter row R
// lands at chunk c ^ (R & 7)).
bool make_desc_tmap(CUtensorMap* m, void* base, uint64_t pages, int H_kv, int rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {32, 4, (cuuint64_t)H_kv, pages};
    cuuint64_t strides[3] = {128, 512, (cuuint64_t)H_kv * 512};
    cuuint32_t box[4] = {32, 4, 1, (cuuint32_t)rows};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int kBlk, bool kOuter>
int launch_decode_blk(const sba_cache& c, const DecodeArgs& a, cudaStream_t stream) {
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)c.num_pages * c.H_kv * kBlk;
    if (!make_kv_tmap(&tk, c.k, rows, kBlk) || !make_kv_tmap(&tv, c.v, rows, kBlk)) return SBA_ERR_CUDA;
    const int smem = Smem<kBlk>::kBytes;
    if (allow_smem<sparse_decode_kernel<kBlk, kOuter>>(smem) != SBA_OK) return SBA_ERR_CUDA;
    dim3 grid(a.num_splits, c.H_kv, c.B);
    return launch(sparse_decode_kernel<kBlk, kOuter>, grid, dim3(kThreads), smem, stream, tk, tv, a);
}

}  // namespace

int launch_sparse_decode(const sba_cache& c, const void* q, const int32_t* sel_idx, const int32_t* sel_cnt,
                         const float* gate_bias, int n_max, float scale, int num_splits, float* o_part,
                         float* lse_part, bool outer, cudaStream_t stream) {
    DecodeArgs a{};
    a.seq_lens = c.seq_lens;
    a.block_table = c.block_table;
    a.status = c.status;
    a.H_q = c.H_q;
    a.H_kv = c.H_kv;
    a.max_blocks = c.max_blocks;
    a.num_pages = c.num_pages;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.gate_bias = gate_bias;
    a.n_max = n_max;
    a.scale_log2 = scale * kLog2e;
    a.num_splits = num_splits;
    a.o_part = o_part;
    a.lse_part = lse_part;
    if (outer) return c.b == 64 ? launch_decode_blk<64, true>(c, a, stream) : launch_decode_blk<128, true>(c, a, stream);
    return c.b == 64 ? launch_decode_blk<64, false>(c, a, stream) : launch_decode_blk<128, false>(c, a, stream);
}

int launch_combine(const float* o_part, const float* lse_part, int B, int H_q, int S, void* out, int out_dtype,
                   float* lse_out, cudaStream_t stream) {
    dim3 grid(H_q, B);
    return launch(combine_kernel, grid, dim3(kHeadDim), 0, stream, o_part, lse_part, H_q, S, out, out_dtype, lse_out);
}

}  // namespace sba
