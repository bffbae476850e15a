// Group block scoring and shared top-n selection.
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation",
// Summary: Quest-style min/max descriptors score the blocks and all query
// heads of a GQA group share one selection; Key points: top-n that always
// keeps the recent local blocks and a minimum count.
// "SAS: Simple Attention Sparsification ...", Method: gate scores are
// softmax-normalised over the historical blocks (or, as in its ablations,
// passed through a sigmoid or injected unnormalised); the current block B0
// keeps a unit gate; the log-gates of the selected blocks go into the attention.
//
// One launch per call.  CTAs of grid (chunk, kv head, sequence) score CHUNK
// blocks each and write fp32 scores to the workspace; the last CTA to finish a
// (sequence, group) -- detected with a plain atomic counter, never a wait --
// runs the selection over that group's N scores in shared memory and resets
// the counter to zero for the next call.
//
// Quest score of block j for group g is
//   sum_{qh in g} sum_c max(q_qh,c mn_c, q_qh,c mx_c) = sum_c (P_c mx_c + M_c mn_c)
// with P_c = sum_qh max(q_qh,c, 0), M_c = sum_qh min(q_qh,c, 0): the sum over
// the group's heads is taken once per call (reassociation only), so each block
// costs one 256-term dot product whatever the group size.
#include <math.h>

#include "common.cuh"
#include "launch.cuh"
#include "select.cuh"

namespace sba {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBlocksPerWarpIter = 8;  // 4 lanes per block descriptor (512 B)
constexpr int kRefSMs = 148;
constexpr int kSelCap = 1024;  // selection buffer (candidates above the group-maximum bound)

struct ScoreArgs {
    sba_cache c;
    const __nv_bfloat16* q;  // [B][M][H_q][d]
    int M;                   // query tokens per sequence sharing the selection (Quest)
    sba_select_params p;
    int32_t* sel_idx;
    int32_t* sel_cnt;
    float* gate_bias;
    int n_max;
    uint32_t* counters;  // [B][H_kv]
    float* scores;       // Quest: [B][H_kv][mb] group scores; gate: [B][H_q][mb] logits u
    float* mz;           // gate: [B][H_q][n_chunks][2] (chunk max, chunk sum of exp(u - max))
    int chunk;           // blocks per CTA, multiple of 64
};

struct WsLayout {
    size_t counters, scores, mz, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const sba_cache& c, const sba_select_params& p, int chunk) {
    WsLayout w{};
    const int n_chunks = (c.max_blocks + chunk - 1) / chunk;
    size_t off = 0;
    w.counters = off;
    off += align256(sizeof(uint32_t) * c.B * c.H_kv);
    w.scores = off;
    const int rows = p.scorer == SBA_SCORER_GATE ? c.H_q : c.H_kv;
    off += align256(sizeof(float) * (size_t)c.B * rows * c.max_blocks);
    w.mz = off;
    if (p.scorer == SBA_SCORER_GATE) off += align256(sizeof(float) * 2 * (size_t)c.B * c.H_q * n_chunks);
    w.total = off;
    return w;
}

template <int kScorer>
__global__ void __launch_bounds__(kThreads) score_select_kernel(ScoreArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ uint32_t hist[256];
    __shared__ int warp_tot[kWarps];
    __shared__ uint32_t sh[2];
    __shared__ int is_last;
    __shared__ int sel_misc[2];
    __shared__ float lse_s[kMaxGroup];
    __shared__ __align__(16) float q_s[kMaxGroup][kHeadDim];

    pdl_wait();
    pdl_trigger();

    const sba_cache& c = a.c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.z, h = blockIdx.y, chunk_id = blockIdx.x;
    const int G = c.H_q / c.H_kv;
    const int mb = c.max_blocks;
    int len = __ldg(c.seq_lens + s);
    int N = blocks_of(len, c.b);
    if (N > mb) {
        if (tid == 0 && chunk_id == 0 && h == 0) report(c.status, SBA_DEV_BAD_POSITION);
        N = mb;
    }
    const int L = num_local(N, a.p);
    // blocks scored: Quest ranks [0, N-L); the gate needs u over all historical blocks [0, N-1)
    const int n_scored = kScorer == SBA_SCORER_GATE ? max(N - 1, 0) : N - L;
    const int j0 = chunk_id * a.chunk;
    const int j1 = min(j0 + a.chunk, n_scored);

    uint32_t* keys = reinterpret_cast<uint32_t*>(dyn);                  // [mb] (selection)
    float* u_s = reinterpret_cast<float*>(dyn);                          // [G][chunk] (gate, aliases keys)
    const size_t main_words = max((size_t)mb, (size_t)G * a.chunk);
    int* pages_s = reinterpret_cast<int*>(dyn + main_words * 4);         // [chunk]

    // ---- prefetch the chunk's physical pages ----
    for (int j = j0 + tid; j < j1; j += kThreads) {
        const int64_t p = page_of(c, s, j, c.status);
        pages_s[j - j0] = (int)p;
    }

    const int qt = lane & 3, sub = lane >> 2;
    if (kScorer == SBA_SCORER_QUEST) {
        // the group's coefficients P_c = sum of max(q_c, 0) and M_c = sum of min(q_c, 0) over its
        // query rows (several query tokens of a sequence: their heads join the group's sum, ReSA
        // Summary), by the whole CTA: thread t takes channels 8 (t / 16) .. + 7 of every 16th row
        // from row t % 16 (16-byte loads), the 16 row lanes of a half warp summed by shuffles
        static_assert(kThreads == 256, "16 channel groups x 16 row lanes");
        __shared__ float coef_pm[2][kHeadDim];  // [P, M][channel]
        {
            const int cg = tid >> 4, rl = tid & 15;
            float pp[8], mm[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pp[e] = mm[e] = 0.f;
            const int R = G * a.M;
#pragma unroll 4
            for (int gi = rl; gi < R; gi += 16) {
                const int g = gi % G, qi = gi / G;
                const uint4 w = __ldg(reinterpret_cast<const uint4*>(
                    a.q + (((int64_t)s * a.M + qi) * c.H_q + h * G + g) * kHeadDim) + cg);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = bf16_lo(ws[e]), x1 = bf16_hi(ws[e]);
                    pp[2 * e] += fmaxf(x0, 0.f);
                    mm[2 * e] += fminf(x0, 0.f);
                    pp[2 * e + 1] += fmaxf(x1, 0.f);
                    mm[2 * e + 1] += fminf(x1, 0.f);
                }
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pp[e] += __shfl_xor_sync(0xffffffffu, pp[e], o);
                    mm[e] += __shfl_xor_sync(0xffffffffu, mm[e], o);
                }
            if (rl == 0)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    coef_pm[0][8 * cg + e] = pp[e];
                    coef_pm[1][8 * cg + e] = mm[e];
                }
        }
        __syncthreads();  // coefficients (and pages_s) ready
        // this lane's 64 descriptor values: qt 0/1 = min row channels 0-63/64-127 (weights M),
        // qt 2/3 = max row (weights P)
        const int ch0 = (qt & 1) * 64;
        const float* cf = coef_pm[qt >= 2 ? 0 : 1] + ch0;
        float coef[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) coef[e] = cf[e];
        const uint4* desc = reinterpret_cast<const uint4*>(c.desc);
        float* out = a.scores + ((int64_t)s * c.H_kv + h) * mb;
        for (int base = j0 + warp * kBlocksPerWarpIter; base < j1; base += kWarps * kBlocksPerWarpIter) {
            const int j = base + sub;
            float acc = 0.f;
            if (j < j1) {
                const int page = pages_s[j - j0];
                if (page >= 0) {
                    const uint4* ptr = desc + ((int64_t)page * c.H_kv + h) * 32 + qt * 8;
                    uint4 w[8];
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) w[k8] = __ldg(ptr + k8);
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) {
                        const uint32_t ws[4] = {w[k8].x, w[k8].y, w[k8].z, w[k8].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            acc = fmaf(coef[8 * k8 + 2 * e], bf16_lo(ws[e]), acc);
                            acc = fmaf(coef[8 * k8 + 2 * e + 1], bf16_hi(ws[e]), acc);
                        }
                    }
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (qt == 0 && j < j1) out[j] = acc + 0.0f;
        }
    } else {
        // gate: u_qh,j = q_qh . kg_j for the group's G heads; lane quarter qt owns channels qt*32..qt*32+31
        for (int i = tid; i < G * kHeadDim; i += kThreads) {
            const int g = i / kHeadDim, ch = i % kHeadDim;
            q_s[g][ch] = __bfloat162float(a.q[((int64_t)s * c.H_q + h * G + g) * kHeadDim + ch]);
        }
        __syncthreads();
        const float4* kg = reinterpret_cast<const float4*>(c.kg);
        for (int base = j0 + warp * kBlocksPerWarpIter; base < j1; base += kWarps * kBlocksPerWarpIter) {
            const int j = base + sub;
            float acc[kMaxGroup];
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g) acc[g] = 0.f;
            if (j < j1) {
                const int page = pages_s[j - j0];
                if (page >= 0) {
                    const float4* ptr = kg + ((int64_t)page * c.H_kv + h) * 32 + qt * 8;
                    float4 w[8];
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) w[k8] = __ldg(ptr + k8);
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) {
#pragma unroll
                        for (int g = 0; g < kMaxGroup; ++g) {
                            if (g < G) {
                                const float4 qv = *reinterpret_cast<const float4*>(&q_s[g][qt * 32 + 4 * k8]);
                                acc[g] = fmaf(qv.x, w[k8].x, acc[g]);
                                acc[g] = fmaf(qv.y, w[k8].y, acc[g]);
                                acc[g] = fmaf(qv.z, w[k8].z, acc[g]);
                                acc[g] = fmaf(qv.w, w[k8].w, acc[g]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g) {
                if (g < G) {
                    float v = acc[g];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    if (qt == 0 && j < j1) {
                        a.scores[((int64_t)s * c.H_q + h * G + g) * mb + j] = v;
                        u_s[g * a.chunk + (j - j0)] = v;
                    }
                }
            }
        }
        __syncthreads();
        // per-head (max, sum exp(u - max)) of this chunk
        const int n_chunks = gridDim.x;
        for (int g = warp; g < G; g += kWarps) {
            float m = -INFINITY;
            for (int i = lane; i < j1 - j0; i += 32) m = fmaxf(m, u_s[g * a.chunk + i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float z = 0.f;
            if (m > -INFINITY)
                for (int i = lane; i < j1 - j0; i += 32) z += expf(u_s[g * a.chunk + i] - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if (lane == 0) {
                float* dst = a.mz + (((int64_t)s * c.H_q + h * G + g) * n_chunks + chunk_id) * 2;
                dst[0] = m;
                dst[1] = z;
            }
        }
    }

    // ---- completion count: the last CTA of this (sequence, group) selects ----
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t prev = atomicAdd(a.counters + s * c.H_kv + h, 1u);
        is_last = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    const int n_sel = num_selected(N, a.p);
    const int NC = N - L;  // ranked candidates [0, NC); locals [NC, N)
    const int k = n_sel - L;
    if (kScorer == SBA_SCORER_QUEST) {
        const float* sc = a.scores + ((int64_t)s * c.H_kv + h) * mb;
        for (int j = tid; j < NC; j += kThreads) keys[j] = orderable_key(__ldcg(sc + j));
    } else {
        const int n_chunks = gridDim.x;
        const int act = a.p.gate_act;  // sigmoid and unnormalised gates need no normaliser
        if (act != SBA_GATE_SOFTMAX)
            for (int g = tid; g < G; g += kThreads) lse_s[g] = 0.f;
        for (int g = warp; act == SBA_GATE_SOFTMAX && g < G; g += kWarps) {
            const float* mzp = a.mz + ((int64_t)s * c.H_q + h * G + g) * n_chunks * 2;
            float M = -INFINITY;
            for (int i = lane; i < n_chunks; i += 32) M = fmaxf(M, __ldcg(mzp + 2 * i));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            float Z = 0.f;
            if (M > -INFINITY)
                for (int i = lane; i < n_chunks; i += 32) {
                    const float m = __ldcg(mzp + 2 * i);
                    if (m > -INFINITY) Z += __ldcg(mzp + 2 * i + 1) * expf(m - M);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
            if (lane == 0) lse_s[g] = M > -INFINITY ? M + logf(Z) : -INFINITY;
        }
        __syncthreads();
        // four blocks per thread and round, their G scores' loads in flight together
        const float* sc0 = a.scores + ((int64_t)s * c.H_q + h * G) * mb;
        for (int j0r = 0; j0r < NC; j0r += 4 * kThreads) {
            float u[4][kMaxGroup];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = j0r + x * kThreads + tid;
#pragma unroll
                for (int g = 0; g < kMaxGroup; ++g) u[x][g] = (g < G && j < NC) ? __ldcg(sc0 + (int64_t)g * mb + j) : 0.f;
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = j0r + x * kThreads + tid;
                float sc = 0.f;
#pragma unroll
                for (int g = 0; g < kMaxGroup; ++g)
                    if (g < G) sc += gate_of(u[x][g], lse_s[g], act);
                if (j < NC) keys[j] = orderable_key(sc);
            }
        }
    }
    __syncthreads();
    int32_t* out = a.sel_idx + ((int64_t)s * c.H_kv + h) * a.n_max;
    {
        uint32_t* gscr = reinterpret_cast<uint32_t*>(dyn + (main_words + a.chunk) * 4);
        uint32_t* bkey = gscr + (mb + 3) / 4 + 4;
        int* bidx = reinterpret_cast<int*>(bkey + kSelCap);
        int* brank = bidx + kSelCap;
        select_fast<kThreads>(keys, NC, N, k, out, a.n_max, gscr, bkey, bidx, brank, kSelCap, sel_misc, hist, warp_tot,
                              sh);
    }
    if (n_sel > a.n_max && tid == 0) report(c.status, SBA_DEV_BAD_SELECTION);
    const int n_out = min(n_sel, a.n_max);
    if (tid == 0) a.sel_cnt[s * c.H_kv + h] = n_out;
    if (kScorer == SBA_SCORER_GATE && a.gate_bias != nullptr) {
        __syncthreads();
        for (int i = tid; i < n_out * G; i += kThreads) {
            const int pos = i / G, g = i % G;
            const int j = __ldcg(out + pos);
            const float bias = j == N - 1 ? 0.f
                                          : log_gate_of(__ldcg(a.scores + ((int64_t)s * c.H_q + h * G + g) * mb + j),
                                                        lse_s[g], a.p.gate_act);
            a.gate_bias[((int64_t)s * c.H_q + h * G + g) * a.n_max + pos] = bias;
        }
    }
    if (tid == 0) a.counters[s * c.H_kv + h] = 0u;  // ready for the next call
}

}  // namespace

int score_chunk_blocks(const sba_cache& c) {
    int chunk = kWarps * kBlocksPerWarpIter;
    const int64_t units = (int64_t)c.B * c.H_kv;
    while (chunk < 1024 && units * ((c.max_blocks + chunk - 1) / chunk) > 4 * kRefSMs) chunk *= 2;
    return chunk;
}

size_t score_workspace_bytes(const sba_cache& c, const sba_select_params& p) {
    return ws_layout(c, p, score_chunk_blocks(c)).total;
}

static size_t score_smem_bytes(const sba_cache& c, int chunk) {
    const int G = c.H_q / c.H_kv;
    const size_t main_words = c.max_blocks > G * chunk ? (size_t)c.max_blocks : (size_t)G * chunk;
    const size_t sel_words = (size_t)(c.max_blocks + 3) / 4 + 4 + 3 * kSelCap;
    return (main_words + chunk + sel_words) * 4;
}

int launch_score_select(const sba_cache& c, const void* q, int M, const sba_select_params& p, int32_t* sel_idx,
                        int32_t* sel_cnt, float* gate_bias, int n_max, void* ws, cudaStream_t stream) {
    const int chunk = score_chunk_blocks(c);
    const WsLayout w = ws_layout(c, p, chunk);
    ScoreArgs a{};
    a.c = c;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.M = M;
    a.p = p;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.gate_bias = gate_bias;
    a.n_max = n_max;
    a.counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + w.counters);
    a.scores = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.scores);
    a.mz = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.mz);
    a.chunk = chunk;
    const size_t smem = score_smem_bytes(c, chunk);
    dim3 grid((c.max_blocks + chunk - 1) / chunk, c.H_kv, c.B);
    if (smem > (size_t)200 * 1024) return SBA_ERR_UNSUPPORTED;
    if (p.scorer == SBA_SCORER_GATE) {
        if (allow_smem<score_select_kernel<SBA_SCORER_GATE>>((int)smem) != SBA_OK) return SBA_ERR_CUDA;
        return launch(score_select_kernel<SBA_SCORER_GATE>, grid, dim3(kThreads), smem, stream, a);
    }
    if (allow_smem<score_select_kernel<SBA_SCORER_QUEST>>((int)smem) != SBA_OK) return SBA_ERR_CUDA;
    return launch(score_select_kernel<SBA_SCORER_QUEST>, grid, dim3(kThreads), smem, stream, a);
}

}  // namespace sba
