// Fused decode step: append -> descriptor refresh -> block scoring -> shared
// top-n selection -> sparse attention -> merge, in ONE launch per layer.
//
// Same method as the separate calls ("Rectified Sparse Attention for
// Efficient Long-Sequence Generation", Summary and Key points; "SAS: Simple
// Attention Sparsification ...", Method), organised for B200:
//  - one thread-block CLUSTER of C CTAs (one CTA per SM) per (sequence, KV
//    group); CTA r owns slice r of the sequence's scored blocks and share r
//    of the selected blocks for attention;
//  - one shared-memory ring of 32 KB stages, filled by a producer warp: a
//    contiguous cache's descriptors arrive 64 per stage in one 4-D TMA load,
//    a paged cache's are streamed by every warp with 16-byte loads straight
//    into registers; K/V tiles come with 2-D TMA loads (128-B swizzle);
//  - the selection is replicated: every CTA pushes each key (an order-preserving
//    u32 of the block's score) to every peer as it is produced, and the maxima
//    of groups of its keys (distributed shared memory); after one cluster
//    barrier each CTA derives the same lower bound T0 of the n-th score from the
//    group maxima (k group maxima are k distinct candidates), gathers the keys
//    >= T0 from its own copy and ranks that short list exactly.  Scores never
//    reach global memory;
//  - partial (O, LSE) of the CTAs are pushed to the merging CTA of each output
//    element; all pushes precede a cluster barrier, after which every CTA reads
//    only its own shared memory;
//  - every CTA loads a 1/C share of the step's appended K/V rows at the start
//    and stores it after scoring, ahead of the cluster barrier that precedes
//    the decode's tile loads; the descriptors of the touched blocks are
//    recomputed by the producer warp from the K tiles the decode stages anyway
//    (the touched blocks are local, hence selected).  When a touched block is
//    one the step itself scores (e.g. no local blocks), CTA 0 appends and
//    refreshes it from global memory first and a cluster barrier orders that
//    before the scoring.
// No workspace: every intermediate lives in shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "decode_tile.cuh"
#include "launch.cuh"
#include "select.cuh"

namespace sba {

bool make_kv_tmap(CUtensorMap* m, void* base, uint64_t rows, int blk);                // decode.cu
bool make_desc_tmap(CUtensorMap* m, void* base, uint64_t pages, int H_kv, int rows);  // decode.cu

namespace {

constexpr int kGW = kDecodeConsumerWarps;  // warps of one consumer group (4 token slots)
constexpr int kGroups = 2;                  // consumer groups: alternate ring stages
constexpr int kCW = kGW * kGroups;          // consumer warps
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kProducer = kCW;
constexpr int kMaxCluster = 16;
constexpr int kDescBytes = 512;
static_assert(kCW == 8, "the merge weights are read as two float4 per row");

struct StepArgs {
    sba_cache c;
    const __nv_bfloat16* q;
    const uint4* k_new;
    const uint4* v_new;
    const int32_t* pos_start;
    int n_new;
    const float* gate_A;  // [128][384]: folded gate projection
    sba_select_params p;
    float scale_log2;
    void* out;
    int out_dtype;
    float* lse_out;
    int32_t* sel_idx;
    int32_t* sel_cnt;
    float* gate_bias;
    int n_max;
    // shared-memory layout (bytes from the 1024-aligned base) and capacities
    int n_stages;
    int slice;      // largest slice: ceil(max_blocks / C) rounded up to a multiple of 4
    int off_keys, off_pages, off_u, off_kall, off_gm, off_crank, off_sel, off_selp, off_recv, off_bars;
    int ccap;       // candidates ranked exactly (keys at or above the group-maxima bound)
    int sel_cap;    // words in sel / sel_page
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

// Reduce-scatter of NB per-block partial sums (V values each) over the 32
// lanes: on return out[] holds, in every lane, the full sums of block
// rs_block<NB>(lane).
template <int NB, int V>
__device__ __forceinline__ void reduce_scatter(float (&v)[NB][V], float (&out)[V], int lane) {
    int n = NB;
#pragma unroll
    for (int m = 16; m >= (NB == 8 ? 4 : 8); m >>= 1) {
        const bool up = (lane & m) != 0;
        const int half = n >> 1;
#pragma unroll
        for (int k = 0; k < NB / 2; ++k) {
            if (k < half) {
#pragma unroll
                for (int x = 0; x < V; ++x) {
                    const float send = up ? v[k][x] : v[k + half][x];
                    const float keep = up ? v[k + half][x] : v[k][x];
                    v[k][x] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
        }
        n = half;
    }
#pragma unroll
    for (int x = 0; x < V; ++x) {
        float t = v[0][x];
        if (NB == 4) t += __shfl_xor_sync(0xffffffffu, t, 4);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        out[x] = t;
    }
}

template <int NB>
__device__ __forceinline__ int rs_block(int lane) {
    return NB == 8 ? (((lane >> 4) & 1) << 2) | (((lane >> 3) & 1) << 1) | ((lane >> 2) & 1)
                   : (((lane >> 4) & 1) << 1) | ((lane >> 3) & 1);
}

// CTA 0: write the step's new tokens of (s, h) into the cache.
// Element e of the step's new rows of (s, h): per token 16 x 16 B of K, then 16 x 16 B of V.
__device__ __forceinline__ const uint4* append_src(const StepArgs& a, int s, int h, int e) {
    const int tok = e >> 5, half = (e >> 4) & 1, l = e & 15;
    return (half ? a.v_new : a.k_new) + (((int64_t)s * a.n_new + tok) * a.c.H_kv + h) * 16 + l;
}
__device__ __forceinline__ void append_store(const StepArgs& a, int s, int h, int p0, int e, uint4 v) {
    const sba_cache& c = a.c;
    const int tok = e >> 5, half = (e >> 4) & 1, l = e & 15;
    const int pos = p0 + tok;
    const int64_t page = page_of(c, s, pos / c.b, c.status);
    if (page < 0) return;
    reinterpret_cast<uint4*>(half ? c.v : c.k)[((page * c.H_kv + h) * c.b + pos % c.b) * 16 + l] = v;
}

// Elements [e0, e1) of the step's new rows, written through the block table.
__device__ __noinline__ void append_rows(const StepArgs& a, int s, int h, int p0, int e0, int e1, int tid) {
    for (int e = e0 + tid; e < e1; e += kThreads) append_store(a, s, h, p0, e, __ldg(append_src(a, s, h, e)));
    fence_proxy_async_global();
}

// Descriptor of block j of (s, h) from global memory (threads 0..127, one
// channel each).  Quest: min/max rows; gate: pooled -> kg = A pooled.
template <int kScorer>
__device__ __noinline__ void refresh_from_global(const StepArgs& a, int s, int h, int j, int len, float* pooled, int tid) {
    const sba_cache& c = a.c;
    const int64_t page = page_of(c, s, j, tid == 0 ? c.status : nullptr);
    const int cnt = min(c.b, len - j * c.b);
    if (page >= 0 && cnt > 0 && tid < kHeadDim) {
        const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(c.k) + (page * c.H_kv + h) * c.b * kHeadDim;
        float lo = INFINITY, hi = -INFINITY, sum = 0.f;
        for (int t = 0; t < cnt; ++t) {
            const float x = __bfloat162float(kt[t * kHeadDim + tid]);
            lo = fminf(lo, x);
            hi = fmaxf(hi, x);
            sum += x;
        }
        if (kScorer == SBA_SCORER_QUEST) {
            __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(c.desc) + (page * c.H_kv + h) * 2 * kHeadDim;
            d[tid] = __float2bfloat16_rn(lo);
            d[kHeadDim + tid] = __float2bfloat16_rn(hi);
        } else {
            pooled[tid] = hi;
            pooled[kHeadDim + tid] = lo;
            pooled[2 * kHeadDim + tid] = sum / (float)cnt;
        }
    }
    if (kScorer == SBA_SCORER_GATE) {
        __syncthreads();
        if (page >= 0 && cnt > 0 && tid < kHeadDim) {
            const float* Ar = a.gate_A + (int64_t)tid * 3 * kHeadDim;
            float acc = 0.f;
            for (int i = 0; i < 3 * kHeadDim; ++i) acc = fmaf(__ldg(Ar + i), pooled[i], acc);
            c.kg[(page * c.H_kv + h) * kHeadDim + tid] = acc;
        }
        __syncthreads();
    }
}

__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Descriptor of a touched block from its K rows staged in shared memory (one or two 64-row
// stages), by one warp: lane = 16-byte chunk (8 channels) of a row x token parity.  The min,
// max (exact in bf16) and, for the gate, the fp32 sum accumulate over the stages.
struct RefreshAcc {
    uint32_t mn[4], mx[4];
    float sm[8];
};

__device__ __forceinline__ void refresh_init(RefreshAcc& acc) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc.mn[e] = 0x7f807f80u;  // +inf, +inf
        acc.mx[e] = 0xff80ff80u;  // -inf, -inf
        acc.sm[2 * e] = acc.sm[2 * e + 1] = 0.f;
    }
}

template <int kScorer>
__device__ __forceinline__ void refresh_accum(RefreshAcc& acc, const uint8_t* stage, int valid, int lane) {
    using TG = TileGeom<64>;
    const int ck = lane & 15, cc = ck & 7;
    const uint8_t* kt = stage + (ck >> 3) * TG::kHalf;
#pragma unroll 4
    for (int t = lane >> 4; t < valid; t += 2) {
        const uint4 w = *reinterpret_cast<const uint4*>(kt + t * 128 + ((cc ^ (t & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc.mn[e] = bf16x2_min(acc.mn[e], ws[e]);
            acc.mx[e] = bf16x2_max(acc.mx[e], ws[e]);
            if (kScorer == SBA_SCORER_GATE) {
                acc.sm[2 * e] += bf16_lo(ws[e]);
                acc.sm[2 * e + 1] += bf16_hi(ws[e]);
            }
        }
    }
}

// Quest: the min/max rows go to the cache; gate: the pooled [max | min | avg] summary is
// pushed to every CTA of the cluster, which project it after the merge.
template <int kScorer>
__device__ __forceinline__ void refresh_finish(const sba_cache& c, RefreshAcc& acc, int valid, int64_t pg, int h,
                                               float* pooled_b0, int C, int lane) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {  // the other token parity
        acc.mn[e] = bf16x2_min(acc.mn[e], __shfl_xor_sync(0xffffffffu, acc.mn[e], 16));
        acc.mx[e] = bf16x2_max(acc.mx[e], __shfl_xor_sync(0xffffffffu, acc.mx[e], 16));
        if (kScorer == SBA_SCORER_GATE) {
            acc.sm[2 * e] += __shfl_xor_sync(0xffffffffu, acc.sm[2 * e], 16);
            acc.sm[2 * e + 1] += __shfl_xor_sync(0xffffffffu, acc.sm[2 * e + 1], 16);
        }
    }
    if (lane >= 16) return;
    const int ck = lane;
    if (kScorer == SBA_SCORER_QUEST) {
        uint8_t* d = reinterpret_cast<uint8_t*>(c.desc) + (pg * c.H_kv + h) * 2 * kHeadDim * 2;
        *reinterpret_cast<uint4*>(d + ck * 16) = make_uint4(acc.mn[0], acc.mn[1], acc.mn[2], acc.mn[3]);
        *reinterpret_cast<uint4*>(d + 2 * kHeadDim + ck * 16) = make_uint4(acc.mx[0], acc.mx[1], acc.mx[2], acc.mx[3]);
    } else {
        const float inv = 1.f / (float)valid;
        const uint32_t* mx = acc.mx;
        const uint32_t* mn = acc.mn;
        const float* sm = acc.sm;
        const float4 hi0 = make_float4(bf16_lo(mx[0]), bf16_hi(mx[0]), bf16_lo(mx[1]), bf16_hi(mx[1]));
        const float4 hi1 = make_float4(bf16_lo(mx[2]), bf16_hi(mx[2]), bf16_lo(mx[3]), bf16_hi(mx[3]));
        const float4 lo0 = make_float4(bf16_lo(mn[0]), bf16_hi(mn[0]), bf16_lo(mn[1]), bf16_hi(mn[1]));
        const float4 lo1 = make_float4(bf16_lo(mn[2]), bf16_hi(mn[2]), bf16_lo(mn[3]), bf16_hi(mn[3]));
        const float4 av0 = make_float4(sm[0] * inv, sm[1] * inv, sm[2] * inv, sm[3] * inv);
        const float4 av1 = make_float4(sm[4] * inv, sm[5] * inv, sm[6] * inv, sm[7] * inv);
        auto bits = [](float4 v) {
            return make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w));
        };
        for (int p = 0; p < C; ++p) {
            st_peer_v4(peer_addr(pooled_b0 + 8 * ck, p), bits(hi0));
            st_peer_v4(peer_addr(pooled_b0 + 8 * ck + 4, p), bits(hi1));
            st_peer_v4(peer_addr(pooled_b0 + kHeadDim + 8 * ck, p), bits(lo0));
            st_peer_v4(peer_addr(pooled_b0 + kHeadDim + 8 * ck + 4, p), bits(lo1));
            st_peer_v4(peer_addr(pooled_b0 + 2 * kHeadDim + 8 * ck, p), bits(av0));
            st_peer_v4(peer_addr(pooled_b0 + 2 * kHeadDim + 8 * ck + 4, p), bits(av1));
        }
    }
}

// Quest weights of this lane's 16 bytes of a descriptor: lane < 16 holds MIN row channels
// 8*lane..+7 (weight M = sum over the group's heads of min(q, 0)); lane >= 16 the MAX row
// channels 8*(lane-16)..+7 (weight P = sum of max(q, 0)).
__device__ __forceinline__ void quest_coef(float (&coef)[8], const __nv_bfloat16* qg, int G, int lane) {
    const int ch0 = (lane & 15) * 8;
    const bool use_max = lane >= 16;
    uint4 w[kMaxGroup];  // every head's load in flight at once
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
        if (g < G) w[g] = __ldg(reinterpret_cast<const uint4*>(qg + (int64_t)g * kHeadDim + ch0));
#pragma unroll
    for (int e = 0; e < 8; ++e) coef[e] = 0.f;
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        if (g >= G) break;
        const uint32_t ws[4] = {w[g].x, w[g].y, w[g].z, w[g].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo(ws[e]), x1 = bf16_hi(ws[e]);
            coef[2 * e] += use_max ? fmaxf(x0, 0.f) : fminf(x0, 0.f);
            coef[2 * e + 1] += use_max ? fmaxf(x1, 0.f) : fminf(x1, 0.f);
        }
    }
}

// Physical page of block j without reporting (speculative lookups).
__device__ __forceinline__ int page_quiet(const sba_cache& c, int s, int j) {
    const int64_t p = c.block_table ? (int64_t)__ldg(c.block_table + (int64_t)s * c.max_blocks + j)
                                    : (int64_t)s * c.max_blocks + j;
    return (p < 0 || p >= c.num_pages) ? -1 : (int)p;
}

// Paged cache scoring of blocks [j0, js1) (their pages in `pages`): Quest keys into `keys` and
// every CTA's `kall`, or the gate's u into u_s.  Out of line: a contiguous cache never runs it.
template <int kScorer, int kGM>
__device__ __noinline__ void score_paged(const StepArgs& a, int s, int h, int G, int j0, int js1, const int* pages,
                                         uint32_t* keys, uint32_t* kall, bool trivial, int C, float* u_s, int ustride,
                                         int warp, int lane) {
    const sba_cache& c = a.c;
    // Paged cache: every warp streams descriptors straight into registers: kRB blocks per
    // warp and round, lane l holding bytes [16 l, 16 l + 16) of each 512-byte descriptor;
    // the next round's loads are in flight while the current round is reduced.

        constexpr int kNW = kThreads / 32;
        constexpr int kRB = (kScorer == SBA_SCORER_GATE && kGM > 8) ? 4 : 8;  // (register budget)
        const uint8_t* src = (kScorer == SBA_SCORER_QUEST ? reinterpret_cast<const uint8_t*>(c.desc)
                                                          : reinterpret_cast<const uint8_t*>(c.kg)) +
                             (int64_t)h * kDescBytes + lane * 16;
        const int64_t pstride = (int64_t)c.H_kv * kDescBytes;
        float coef[8];
        float qg[kGM][4];  // gate: kGM = G rounded up to a power of two
        if (kScorer == SBA_SCORER_QUEST) {
            quest_coef(coef, a.q + ((int64_t)s * c.H_q + h * G) * kHeadDim, G, lane);
        } else {
            // gate: lane owns channels 4*lane..4*lane+3 of the fp32 gate key
#pragma unroll
            for (int g = 0; g < kGM; ++g) {
                if (g < G) {
                    const uint2 w = __ldg(reinterpret_cast<const uint2*>(a.q + ((int64_t)s * c.H_q + h * G + g) * kHeadDim +
                                                                        4 * lane));
                    qg[g][0] = bf16_lo(w.x);
                    qg[g][1] = bf16_hi(w.x);
                    qg[g][2] = bf16_lo(w.y);
                    qg[g][3] = bf16_hi(w.y);
                } else {
                    qg[g][0] = qg[g][1] = qg[g][2] = qg[g][3] = 0.f;
                }
            }
        }
        uint4 wc[kRB], wn[kRB];
        auto load_round = [&](int base, uint4(&w)[kRB]) {
#pragma unroll
            for (int b = 0; b < kRB; ++b) {
                const int j = base + b;
                const int pg = j < js1 ? pages[j - j0] : -1;
                w[b] = pg >= 0 ? ld_stream_v4(src + pg * pstride) : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        int base = j0 + warp * kRB;
        if (base < js1) load_round(base, wc);
        for (; base < js1; base += kNW * kRB) {
            if (base + kNW * kRB < js1) load_round(base + kNW * kRB, wn);
            if (kScorer == SBA_SCORER_QUEST) {
                float part[kRB][1];
#pragma unroll
                for (int b = 0; b < kRB; ++b) {
                    const uint32_t ws[4] = {wc[b].x, wc[b].y, wc[b].z, wc[b].w};
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc = fmaf(coef[2 * e], bf16_lo(ws[e]), acc);
                        acc = fmaf(coef[2 * e + 1], bf16_hi(ws[e]), acc);
                    }
                    part[b][0] = acc;
                }
                float tot[1];
                reduce_scatter<kRB, 1>(part, tot, lane);
                const int j = base + rs_block<kRB>(lane);
                if ((lane & 3) == 0 && j < js1) {
                    const uint32_t key = pages[j - j0] >= 0 ? orderable_key(tot[0]) : 0u;
                    keys[j - j0] = key;
                    if (!trivial)
                        for (int p = 0; p < C; ++p) st_peer_u32(peer_addr(kall + j, p), key);
                }
            } else {
#pragma unroll
                for (int q4 = 0; q4 < kRB; q4 += 4) {
                    float part[4][kGM];
#pragma unroll
                    for (int b4 = 0; b4 < 4; ++b4) {
                        const uint4 w = wc[q4 + b4];
                        const float x0 = __uint_as_float(w.x), x1 = __uint_as_float(w.y), x2 = __uint_as_float(w.z),
                                    x3 = __uint_as_float(w.w);
#pragma unroll
                        for (int g = 0; g < kGM; ++g) {
                            float acc = qg[g][0] * x0;
                            acc = fmaf(qg[g][1], x1, acc);
                            acc = fmaf(qg[g][2], x2, acc);
                            acc = fmaf(qg[g][3], x3, acc);
                            part[b4][g] = acc;
                        }
                    }
                    float tot[kGM];
                    reduce_scatter<4, kGM>(part, tot, lane);
                    const int j = base + q4 + rs_block<4>(lane);
                    if ((lane & 7) == 0 && j < js1) {
                        const bool ok = pages[j - j0] >= 0;
#pragma unroll
                        for (int g = 0; g < kGM; ++g)
                            if (g < G) u_s[g * ustride + (j - j0)] = ok ? tot[g] : -INFINITY;
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < kRB; ++b) wc[b] = wn[b];
        }
}

template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmD, const __grid_constant__ StepArgs a) {
    // The ring holds 64-token stages (32 KB): a block of 128 tokens takes two consecutive fills,
    // and a descriptor chunk is 64 descriptors.
    using TG = TileGeom<64>;
    constexpr int kSub = kBlk / 64;   // ring fills per block
    constexpr int kSC = 64;           // descriptors per scoring fill
    constexpr int kMaxLocal = 64;
    __shared__ uint32_t hist[256];
    __shared__ int warp_tot[kThreads / 32];
    __shared__ uint32_t sh[2];
    __shared__ int misc[4];
    __shared__ float lse_s[kMaxGroup];
    __shared__ float lse_all[kMaxCluster * kMaxGroup];
    __shared__ __align__(16) float wgt_s[kMaxGroup][kCW];  // merge weights of the consumer warps
    __shared__ float cw_s[kMaxGroup][kMaxCluster];       // merge weights of the cluster's CTAs
    __shared__ float rlse_s[kMaxGroup];
    __shared__ float mz_all[kMaxCluster * kMaxGroup][2];
    __shared__ int local_page[kMaxLocal];
    __shared__ __align__(16) float pooled[3 * kHeadDim];     // refresh-before-score scratch
    __shared__ __align__(16) float pooled_b0[3 * kHeadDim];  // pushed pooled summary of B0

    extern __shared__ uint8_t dyn_raw[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    const int NSt = a.n_stages;
    uint32_t* keys = reinterpret_cast<uint32_t*>(dyn + a.off_keys);  // own slice
    int* pages = reinterpret_cast<int*>(dyn + a.off_pages);          // own slice
    float* u_s = reinterpret_cast<float*>(dyn + a.off_u);            // gate: [G][slice]
    int* crank = reinterpret_cast<int*>(dyn + a.off_crank);
    int* sel = reinterpret_cast<int*>(dyn + a.off_sel);
    int* sel_page = reinterpret_cast<int*>(dyn + a.off_selp);
    float* recv_o = reinterpret_cast<float*>(dyn + a.off_recv);
    uint64_t* full = reinterpret_cast<uint64_t*>(dyn + a.off_bars);
    uint64_t* empty = full + NSt;
    StageInfo* info = reinterpret_cast<StageInfo*>(empty + NSt);
    // after the decode: per-warp merge area (aliases the ring)
    float* merge_o = reinterpret_cast<float*>(dyn);
    float* merge_ml = merge_o + kCW * 16 * kMergeStride;

    const sba_cache& c = a.c;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = (int)cluster_rank(), C = (int)cluster_size();
    const int h = blockIdx.y, s = blockIdx.z;
    const int G = c.H_q / c.H_kv;
    const int mb = c.max_blocks;
    const int ustride = a.slice;  // row stride of u_s: the largest slice

    if (tid == 0) {
        for (int i = 0; i < NSt; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGW);  // one consumer group releases a stage
        }
        fence_mbar_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        if (!kPaged) prefetch_tmap(&tmD);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const int len = __ldg(c.seq_lens + s);  // (both loads in flight while the work below is issued)
    const int p0raw = a.n_new > 0 ? __ldg(a.pos_start + s) : 0;
    // A contiguous cache's descriptors need no length to be located: the first ring stages of
    // this CTA's slice (a fixed share of max_blocks) are requested before the lengths arrive.
    constexpr bool contiguous = !kPaged;
    const int nspec = contiguous ? min(NSt, (a.slice + kSC - 1) / kSC) : 0;
    if (contiguous && warp == kProducer && lane == 0)
        for (int f = 0; f < nspec; ++f) {
            mbar_arrive_expect_tx(&full[f], TG::kStage);
            tma_load_4d(dyn + (size_t)f * TG::kStage, &tmD, &full[f], 0, 0, h, s * mb + r * a.slice + f * kSC);
        }

    // ... nor do the query-side scoring coefficients of the consumer warps (ring scoring)
    constexpr int NTq = kGM > 8 ? 2 : 1;  // gate: 8-head n-tiles
    float coef[8];
    uint32_t qf[NTq][8][4];
    if (contiguous && warp < kCW) {
        if (kScorer == SBA_SCORER_QUEST) {
            quest_coef(coef, a.q + ((int64_t)s * c.H_q + h * G) * kHeadDim, G, lane);
        } else {
            // B fragments: head nt*8 + lane/4, channels 16p + 4(lane%4) + 0..3 (bf16 is exact in tf32)
#pragma unroll
            for (int nt = 0; nt < NTq; ++nt) {
                const int head = nt * 8 + (lane >> 2);
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    uint2 w = make_uint2(0u, 0u);
                    if (head < G)
                        w = __ldg(reinterpret_cast<const uint2*>(a.q + ((int64_t)s * c.H_q + h * G + head) * kHeadDim +
                                                                16 * p + 4 * (lane & 3)));
                    qf[nt][p][0] = w.x << 16;
                    qf[nt][p][1] = w.x & 0xffff0000u;
                    qf[nt][p][2] = w.y << 16;
                    qf[nt][p][3] = w.y & 0xffff0000u;
                }
            }
        }
    }

    // ---------------- shapes of this (sequence, group) ----------------
    int N = blocks_of(len, kBlk);
    if (N > mb) {
        if (tid == 0 && r == 0) report(c.status, SBA_DEV_BAD_POSITION);
        N = mb;
    }
    const int L = num_local(N, a.p);
    const int n_sel = min(num_selected(N, a.p), a.sel_cap);
    const int NC = N - L;                                               // ranked candidates [0, NC)
    const int NSc = kScorer == SBA_SCORER_GATE ? max(N - 1, 0) : NC;   // blocks this step scores
    // this sequence's scored blocks [0, NSc) in C equal slices (sequences differ in length)
    // (a contiguous cache keeps the fixed slices its early loads assumed)
    const int slice = contiguous ? a.slice : min(max(4, ((NSc + C - 1) / C + 3) & ~3), a.slice);
    const int j0 = min(r * slice, NSc), js1 = min(j0 + slice, NSc);    // my scored blocks [j0, js1)
    const int jc1 = max(j0, min(js1, NC));                              // my ranked candidates [j0, jc1)
    for (int j = j0 + tid; j < js1; j += kThreads) {
        const int pg = page_quiet(c, s, j);
        pages[j - j0] = pg;
        if (pg < 0) report(c.status, SBA_DEV_BAD_PAGE);
    }
    const int k = n_sel - L;
    const bool trivial = k <= 0 || k >= NC;  // take none / all of the candidates
    // Selection geometry, known before scoring.  Every CTA receives every key (kall) and every
    // CTA's group maxima (gmx: groups of gs blocks aligned to each slice) while the keys are
    // produced, so that one cluster barrier later each CTA selects on its own.  The group size
    // is the largest power of two in [4, 128] leaving >= 2k groups (T0 below costs ~ng^2
    // comparisons, the exact rank ~m^2 for the m keys >= T0; more groups give a tighter T0).
    int gsh = 7;
    if (!trivial)
        while (gsh > 2 && ((NC + (1 << gsh) - 1) >> gsh) < 2 * k) --gsh;
    const int gs = 1 << gsh;
    int goff = 0, ng = 0;
    for (int p = 0; p < C; ++p) {
        const int b0 = min(p * slice, NC);
        const int ngp = (min(b0 + slice, NC) - b0 + gs - 1) >> gsh;
        goff += p < r ? ngp : 0;
        ng += ngp;
    }
    // (the gate's keys are produced after scoring, when the ring is idle everywhere)
    uint32_t* kall = kScorer == SBA_SCORER_GATE ? reinterpret_cast<uint32_t*>(dyn)
                                                : reinterpret_cast<uint32_t*>(dyn + a.off_kall);
    uint32_t* gmx = reinterpret_cast<uint32_t*>(dyn + a.off_gm);
    for (int i = tid; i < L && i < kMaxLocal; i += kThreads) local_page[i] = page_quiet(c, s, NC + i);

    int n_new = a.n_new, p0 = 0, tb0 = 1, tb1 = 0;
    if (n_new > 0) {
        p0 = p0raw;
        if (p0 < 0 || (int64_t)p0 + n_new > (int64_t)mb * kBlk) {
            if (tid == 0 && r == 0) report(c.status, SBA_DEV_BAD_POSITION);
            n_new = 0;
        } else {
            tb0 = p0 / kBlk;
            tb1 = min((p0 + n_new - 1) / kBlk, N - 1);
        }
    }
    const bool touched_scored = n_new > 0 && tb0 <= tb1 && tb0 < NSc;

    // ---------------- append (and, if needed, refresh before scoring) ----------------
    // When a touched block is scored, CTA 0 writes the new rows and refreshes those blocks
    // before anyone scores.  Otherwise each CTA loads its share of the rows now (one element
    // per thread; a share above the CTA's threads is written at once) and stores it after
    // scoring, before the cluster barriers that order it ahead of the decode's tile loads.
    uint4 app_v = make_uint4(0u, 0u, 0u, 0u);
    int app_e = -1;
    if (touched_scored) {
        if (r == 0) {
            append_rows(a, s, h, p0, 0, n_new * 32, tid);
            __syncthreads();
            for (int j = tb0; j <= tb1; ++j) refresh_from_global<kScorer>(a, s, h, j, len, pooled, tid);
            fence_proxy_async_global();
        }
        cluster_sync();
    } else if (n_new > 0) {
        const int total = n_new * 32, per = (total + C - 1) / C;
        const int e0 = min(r * per, total), e1 = min(e0 + per, total);
        if (e0 + tid < e1) {
            app_e = e0 + tid;
            app_v = __ldg(append_src(a, s, h, app_e));
        }
        if (e1 - e0 > kThreads) append_rows(a, s, h, p0, e0 + kThreads, e1, tid);
    }

    // ---------------- phase 1: score this CTA's slice ----------------
    __syncthreads();  // page ids of the slice
    uint32_t fill = 0;  // ring fills so far (consecutive fills alternate consumer groups)
    if (!kPaged) {
        // Contiguous cache: one TMA load brings the descriptors of kBlk consecutive blocks into
        // a ring stage (128-byte quarter rows, 128-byte swizzle); the two consumer groups take
        // alternate stages, each warp 16 descriptors (one tensor-core tile for the gate) per
        // 64 of the stage.
        // Fills [0, nspec) were requested early.  Normally they are chunks 0.. of the slice (those
        // past its end are drained unread); after a refresh before scoring their contents may
        // be stale, so they are drained and every chunk is requested again.
        const int nch = (js1 - j0 + kSC - 1) / kSC;
        const int skip = touched_scored ? nspec : 0;
        const int ntot = touched_scored ? nspec + nch : max(nch, nspec);
        if (warp == kProducer) {
            if (lane == 0) {
                bool alive = true;
                for (int f = nspec; f < ntot && alive; ++f) {
                    const int st = f % NSt;
                    if (f >= NSt) alive = mbar_wait(&empty[st], ((f / NSt) - 1) & 1, c.status);
                    if (alive) {
                        mbar_arrive_expect_tx(&full[st], TG::kStage);
                        tma_load_4d(dyn + (size_t)st * TG::kStage, &tmD, &full[st], 0, 0, h,
                                    s * mb + j0 + (f - skip) * kSC);
                    }
                }
            }
        } else {
            const int grp = warp / kGW, gw = warp % kGW;
            constexpr int kIt = kSC / 64;          // 16-descriptor pieces of a stage per warp
            bool alive = true;
            for (int f = grp; f < ntot; f += kGroups) {
                const int st = f % NSt;
                if (alive) alive = mbar_wait(&full[st], (f / NSt) & 1, c.status);
                const int cb = j0 + (f - skip) * kSC;
                // (<= 0: a drained fill, or a stage whose wait ran out: nothing of it is read)
                const int nblk = (f < skip || !alive) ? 0 : min(kSC, js1 - cb);
                const uint8_t* stage = dyn + (size_t)st * TG::kStage;
                if (kScorer == SBA_SCORER_QUEST) {
#pragma unroll
                    for (int it = 0; it < kIt; ++it) {
                        // two independent rounds of 8 descriptors, lane l = bytes [16 l, 16 l + 16) of each
                        const int n0 = 16 * gw + 64 * it;
                        if (n0 >= nblk) break;
                        float part[2][8][1];
#pragma unroll
                        for (int rd = 0; rd < 2; ++rd)
#pragma unroll
                            for (int b8 = 0; b8 < 8; ++b8) {
                                const int R = (n0 + 8 * rd + b8) * 4 + (lane >> 3);
                                const uint4 w =
                                    *reinterpret_cast<const uint4*>(stage + R * 128 + (((lane & 7) ^ (R & 7)) << 4));
                                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                                float acc = 0.f;
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    acc = fmaf(coef[2 * e], bf16_lo(ws[e]), acc);
                                    acc = fmaf(coef[2 * e + 1], bf16_hi(ws[e]), acc);
                                }
                                part[rd][b8][0] = acc;
                            }
                        float tot[2][1];
                        reduce_scatter<8, 1>(part[0], tot[0], lane);
                        reduce_scatter<8, 1>(part[1], tot[1], lane);
#pragma unroll
                        for (int rd = 0; rd < 2; ++rd) {
                            const int i = n0 + 8 * rd + rs_block<8>(lane);
                            if ((lane & 3) == 0 && i < nblk) {
                                const int jl = cb + i - j0;
                                const uint32_t key = pages[jl] >= 0 ? orderable_key(tot[rd][0]) : 0u;
                                keys[jl] = key;
                                if (!trivial)
                                    for (int p = 0; p < C; ++p) st_peer_u32(peer_addr(kall + j0 + jl, p), key);
                            }
                        }
                    }
                } else {
                    // u = q . kg on tensor cores: tiles of 16 blocks (rows) x 8 heads (columns);
                    // kg = hi + lo (hi = kg truncated to tf32 by a bit mask -- a full-rate logic op,
                    // where a rounding conversion runs at a fraction of the issue rate -- and lo = the
                    // exact remainder, read by the MMA truncated to tf32: about 21 bits of kg); four
                    // accumulators per tile (channel half x hi/lo) keep the MMA chains short, and
                    // a warp's tiles of the stage run interleaved when registers allow
                    constexpr int kTl = (kIt == 2 && NTq == 1) ? 2 : 1;
                    const int gq = lane >> 2, t = lane & 3;
#pragma unroll
                    for (int it0 = 0; it0 < kIt; it0 += kTl) {
                        if (16 * gw + 64 * it0 >= nblk) break;
                        float acc[kTl][NTq][4][4];
#pragma unroll
                        for (int tl = 0; tl < kTl; ++tl)
#pragma unroll
                            for (int nt = 0; nt < NTq; ++nt)
#pragma unroll
                                for (int x = 0; x < 4; ++x)
                                    acc[tl][nt][x][0] = acc[tl][nt][x][1] = acc[tl][nt][x][2] = acc[tl][nt][x][3] = 0.f;
                        // every shared-memory read of the tile first, so that they are all in flight
                        // together; the MMA chains then run on registers
                        float4 xs[kTl][8][2];
#pragma unroll
                        for (int p = 0; p < 8; ++p)
#pragma unroll
                            for (int tl = 0; tl < kTl; ++tl) {
                                const int n0 = 16 * gw + 64 * (it0 + tl);
                                const int R0 = (n0 + gq) * 4 + (p >> 1);
                                const int off = ((((p & 1) << 2) | t) ^ (R0 & 7)) << 4;
                                xs[tl][p][0] = *reinterpret_cast<const float4*>(stage + R0 * 128 + off);
                                xs[tl][p][1] = *reinterpret_cast<const float4*>(stage + (R0 + 32) * 128 + off);
                            }
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
#pragma unroll
                            for (int tl = 0; tl < kTl; ++tl) {
                                const float4 x0 = xs[tl][p][0];
                                const float4 x1 = xs[tl][p][1];
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const float v[4] = {e ? x0.z : x0.x, e ? x1.z : x1.x, e ? x0.w : x0.y,
                                                        e ? x1.w : x1.y};
                                    uint32_t hi[4], lo[4];
#pragma unroll
                                    for (int u = 0; u < 4; ++u) {  // (the MMA reads the top 19 bits of each)
                                        hi[u] = __float_as_uint(v[u]) & 0xffffe000u;  // v truncated to tf32
                                        lo[u] = __float_as_uint(v[u] - __uint_as_float(hi[u]));
                                    }
                                    const int ah = (p >> 2) * 2;  // accumulator pair of this channel half
#pragma unroll
                                    for (int nt = 0; nt < NTq; ++nt) {
                                        mma_tf32_1688(acc[tl][nt][ah], hi, qf[nt][p][2 * e], qf[nt][p][2 * e + 1]);
                                        mma_tf32_1688(acc[tl][nt][ah + 1], lo, qf[nt][p][2 * e], qf[nt][p][2 * e + 1]);
                                    }
                                }
                            }
                        }
                        // u of blocks n0 + gq (elements 0, 1) and n0 + gq + 8 (2, 3), heads nt*8 + 2t (+1)
#pragma unroll
                        for (int tl = 0; tl < kTl; ++tl)
#pragma unroll
                            for (int hb = 0; hb < 2; ++hb) {
                                const int i = 16 * gw + 64 * (it0 + tl) + gq + 8 * hb;
                                if (i < nblk) {
                                    const int jl = cb + i - j0;
                                    const bool ok = pages[jl] >= 0;
#pragma unroll
                                    for (int nt = 0; nt < NTq; ++nt)
#pragma unroll
                                        for (int x = 0; x < 2; ++x) {
                                            const int hd = nt * 8 + 2 * t + x, el = 2 * hb + x;
                                            const float u = (acc[tl][nt][0][el] + acc[tl][nt][2][el]) +
                                                            (acc[tl][nt][1][el] + acc[tl][nt][3][el]);
                                            if (hd < G) u_s[hd * ustride + jl] = ok ? u : -INFINITY;
                                        }
                                }
                            }
                    }
                }
                fence_proxy_async_smem();  // these reads before the next TMA write of the stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
        }
        fill = (uint32_t)ntot;
    } else {
        score_paged<kScorer, kGM>(a, s, h, G, j0, js1, pages, keys, kall, trivial, C, u_s, ustride, warp, lane);
    }
    __syncthreads();
    if (app_e >= 0) append_store(a, s, h, p0, app_e, app_v);  // (its proxy fence comes before barrier B)

    // ---------------- phase 2: distributed selection ----------------
    if (kScorer == SBA_SCORER_GATE) {
        // softmax gates: per-head (max, sum exp(u - max)) over this CTA's scored blocks, one warp
        // per head, pushed to every CTA; sigmoid and unnormalised gates need no normaliser (lse = 0
        // below).  Exponentials are exp2 of log2(e)-scaled arguments (one special-function op each).
        const bool softmax_gate = a.p.gate_act == SBA_GATE_SOFTMAX;
        if (softmax_gate) {
            for (int g = warp; g < G; g += kThreads / 32) {
                float m = -INFINITY;
                for (int i = lane; i < js1 - j0; i += 32) m = fmaxf(m, u_s[g * ustride + i]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                float z = 0.f;
                if (m > -INFINITY)
                    for (int i = lane; i < js1 - j0; i += 32) z += exp2f((u_s[g * ustride + i] - m) * kLog2e);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                for (int p = lane; p < C; p += 32) {
                    st_peer_f32(peer_addr(&mz_all[r * G + g][0], p), m);
                    st_peer_f32(peer_addr(&mz_all[r * G + g][1], p), z);
                }
            }
            cluster_sync();  // gate round: every CTA's softmax partials pushed
            // LSE of head g by warp g: lane p reads CTA p's pair (C <= 16 lanes)
            for (int g = warp; g < G; g += kThreads / 32) {
                const float m = lane < C ? mz_all[lane * G + g][0] : -INFINITY;
                const float z = lane < C ? mz_all[lane * G + g][1] : 0.f;
                float M = m;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
                float Z = (M > -INFINITY && m > -INFINITY) ? z * exp2f((m - M) * kLog2e) : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
                if (lane == 0) lse_s[g] = M > -INFINITY ? M + logf(Z) : -INFINITY;
            }
        } else if (tid < G) {
            lse_s[tid] = 0.f;
        }
        __syncthreads();
        // group score of my ranked blocks: sum over the group of g (softmax: exp(u - LSE); raw:
        // exp(u); sigmoid: 1 / (1 + exp(-u))), four blocks per thread, pushed to every CTA
        const bool sigmoid_gate = a.p.gate_act == SBA_GATE_SIGMOID;
        for (int v = tid; 4 * v < jc1 - j0; v += kThreads) {
            const int jl = 4 * v;
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int g = 0; g < G; ++g) {
                const float4 u4 = *reinterpret_cast<const float4*>(u_s + g * ustride + jl);
                if (sigmoid_gate) {
                    sc[0] += gate_of(u4.x, 0.f, SBA_GATE_SIGMOID);
                    sc[1] += gate_of(u4.y, 0.f, SBA_GATE_SIGMOID);
                    sc[2] += gate_of(u4.z, 0.f, SBA_GATE_SIGMOID);
                    sc[3] += gate_of(u4.w, 0.f, SBA_GATE_SIGMOID);
                } else {
                    sc[0] += exp2f((u4.x - lse_s[g]) * kLog2e);
                    sc[1] += exp2f((u4.y - lse_s[g]) * kLog2e);
                    sc[2] += exp2f((u4.z - lse_s[g]) * kLog2e);
                    sc[3] += exp2f((u4.w - lse_s[g]) * kLog2e);
                }
            }
            uint32_t kk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                kk[e] = (jl + e < jc1 - j0 && pages[jl + e] >= 0) ? orderable_key(sc[e]) : 0u;
            const uint4 k4 = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            *reinterpret_cast<uint4*>(keys + jl) = k4;
            if (!trivial)
                for (int p = 0; p < C; ++p) st_peer_v4(peer_addr(kall + j0 + jl, p), k4);
        }
        __syncthreads();
    }
    // my keys are final: the maxima of my slice's groups go to every CTA (four keys per thread,
    // groups of gs/4 lanes); zeros (never larger) pad the vectors the rank counts read
    const int S0 = ng * 8 <= kThreads ? 8 : ng * 4 <= kThreads ? 4 : ng * 2 <= kThreads ? 2 : 1;
    const int nv0 = (ng + 4 * S0 - 1) / (4 * S0) * S0;
    if (!trivial) {
        const int nown = jc1 - j0, lpg = gs / 4;
        const uint4* kv = reinterpret_cast<const uint4*>(keys);
        const int nvo = (nown + 3) / 4;
        for (int v0 = warp * 32; v0 < nvo; v0 += kThreads) {
            const int v = v0 + lane;
            uint32_t m = 0;
            if (v < nvo) {
                const uint4 q = kv[v];
                const int j = 4 * v;
                m = max(max(j < nown ? q.x : 0u, j + 1 < nown ? q.y : 0u),
                        max(j + 2 < nown ? q.z : 0u, j + 3 < nown ? q.w : 0u));
            }
            for (int o = 1; o < lpg; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((lane & (lpg - 1)) == 0 && v < nvo)
                for (int p = 0; p < C; ++p) st_peer_u32(peer_addr(gmx + goff + v / lpg, p), m);
        }
        for (int i = ng + tid; i < 4 * nv0; i += kThreads) gmx[i] = 0u;
        if (tid == 0) misc[0] = -1;  // T0 (atomic minimum below)
    }
    // every CTA's keys and group maxima are in every CTA: each selects on its own
    if (app_e >= 0) fence_proxy_async_global();  // the appended rows, for the decode's tile loads
    cluster_sync();
    if (trivial) {
        const int first = k <= 0 ? NC : 0;
        for (int i = tid; i < N - first; i += kThreads) {
            sel[i] = first + i;
            sel_page[i] = first + i >= NC ? local_page[first + i - NC] : -1;
        }
    } else {
        const int nv = (NC + 3) / 4;
        uint32_t* gm = gmx;
        // candidates (and the fallback's scratch) in the idle ring, after the gate's keys
        uint32_t* scr = kScorer == SBA_SCORER_GATE ? kall + ((NC + 127) & ~127) : reinterpret_cast<uint32_t*>(dyn);
        uint32_t* ck = scr;
        int* ci = reinterpret_cast<int*>(ck + a.ccap + 32);
        // T0 = the k-th largest group maximum (k group maxima are k distinct blocks; with fewer
        // than k groups T0 = 0).  Every thread counts, for one group maximum, the larger ones
        // among a 1/S share of them.
        uint32_t T0 = 0;
        if (ng >= k) {
            const uint4* gv = reinterpret_cast<const uint4*>(gm);
            for (int t0 = 0; t0 < ng * S0; t0 += kThreads) {
                const int t = t0 + tid, g = t / S0, sg = t % S0;
                int n0 = 0, n1 = 0, n2 = 0, n3 = 0;
                uint32_t x = 0;
                if (g < ng) {
                    x = gm[g];
#pragma unroll 4
                    for (int v = sg; v < nv0; v += S0) {
                        const uint4 y = gv[v];
                        n0 += y.x > x;
                        n1 += y.y > x;
                        n2 += y.z > x;
                        n3 += y.w > x;
                    }
                }
                int n = (n0 + n1) + (n2 + n3);
                for (int o = 1; o < S0; o <<= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
                uint32_t cand = (g < ng && n < k) ? x : 0xffffffffu;
                cand = __reduce_min_sync(0xffffffffu, cand);
                if (lane == 0 && cand != 0xffffffffu) atomicMin(reinterpret_cast<unsigned*>(&misc[0]), cand);
            }
            __syncthreads();
            T0 = (uint32_t)misc[0];
        }
        // the keys >= T0 in ascending block order: thread t scans a contiguous run of vectors (an
        // odd number of them, so that a warp's 16-byte reads fall in distinct banks)
        const uint4* kv = reinterpret_cast<const uint4*>(kall);
        const int perv = ((nv + kThreads - 1) / kThreads) | 1;
        const int v0r = min(tid * perv, nv), v1r = min(v0r + perv, nv);
        int cnt = 0;
        for (int v = v0r; v < v1r; ++v) {
            const uint4 q = kv[v];
            const int j = 4 * v;
            cnt += (q.x >= T0) + ((q.y >= T0) & (j + 1 < NC)) + ((q.z >= T0) & (j + 2 < NC)) +
                   ((q.w >= T0) & (j + 3 < NC));
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int pos = incl - cnt, m = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const int x = warp_tot[w];
            pos += w < warp ? x : 0;
            m += x;
        }
        if (m <= a.ccap) {
            for (int v = v0r; v < v1r; ++v) {
                const uint4 q = kv[v];
                const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (qs[e] >= T0 && 4 * v + e < NC) {
                        ck[pos] = qs[e];
                        ci[pos] = 4 * v + e;
                        ++pos;
                    }
            }
            const int S = m * 8 <= kThreads ? 8 : m * 4 <= kThreads ? 4 : m * 2 <= kThreads ? 2 : 1;
            const int nvec = (m + 4 * S - 1) / (4 * S) * S;  // 16-byte vectors of the ranking, padded
            for (int i = m + tid; i < 4 * nvec; i += kThreads) {  // pads rank below everything
                ck[i] = 0u;
                ci[i] = 0x7fffffff;
            }
            __syncthreads();
            // exact rank in (key desc, index asc) of every candidate, S threads per candidate
            const uint4* kv4 = reinterpret_cast<const uint4*>(ck);
            const int4* iv4 = reinterpret_cast<const int4*>(ci);
            for (int t0 = 0; t0 < m * S; t0 += kThreads) {
                const int t = t0 + tid, i = t / S, sg = t % S;
                int n0 = 0, n1 = 0;
                if (i < m) {
                    const uint32_t ki = ck[i];
                    const int xi = ci[i];
#pragma unroll 2
                    for (int v = sg; v < nvec; v += S) {
                        const uint4 y = kv4[v];
                        const int4 z = iv4[v];
                        n0 += (y.x > ki) | ((y.x == ki) & (z.x < xi));
                        n1 += (y.y > ki) | ((y.y == ki) & (z.y < xi));
                        n0 += (y.z > ki) | ((y.z == ki) & (z.z < xi));
                        n1 += (y.w > ki) | ((y.w == ki) & (z.w < xi));
                    }
                }
                int n = n0 + n1;
                for (int o = 1; o < S; o <<= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
                if (i < m && sg == 0) crank[i] = n;
            }
            __syncthreads();
            // the k best, in ascending block order: output position = selected ones before
            for (int t0 = 0, run = 0; t0 < m; t0 += kThreads) {
                const int i = t0 + tid;
                const bool take = i < m && crank[i] < k;
                const unsigned bal = __ballot_sync(0xffffffffu, take);
                if (lane == 0) warp_tot[warp] = __popc(bal);
                __syncthreads();
                int off = run, tot = 0;
                for (int w = 0; w < kThreads / 32; ++w) {
                    const int x = warp_tot[w];
                    off += w < warp ? x : 0;
                    tot += x;
                }
                if (take) sel[off + __popc(bal & ((1u << lane) - 1u))] = ci[i];
                run += tot;
                __syncthreads();
            }
        } else {
            // too many keys >= T0 (e.g. many equal scores): the exact selection on all keys
            uint32_t* gscr = scr;
            uint32_t* bkey = gscr + ((NC + 3) / 4 + 4);
            int* bidx = reinterpret_cast<int*>(bkey + 1024);
            int* brank = bidx + 1024;
            __syncthreads();
            select_fast<kThreads>(kall, NC, NC, k, sel, a.sel_cap, gscr, bkey, bidx, brank, 1024, misc + 2, hist,
                                  warp_tot, sh);
            __syncthreads();
        }
        // pages of the selected blocks: from the slice owners (or computed, for a contiguous cache)
        for (int i = tid; i < k; i += kThreads) {
            const int j = sel[i];
            const int p = j / slice;
            sel_page[i] = !kPaged ? page_quiet(c, s, j)
                          : p == r                 ? pages[j - j0]
                                                   : (int)ld_peer_u32(peer_addr(pages + (j - p * slice), p));
        }
        for (int i = tid; i < L; i += kThreads) {
            sel[k + i] = NC + i;
            sel_page[k + i] = i < kMaxLocal ? local_page[i] : -1;
        }
    }
    __syncthreads();
    if (r == 0) {
        if (a.sel_idx)
            for (int i = tid; i < n_sel && i < a.n_max; i += kThreads)
                a.sel_idx[((int64_t)s * c.H_kv + h) * a.n_max + i] = sel[i];
        if (a.sel_cnt && tid == 0) a.sel_cnt[s * c.H_kv + h] = min(n_sel, a.n_max);
    }

    // ---------------- phase 3: decode this CTA's share of the selection ----------------
    const int i0 = (int)((int64_t)n_sel * r / C), i1 = (int)((int64_t)n_sel * (r + 1) / C);
    const bool tile_refresh = n_new > 0 && !touched_scored;
    const int E = G * kHeadDim;         // merge elements (row, channel) of this group
    const int share = (E + C - 1) / C;  // elements merged by each CTA
    if (warp == kProducer) {
        // page ids the selection did not carry (locals past kMaxLocal, or all blocks when
        // every candidate is taken) are looked up here, 32 at a time
        for (int g0 = i0; g0 < i1; g0 += 32) {
            const int i = g0 + lane;
            if (i < i1 && sel_page[i] < 0) {
                const int j = sel[i];
                sel_page[i] = (j >= 0 && j < N) ? (int)page_of(c, s, j, c.status) : -1;
            }
        }
        __syncwarp();
        bool alive = true;
        // Blocks touched by this step's append get their descriptors from their staged K rows,
        // here: when the stage of a touched block's first fill is about to be reused (its other
        // fill, issued after it, is then waited for), or, for the last fills, after the loop.
        auto touched = [&](int i) {
            const int j = sel[i];
            return tile_refresh && j >= tb0 && j <= tb1 && sel_page[i] >= 0;
        };
        const uint32_t fill0 = fill;  // the first fill of this phase (the ring may hold descriptor chunks before)
        auto refresh = [&](int i) {   // block at position i, all of whose fills have been issued
            const int j = sel[i], valid = min(kBlk, len - j * kBlk);
            RefreshAcc acc;
            refresh_init(acc);
            bool ok = true;
#pragma unroll
            for (int sb = 0; sb < kSub; ++sb) {
                const uint32_t f = fill0 + (uint32_t)((i - i0) * kSub + sb);
                if (lane == 0) ok = mbar_wait(&full[f % NSt], (f / NSt) & 1, c.status) && ok;
                if (__shfl_sync(0xffffffffu, ok, 0))
                    refresh_accum<kScorer>(acc, dyn + (size_t)(f % NSt) * TG::kStage, min(64, max(0, valid - 64 * sb)),
                                           lane);
            }
            if (__shfl_sync(0xffffffffu, ok, 0))
                refresh_finish<kScorer>(c, acc, valid, sel_page[i], h, pooled_b0, C, lane);
            fence_proxy_async_smem();  // these generic reads before the next TMA writes of the stages
            __syncwarp();
        };
        for (int i = i0; i < i1; ++i) {
#pragma unroll 1
            for (int sb = 0; sb < kSub; ++sb, ++fill) {
                const int st = fill % NSt;
                if (fill >= (uint32_t)NSt) {
                    if (lane == 0 && alive) alive = mbar_wait(&empty[st], ((fill / NSt) - 1) & 1, c.status);
                    alive = __shfl_sync(0xffffffffu, alive, 0);
                    const uint32_t prev = fill - NSt;  // the fill whose stage is reused now
                    if (alive && prev >= fill0 && (prev - fill0) % kSub == 0) {
                        const int ip = i0 + (int)((prev - fill0) / kSub);
                        if (touched(ip)) refresh(ip);
                    }
                }
                if (lane == 0 && alive) {
                    const int j = sel[i];
                    const int pg = (j >= 0 && j < N) ? sel_page[i] : -1;
                    StageInfo inf;
                    inf.j = j;
                    inf.valid = pg >= 0 ? min(64, max(0, min(kBlk, len - j * kBlk) - 64 * sb)) : 0;
                    inf.ok = pg >= 0;
                    inf.pos = i;
                    info[st] = inf;
                    if (pg >= 0) {
                        uint8_t* base = dyn + (size_t)st * TG::kStage;
                        const int y = (pg * c.H_kv + h) * kBlk + 64 * sb;
                        mbar_arrive_expect_tx(&full[st], TG::kStage);
                        tma_load_2d(base, &tmK, &full[st], 0, y);
                        tma_load_2d(base + TG::kHalf, &tmK, &full[st], 64, y);
                        tma_load_2d(base + 2 * TG::kHalf, &tmV, &full[st], 0, y);
                        tma_load_2d(base + 3 * TG::kHalf, &tmV, &full[st], 64, y);
                    } else {
                        if (sb == 0) report(c.status, SBA_DEV_BAD_SELECTION);
                        mbar_arrive(&full[st]);
                    }
                }
                __syncwarp();
            }
        }
        // touched blocks whose first fill's stage was not reused in the loop
        for (uint32_t prev = max(fill0, fill >= (uint32_t)NSt ? fill - NSt : 0u); prev < fill; ++prev) {
            if (!alive || (prev - fill0) % kSub != 0) continue;
            const int ip = i0 + (int)((prev - fill0) / kSub);
            if (touched(ip)) refresh(ip);
        }
        named_sync(4, kThreads);  // the ring becomes the merge area
    } else {
        uint32_t qb[kNH][8][2];
        load_q_frags_t<kNH>(qb, a.q + ((int64_t)s * c.H_q + h * G) * kHeadDim, G, lane);
        const int t4 = lane & 3;                      // this lane's heads: 8nh + 2*t4 + x
        const int grp = warp / kGW, gw = warp % kGW;  // consumer group, token slot
        DecodeStateT<kNH> dst;
        decode_state_init_t<kNH>(dst);
        bool alive = true;
        for (int fi = 0; fi < (i1 - i0) * kSub; ++fi, ++fill) {
            if ((int)(fill & 1) != grp) continue;  // the other group's fill
            const int st = fill % NSt;
            if (alive) {
                alive = mbar_wait(&full[st], (fill / NSt) & 1, c.status);
                // a wait that ran out leaves this warp's partial empty: after a timeout (reported
                // in the status word) the merge sees no tokens from it rather than a stale stage
                if (!alive) decode_state_init_t<kNH>(dst);
            }
            const StageInfo inf = alive ? info[st] : StageInfo{0, 0, 0, 0};
            uint8_t* stage = dyn + (size_t)st * TG::kStage;
            if (inf.ok) {
                // SAS log-gate of this block (natural log) for this lane's heads, 0 for the current
                // block B0
                float gb[kNH][2];
#pragma unroll
                for (int nh = 0; nh < kNH; ++nh) gb[nh][0] = gb[nh][1] = 0.f;
                if (kScorer == SBA_SCORER_GATE && inf.j != N - 1) {
                    const int owner = inf.j / slice, off = inf.j - owner * slice;
#pragma unroll
                    for (int nh = 0; nh < kNH; ++nh)
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            const int hd = nh * 8 + 2 * t4 + x;
                            if (hd < G) gb[nh][x] = log_gate_of(ld_peer_f32(peer_addr(u_s + hd * ustride + off, owner)),
                                                                lse_s[hd], a.p.gate_act);
                        }
                }
                if (kScorer == SBA_SCORER_GATE && a.gate_bias && gw == 0 && lane < 4 && inf.pos < a.n_max &&
                    fi % kSub == 0) {
#pragma unroll
                    for (int nh = 0; nh < kNH; ++nh)
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            const int hd = nh * 8 + 2 * t4 + x;
                            if (hd < G) a.gate_bias[((int64_t)s * c.H_q + h * G + hd) * a.n_max + inf.pos] = gb[nh][x];
                        }
                }
                // the gate in the attention: inside the softmax, on the values, or not at all
                const float gsc = (kScorer == SBA_SCORER_GATE && a.p.log_gate != SBA_LOG_GATE_OFF) ? kLog2e : 0.f;
#pragma unroll
                for (int nh = 0; nh < kNH; ++nh) gb[nh][0] *= gsc, gb[nh][1] *= gsc;
                decode_block_t<kNH>(dst, qb, stage, inf.valid, gb, a.scale_log2, gw, lane,
                                    kScorer == SBA_SCORER_GATE && a.p.log_gate == SBA_LOG_GATE_OUTER);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        named_sync(4, kThreads);  // every consumer (and the producer) is done with the ring: it becomes the merge area
        decode_state_store_t<kNH>(dst, merge_o, merge_ml, warp, lane, G);
        named_sync(3, kCW * 32);
        // per query row: the weight of each consumer warp's partial and the row's LSE over this
        // CTA's blocks (pushed to every CTA); kCW consecutive lanes per row
        if (warp < (G * kCW + 31) / 32) {  // whole warps: every lane takes part in the shuffles
            const int row = tid / kCW, w = tid % kCW;
            const bool act = row < G;  // (rows come in groups of kCW lanes)
            const float mw = act ? merge_ml[(w * 16 + row) * 2] : -INFINITY;
            const float lw = act ? merge_ml[(w * 16 + row) * 2 + 1] : 0.f;
            float M = mw;
#pragma unroll
            for (int o = 1; o < kCW; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            float ls = f * lw;
#pragma unroll
            for (int o = 1; o < kCW; o <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            if (act) {
                wgt_s[row][w] = ls > 0.f ? f / ls : 0.f;
                const float lse = ls > 0.f ? (M + log2f(ls)) * kLn2 : -INFINITY;
                for (int p = w; p < C; p += kCW) st_peer_f32(peer_addr(&lse_all[r * G + row], p), lse);
            }
        }
        named_sync(3, kCW * 32);
        // this CTA's normalised partial O of every element, pushed to the element's merging CTA
        for (int e = tid; e < E; e += kCW * 32) {
            const int row = e / kHeadDim, ch = e % kHeadDim;
            const float4 w0 = *reinterpret_cast<const float4*>(&wgt_s[row][0]);
            const float4 w1 = *reinterpret_cast<const float4*>(&wgt_s[row][4]);
            const float* mo = merge_o + row * kMergeStride + ch;
            float o = w0.x * mo[0];
            o = fmaf(w0.y, mo[1 * 16 * kMergeStride], o);
            o = fmaf(w0.z, mo[2 * 16 * kMergeStride], o);
            o = fmaf(w0.w, mo[3 * 16 * kMergeStride], o);
            o = fmaf(w1.x, mo[4 * 16 * kMergeStride], o);
            o = fmaf(w1.y, mo[5 * 16 * kMergeStride], o);
            o = fmaf(w1.z, mo[6 * 16 * kMergeStride], o);
            o = fmaf(w1.w, mo[7 * 16 * kMergeStride], o);
            const int p = e / share;
            st_peer_f32(peer_addr(recv_o + r * share + (e - p * share), p), o);
        }
    }

    // ---------------- phase 4: merge the cluster's partials (local data only) ----------------
    cluster_sync();  // every partial pushed; no shared memory is read remotely after this
    {
        // the weight of every CTA's partial in each row of my share (16 lanes per row, lane p for
        // CTA p), then every element of the share as the weighted sum of the C partials
        const int e0 = r * share, e1 = min(e0 + share, E);
        const int rw0 = e0 / kHeadDim, nrw = e1 > e0 ? (e1 - 1) / kHeadDim - rw0 + 1 : 0;
        for (int rp = warp; 2 * rp < nrw; rp += kThreads / 32) {  // (warp-uniform: whole warps shuffle)
            const int rl = 2 * rp + (lane >> 4), p = lane & 15;
            const float l = (rl < nrw && p < C) ? lse_all[p * G + rw0 + rl] : -INFINITY;
            float M = l;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            const float w = M > -INFINITY ? expf(l - M) : 0.f;
            float W = w;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
            if (rl < nrw) {
                cw_s[rl][p] = W > 0.f ? w / W : 0.f;
                if (p == 0) rlse_s[rl] = W > 0.f ? M + logf(W) : -INFINITY;
            }
        }
        __syncthreads();
        for (int e = e0 + tid; e < e1; e += kThreads) {
            const int row = e / kHeadDim, ch = e % kHeadDim, rl = row - rw0;
            float o = 0.f;
#pragma unroll
            for (int p = 0; p < kMaxCluster; ++p)
                if (p < C) o = fmaf(cw_s[rl][p], recv_o[p * share + (e - e0)], o);
            const int64_t orow = (int64_t)s * c.H_q + h * G + row;
            if (a.out_dtype == SBA_OUT_BF16)
                reinterpret_cast<__nv_bfloat16*>(a.out)[orow * kHeadDim + ch] = __float2bfloat16_rn(o);
            else
                reinterpret_cast<float*>(a.out)[orow * kHeadDim + ch] = o;
            if (ch == 0 && a.lse_out) a.lse_out[orow] = rlse_s[rl];
        }
    }
    if (kScorer == SBA_SCORER_GATE && tile_refresh && N >= 1 && tb1 == N - 1) {
        // gate key of the refreshed current block: CTA r computes its channels of kg = A pooled
        const int c0 = kHeadDim * r / C, c1 = kHeadDim * (r + 1) / C;
        const int pg = page_quiet(c, s, N - 1);
        for (int ch = c0 + warp; ch < c1; ch += kThreads / 32) {
            const float* Ar = a.gate_A + (int64_t)ch * 3 * kHeadDim;
            float acc = 0.f;
            for (int i = lane; i < 3 * kHeadDim; i += 32) acc = fmaf(__ldg(Ar + i), pooled_b0[i], acc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0 && pg >= 0) c.kg[((int64_t)pg * c.H_kv + h) * kHeadDim + ch] = acc;
        }
    }
}

// A = Wq^T Wk / sqrt(dg): the gate projection folded into query space.
__global__ void fold_gate_kernel(const float* __restrict__ Wq, const float* __restrict__ Wk, int dg, float* A) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // over 128 x 384
    if (idx >= kHeadDim * 3 * kHeadDim) return;
    const int ch = idx / (3 * kHeadDim), i = idx % (3 * kHeadDim);
    float acc = 0.f;
    for (int r = 0; r < dg; ++r) acc = fmaf(__ldg(Wq + (int64_t)r * kHeadDim + ch), __ldg(Wk + (int64_t)r * 3 * kHeadDim + i), acc);
    A[idx] = acc * rsqrtf((float)dg);
}

struct Plan {
    int C, n_stages, smem, slice, ccap, sel_cap;
    int off_keys, off_pages, off_u, off_kall, off_gm, off_crank, off_sel, off_selp, off_recv, off_bars;
};

int round4(int x) { return (x + 3) & ~3; }

Plan plan_step(const sba_cache& c, const sba_select_params& p, int C, int n_max_sel) {
    Plan pl{};
    pl.C = C;
    const int G = c.H_q / c.H_kv;
    const int stage = 64 * kDescBytes;  // a ring stage: 64 tokens of K and V, or 64 descriptors
    pl.slice = round4((c.max_blocks + C - 1) / C);
    pl.ccap = 1024;
    pl.sel_cap = round4(n_max_sel);
    const int E = G * kHeadDim;
    int off = 0;
    auto take = [&](int words) {
        const int o = off;
        off += round4(words) * 4;
        return o;
    };
    // the ring comes first (1024-aligned); the fallback selection reuses it
    const int min_stages = (kCW * 16 * kMergeStride * 4 + kCW * 16 * 2 * 4 + stage - 1) / stage + 1;
    int ns = 6;
    const int mb128 = (c.max_blocks + 127) & ~127;
    const int kall_words = p.scorer == SBA_SCORER_GATE ? 0 : mb128 + 4;  // (the gate's keys use the ring)
    const int gm_words = C * round4((pl.slice + 3) / 4) + 64;
    const int fixed_bytes = 4 * (round4(pl.slice) * 2 + (p.scorer == SBA_SCORER_GATE ? G * pl.slice : 0) + kall_words +
                                 gm_words + pl.ccap + 2 * pl.sel_cap + round4(C * ((E + C - 1) / C)) + 64);
    const int budget = 227 * 1024 - 1024 /*align*/ - 10 * 1024 /*static shared memory headroom*/;
    while (ns > max(2, min_stages) && ns * stage + fixed_bytes + ns * (16 + (int)sizeof(StageInfo)) > budget) --ns;
    pl.n_stages = ns;
    off = ns * stage;
    pl.off_keys = take(pl.slice);
    pl.off_pages = take(pl.slice);
    pl.off_u = take(p.scorer == SBA_SCORER_GATE ? G * pl.slice : 0);
    pl.off_kall = take(kall_words);
    pl.off_gm = take(gm_words);
    pl.off_crank = take(pl.ccap);
    pl.off_sel = take(pl.sel_cap);
    pl.off_selp = take(pl.sel_cap);
    pl.off_recv = take(C * ((E + C - 1) / C));
    pl.off_bars = off;
    pl.smem = pl.off_bars + ns * (16 + (int)sizeof(StageInfo)) + 1024;
    // the selection keeps the candidates (or the fallback's scratch) in the ring, after the
    // gate's keys
    const int sel_words = (p.scorer == SBA_SCORER_GATE ? mb128 : 0) +
                          max(2 * (pl.ccap + 32), c.max_blocks / 4 + 16 + 3 * 1024);
    if (sel_words * 4 > ns * stage) pl.smem = 1 << 30;
    return pl;
}

template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
cudaError_t prepare_kernel(int smem) {
    auto kern = decode_step_kernel<kBlk, kScorer, kGM, kNH, kPaged>;
    if (allow_smem<decode_step_kernel<kBlk, kScorer, kGM, kNH, kPaged>>(smem) != SBA_OK) return cudaErrorInvalidValue;
    static bool nonportable_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !nonportable_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        nonportable_set[dev] = true;
    }
    return cudaSuccess;
}

cudaLaunchConfig_t step_config(const sba_cache& c, const Plan& pl, cudaStream_t stream, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.C, c.H_kv, c.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cfg;
}

// Clusters of this size the device can keep resident at once (0 if none).
template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
int active_clusters(const sba_cache& c, const Plan& pl) {
    if (prepare_kernel<kBlk, kScorer, kGM, kNH, kPaged>(pl.smem) != cudaSuccess) return 0;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = step_config(c, pl, nullptr, attr);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, decode_step_kernel<kBlk, kScorer, kGM, kNH, kPaged>, &cfg) != cudaSuccess) return 0;
    return active;
}

template <bool kPaged, class F>
int dispatch_shape(const sba_cache& c, const sba_select_params& p, F&& f) {
    const int G = c.H_q / c.H_kv;
    if (p.scorer == SBA_SCORER_QUEST)
        return G <= 8 ? (c.b == 64 ? f.template run<64, SBA_SCORER_QUEST, 1, 1, kPaged>()
                                   : f.template run<128, SBA_SCORER_QUEST, 1, 1, kPaged>())
                      : (c.b == 64 ? f.template run<64, SBA_SCORER_QUEST, 1, 2, kPaged>()
                                   : f.template run<128, SBA_SCORER_QUEST, 1, 2, kPaged>());
    if (G <= 4)
        return c.b == 64 ? f.template run<64, SBA_SCORER_GATE, 4, 1, kPaged>()
                         : f.template run<128, SBA_SCORER_GATE, 4, 1, kPaged>();
    if (G <= 8)
        return c.b == 64 ? f.template run<64, SBA_SCORER_GATE, 8, 1, kPaged>()
                         : f.template run<128, SBA_SCORER_GATE, 8, 1, kPaged>();
    return c.b == 64 ? f.template run<64, SBA_SCORER_GATE, 16, 2, kPaged>()
                     : f.template run<128, SBA_SCORER_GATE, 16, 2, kPaged>();
}

// Kernel instantiation for a cache shape: block size, scorer, (gate) the head count rounded
// up to a power of two, and whether pages go through a block table (each variant holds only
// the scoring path it runs).
template <class F>
int dispatch(const sba_cache& c, const sba_select_params& p, F&& f) {
    return c.block_table != nullptr ? dispatch_shape<true>(c, p, f) : dispatch_shape<false>(c, p, f);
}

struct ActiveClusters {
    const sba_cache& c;
    const Plan& pl;
    template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
    int run() {
        return active_clusters<kBlk, kScorer, kGM, kNH, kPaged>(c, pl);
    }
};

int active_clusters_any(const sba_cache& c, const sba_select_params& p, const Plan& pl) {
    return dispatch(c, p, ActiveClusters{c, pl});
}

template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
int launch_step_t(const sba_cache& c, const StepArgs& a0, const Plan& pl, cudaStream_t stream) {
    CUtensorMap tk, tv, td;
    const uint64_t rows = (uint64_t)c.num_pages * c.H_kv * kBlk;
    // boxes of 64 rows: 64 tokens of a (page, head) tile, or 64 descriptors
    if (!make_kv_tmap(&tk, c.k, rows, 64) || !make_kv_tmap(&tv, c.v, rows, 64)) return SBA_ERR_CUDA;
    if (!make_desc_tmap(&td, kScorer == SBA_SCORER_QUEST ? c.desc : (void*)c.kg, (uint64_t)c.num_pages, c.H_kv, 64))
        return SBA_ERR_CUDA;
    cudaError_t e = prepare_kernel<kBlk, kScorer, kGM, kNH, kPaged>(pl.smem);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    StepArgs a = a0;
    a.n_stages = pl.n_stages;
    a.slice = pl.slice;
    a.off_keys = pl.off_keys;
    a.off_pages = pl.off_pages;
    a.off_u = pl.off_u;
    a.off_kall = pl.off_kall;
    a.off_gm = pl.off_gm;
    a.off_crank = pl.off_crank;
    a.off_sel = pl.off_sel;
    a.off_selp = pl.off_selp;
    a.off_recv = pl.off_recv;
    a.off_bars = pl.off_bars;
    a.ccap = pl.ccap;
    a.sel_cap = pl.sel_cap;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = step_config(c, pl, stream, attr);
    e = cudaLaunchKernelEx(&cfg, decode_step_kernel<kBlk, kScorer, kGM, kNH, kPaged>, tk, tv, td, a);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    return SBA_OK;
}

struct LaunchStep {
    const sba_cache& c;
    const StepArgs& a;
    const Plan& pl;
    cudaStream_t stream;
    template <int kBlk, int kScorer, int kGM, int kNH, bool kPaged>
    int run() {
        return launch_step_t<kBlk, kScorer, kGM, kNH, kPaged>(c, a, pl, stream);
    }
};

int n_max_selected(const sba_cache& c, const sba_select_params& p) {
    const int N_max = (c.max_len + c.b - 1) / c.b;
    return num_selected(N_max, p) > 0 ? num_selected(N_max, p) : 1;
}

}  // namespace

int step_cluster_size_uncached(const sba_cache& c, const sba_select_params& p, int num_sms) {
    // one CTA per SM: the largest C <= 16 with B*H_kv*C <= #SMs whose clusters are all
    // resident at once; failing that, the largest schedulable C
    const int64_t units = (int64_t)c.B * c.H_kv;
    int start = kMaxCluster;
    while (start > 1 && units * start > num_sms) --start;
    for (int pass = 0; pass < 2; ++pass)
        for (int C = start; C >= 1; --C) {
            const Plan pl = plan_step(c, p, C, n_max_selected(c, p));
            if (pl.smem > 227 * 1024) return 0;
            const int active = active_clusters_any(c, p, pl);
            if (active >= 1 && (pass == 1 || C == 1 || active >= units)) return C;
        }
    return 0;
}

// The choice above costs occupancy queries; it depends only on the device and the shapes, so
// it is remembered (a small table, most recent first).
int step_cluster_size(const sba_cache& c, const sba_select_params& p, int num_sms) {
    struct Key {
        int dev, sms, B, H_q, H_kv, b, max_blocks, max_len, n_budget, n_local, n_min, keep_num, keep_den, scorer;
        bool operator==(const Key& o) const { return memcmp(this, &o, sizeof(Key)) == 0; }
    };
    static std::mutex mu;
    static Key keys[16];
    static int vals[16];
    static int n = 0;
    Key k;
    memset(&k, 0, sizeof(k));
    if (cudaGetDevice(&k.dev) != cudaSuccess) return 0;
    k.sms = num_sms;
    k.B = c.B;
    k.H_q = c.H_q;
    k.H_kv = c.H_kv;
    k.b = c.b;
    k.max_blocks = c.max_blocks;
    k.max_len = c.max_len;
    k.n_budget = p.n_budget;
    k.n_local = p.n_local;
    k.n_min = p.n_min;
    k.keep_num = p.keep_num;
    k.keep_den = p.keep_den;
    k.scorer = p.scorer;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < n; ++i)
            if (keys[i] == k) return vals[i];
    }
    const int C = step_cluster_size_uncached(c, p, num_sms);
    if (C > 0) {
        std::lock_guard<std::mutex> lock(mu);
        const int slot = n < 16 ? n++ : 15;
        for (int i = slot; i > 0; --i) {
            keys[i] = keys[i - 1];
            vals[i] = vals[i - 1];
        }
        keys[0] = k;
        vals[0] = C;
    }
    return C;
}

int launch_decode_step(const sba_cache& c, const void* q, const void* k_new, const void* v_new,
                       const int32_t* pos_start, int n_new, const float* gate_A, const sba_select_params& p,
                       float scale, void* out, int out_dtype, float* lse_out, int32_t* sel_idx, int32_t* sel_cnt,
                       float* gate_bias, int n_max, int cluster, cudaStream_t stream) {
    if (cluster < 1) return SBA_ERR_UNSUPPORTED;
    const Plan pl = plan_step(c, p, cluster, n_max_selected(c, p));
    if (pl.smem > 227 * 1024) return SBA_ERR_UNSUPPORTED;
    StepArgs a{};
    a.c = c;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.k_new = reinterpret_cast<const uint4*>(k_new);
    a.v_new = reinterpret_cast<const uint4*>(v_new);
    a.pos_start = pos_start;
    a.n_new = n_new;
    a.gate_A = gate_A;
    a.p = p;
    a.scale_log2 = scale * kLog2e;
    a.out = out;
    a.out_dtype = out_dtype;
    a.lse_out = lse_out;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.gate_bias = gate_bias;
    a.n_max = n_max;
    return dispatch(c, p, LaunchStep{c, a, pl, stream});
}

int launch_fold_gate(const float* Wq, const float* Wk, int dg, float* A, cudaStream_t stream) {
    const int n = kHeadDim * 3 * kHeadDim;
    return launch(fold_gate_kernel, dim3((n + 255) / 256), dim3(256), 0, stream, Wq, Wk, dg, A);
}

}  // namespace sba
