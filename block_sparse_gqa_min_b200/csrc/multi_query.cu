// Several query tokens per sequence sharing one block selection.
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation",
// Summary and Key points: all query heads of a GQA group share one block
// selection, and ReSA is compared with sparse-KV self-speculative decoding,
// which checks several draft tokens with one sparse pass.  The M query tokens
// of a sequence sit at its last M positions (len-M .. len-1), token i attends
// causally to positions t <= len-M+i of the group's selected blocks (ranked by
// the Quest score summed over the group's heads and the M tokens,
// sba_score_select_multi), and every one of the M*G query rows of a
// (sequence, KV group) reads each staged K/V tile once.  (The dense causal
// pass over every block, the rectification, runs on the tcgen05 tensor cores
// in rect_tc.cu.)
//
// One CTA per (split, KV head x row group, sequence).  A row group is up to
// 128 query rows (row r of a group = token r / G, head r % G), i.e. 8 tiles of
// 16 rows for the bf16 tensor cores (mma.sync m16n8k16, fp32 accumulate).
// Warp 8..: a producer warp streams each block's K and V tiles in 64-token
// stages (four 2-D TMA loads of 64 rows x 128 B, 128-byte swizzle, no
// multicast) into a ring of 32 KB stages guarded by full/empty mbarriers.
// Consumer warp w owns row tile w / TS and every TS-th 16-token chunk of each
// stage (TS = 4, 2 or 1 token slots so that up to 8 consumers are busy); it
// keeps an online base-2 softmax and O (16 rows x 128) in registers, P entering
// PV as bf16 hi + lo parts (about 16 mantissa bits).  The token slots of a row
// tile are merged in shared memory and the split's normalised O and LSE are
// written as [B][M][H_q][S][d] and [B][M][H_q][S], so sba_combine over
// M*H_q rows merges the splits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "decode_tile.cuh"
#include "launch.cuh"

namespace sba {

bool make_kv_tmap(CUtensorMap* m, void* base, uint64_t rows, int blk);  // decode.cu

namespace {

constexpr int kRowsPerCta = 128;           // 8 row tiles of 16
constexpr int kTcRows = 64;                // query rows per group from which the tcgen05 kernel serves the call
constexpr int kMaxConsumers = 8;
constexpr int kMqThreads = (kMaxConsumers + 1) * 32;
constexpr int kMqStages = 6;
constexpr int kMqStage = 32768;            // 64 tokens: K0 K1 V0 V1 halves of 64 rows x 128 B
constexpr int kMqHalf = 8192;
constexpr int kMqSmem = kMqStages * kMqStage + 1024 + 256;

struct MqArgs {
    sba_cache c;
    const __nv_bfloat16* q;  // [B][M][H_q][d]
    int M;
    const int32_t* sel_idx;  // [B][H_kv][n_max]
    const int32_t* sel_cnt;  // [B][H_kv]
    int n_max;
    float scale_log2;
    int num_splits;
    int row_groups;          // CTAs along the M*G query rows of a group
    float* o_part;           // [B][M][H_q][S][d]
    float* lse_part;         // [B][M][H_q][S]
};

struct MqStage {
    int j;      // logical block
    int sb;     // 64-token half of a 128-token block
    int valid;  // tokens of the stage below len
    int ok;
};

struct MqState {
    float o[16][4];
    float m0, m1;  // running max (log2 units) of rows r, r+8
    float l0, l1;
};

// 16 tokens [tok0, tok0 + 16) of a staged 64-token tile for this warp's 16 query rows:
// S = Q K^T, per-row causal limits (lim0, lim1: exclusive, relative to the stage start),
// online softmax, O += P V.
__device__ __forceinline__ void mq_chunk16(MqState& st, const uint32_t (&qa)[8][4], uint32_t kb, uint32_t vb, int tok0,
                                           int lim0, int lim1, float scale_log2, int lane) {
    const int cq = (lane & 3) * 2;
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int row = tok0 + nt * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
            const int chunk = 4 * kp + (lane >> 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(swz(kb + (chunk >> 3) * kMqHalf, row, chunk & 7), b0, b1, b2, b3);
            mma_bf16_16816(sc[nt], qa[2 * kp], b0, b1);
            mma_bf16_16816(sc[nt], qa[2 * kp + 1], b2, b3);
        }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int t = tok0 + nt * 8 + cq;
        sc[nt][0] = t < lim0 ? sc[nt][0] * scale_log2 : -INFINITY;
        sc[nt][1] = t + 1 < lim0 ? sc[nt][1] * scale_log2 : -INFINITY;
        sc[nt][2] = t < lim1 ? sc[nt][2] * scale_log2 : -INFINITY;
        sc[nt][3] = t + 1 < lim1 ? sc[nt][3] * scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(st.m0, mx0), n1 = fmaxf(st.m1, mx1);
    const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
    const float al0 = exp2f(st.m0 - u0), al1 = exp2f(st.m1 - u1);
    st.m0 = n0;
    st.m1 = n1;
    st.l0 *= al0;
    st.l1 *= al1;
    if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            st.o[n][0] *= al0;
            st.o[n][1] *= al0;
            st.o[n][2] *= al1;
            st.o[n][3] *= al1;
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = exp2f(sc[nt][0] - u0);
        sc[nt][1] = exp2f(sc[nt][1] - u0);
        sc[nt][2] = exp2f(sc[nt][2] - u1);
        sc[nt][3] = exp2f(sc[nt][3] - u1);
        st.l0 += sc[nt][0] + sc[nt][1];
        st.l1 += sc[nt][2] + sc[nt][3];
    }
    // O += P V: P (16 rows x 16 tokens) as the A operand, bf16 hi + lo
    uint32_t ph[4], pl[4];
    const float pv[8] = {sc[0][0], sc[0][1], sc[0][2], sc[0][3], sc[1][0], sc[1][1], sc[1][2], sc[1][3]};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(pv[2 * e], pv[2 * e + 1]);
        const float2 hf = __bfloat1622float2(hi);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(pv[2 * e] - hf.x, pv[2 * e + 1] - hf.y);
        ph[e] = *reinterpret_cast<const uint32_t*>(&hi);
        pl[e] = *reinterpret_cast<const uint32_t*>(&lo);
    }
    const int row = tok0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int np = 0; np < 8; ++np) {
        const int chunk = 2 * np + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(swz(vb + (chunk >> 3) * kMqHalf, row, chunk & 7), b0, b1, b2, b3);
        mma_bf16_16816(st.o[2 * np], ph, b0, b1);
        mma_bf16_16816(st.o[2 * np], pl, b0, b1);
        mma_bf16_16816(st.o[2 * np + 1], ph, b2, b3);
        mma_bf16_16816(st.o[2 * np + 1], pl, b2, b3);
    }
}

template <int kBlk>
__global__ void __launch_bounds__(kMqThreads, 1)
    mq_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ MqArgs a) {
    constexpr int kSub = kBlk / 64;
    extern __shared__ uint8_t dyn_raw[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kMqStages], empty[kMqStages], zbar;
    __shared__ MqStage info[kMqStages];
    __shared__ float ml_s[kMaxConsumers][16][2];

    const sba_cache& c = a.c;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = blockIdx.x, h = blockIdx.y % c.H_kv, rg = blockIdx.y / c.H_kv, s = blockIdx.z;
    const int G = c.H_q / c.H_kv;
    const int R = a.M * G;                                  // query rows of the group
    const int row0 = rg * kRowsPerCta;                      // this CTA's first row
    const int rows = max(0, min(kRowsPerCta, R - row0));
    const int RT = (rows + 15) / 16;                        // row tiles
    const int TS = RT <= 2 ? 4 : (RT <= 4 ? 2 : 1);         // token slots per row tile
    const int NCW = max(1, RT * TS);                        // consumer warps (<= 8)
    const int producer = kMaxConsumers;                     // warp index of the producer

    if (tid == 0) {
        for (int i = 0; i < kMqStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NCW);
        }
        mbar_init(&zbar, 1);
        fence_mbar_init();
    }
    if (warp == producer && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    int len = __ldg(c.seq_lens + s);
    int N = blocks_of(len, kBlk);
    if (N > c.max_blocks) {
        if (tid == 0 && sp == 0 && blockIdx.y == 0) report(c.status, SBA_DEV_BAD_POSITION);
        N = c.max_blocks;
        len = N * kBlk;
    }
    const int pos0 = len - a.M;  // first query token's position
    // the group's selection
    int cnt = __ldg(a.sel_cnt + s * c.H_kv + h);
    if (cnt > a.n_max || cnt < 0) {
        if (tid == 0 && sp == 0 && rg == 0) report(c.status, SBA_DEV_BAD_SELECTION);
        cnt = cnt < 0 ? 0 : a.n_max;
    }
    const int32_t* sel = a.sel_idx + ((int64_t)s * c.H_kv + h) * a.n_max;
    const int i0 = (int)((int64_t)cnt * sp / a.num_splits), i1 = (int)((int64_t)cnt * (sp + 1) / a.num_splits);
    const int nfill = (i1 - i0) * kSub;

    const bool consumer = warp < NCW && rows > 0;
    MqState stt;  // a consumer warp's 16 rows (registers), stored for the merge at the end
    if (warp == producer) {
        // ------------------------------ producer ------------------------------
        bool alive = true;
        uint32_t zpar = 0;
        for (int f = 0; f < nfill && alive; ++f) {
            const int i = i0 + f / kSub, sb = f % kSub;
            const int st = f % kMqStages;
            if (f >= kMqStages) {
                if (lane == 0) alive = mbar_wait(&empty[st], ((f / kMqStages) - 1) & 1, c.status);
                alive = __shfl_sync(0xffffffffu, alive, 0);
                if (!alive) break;
            }
            const int j = __ldg(sel + i);
            int pg = -1;
            if (j >= 0 && j < N) {
                pg = (int)page_of(c, s, j, lane == 0 ? c.status : nullptr);
            } else if (lane == 0 && sb == 0) {
                report(c.status, SBA_DEV_BAD_SELECTION);
            }
            const int valid = pg >= 0 ? min(64, max(0, len - j * kBlk - 64 * sb)) : 0;
            if (valid == 0) {
                if (lane == 0) {
                    info[st] = MqStage{j, sb, 0, 0};
                    mbar_arrive(&full[st]);
                }
                __syncwarp();
                continue;
            }
            if (lane == 0) {
                info[st] = MqStage{j, sb, valid, 1};
                uint8_t* base = dyn + (size_t)st * kMqStage;
                const int y = (pg * c.H_kv + h) * kBlk + 64 * sb;
                uint64_t* bar = valid == 64 ? &full[st] : &zbar;
                mbar_arrive_expect_tx(bar, kMqStage);
                tma_load_2d(base, &tmK, bar, 0, y);
                tma_load_2d(base + kMqHalf, &tmK, bar, 64, y);
                tma_load_2d(base + 2 * kMqHalf, &tmV, bar, 0, y);
                tma_load_2d(base + 3 * kMqHalf, &tmV, bar, 64, y);
            }
            if (valid < 64) {
                // rows past len may hold anything (NaN included): zero them in the stage before the
                // consumers see it, so that a zero probability never meets a non-finite value
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&zbar, zpar, c.status);
                zpar ^= 1u;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                uint8_t* base = dyn + (size_t)st * kMqStage;
                for (int e = lane; e < (64 - valid) * 32 && ok; e += 32) {
                    const int r = valid + (e >> 5), part = (e >> 4) & 1, ch = e & 15;  // part: K or V
                    *reinterpret_cast<uint4*>(base + (2 * part + (ch >> 3)) * kMqHalf + r * 128 + ((ch & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[st]);
                if (!ok) alive = false;
            }
            __syncwarp();
        }
    } else if (consumer) {
        // ------------------------------ consumers -----------------------------
        const int rt = warp / TS, ts = warp % TS;
        const int r0 = row0 + rt * 16 + (lane >> 2);  // this lane's rows r0 and r0 + 8 of the group
        const int cq = (lane & 3) * 2;
        // Q rows as m16n8k16 A fragments (zero past the group's rows)
        uint32_t qa[8][4];
        const __nv_bfloat16* qrow[2];
        int lim[2];  // exclusive causal limit (absolute position) of each row; 0 for padding rows
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int r = r0 + 8 * x;
            if (r < R) {
                const int ti = r / G, g = r % G;
                qrow[x] = a.q + (((int64_t)s * a.M + ti) * c.H_q + h * G + g) * kHeadDim;
                lim[x] = pos0 + ti + 1;
            } else {
                qrow[x] = nullptr;
                lim[x] = 0;
            }
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int c0 = ks * 16 + cq;
            qa[ks][0] = qrow[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + c0) : 0u;
            qa[ks][1] = qrow[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + c0) : 0u;
            qa[ks][2] = qrow[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + c0 + 8) : 0u;
            qa[ks][3] = qrow[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + c0 + 8) : 0u;
        }
        const int lim_hi = __reduce_max_sync(0xffffffffu, max(lim[0], lim[1]));  // the tile's furthest row
#pragma unroll
        for (int n = 0; n < 16; ++n) stt.o[n][0] = stt.o[n][1] = stt.o[n][2] = stt.o[n][3] = 0.f;
        stt.m0 = stt.m1 = -INFINITY;
        stt.l0 = stt.l1 = 0.f;
        bool alive = true;
        for (int f = 0; f < nfill; ++f) {
            const int st = f % kMqStages;
            if (alive) {
                alive = mbar_wait(&full[st], (f / kMqStages) & 1, c.status);
                if (!alive) {  // a wait that ran out (reported): this warp contributes nothing
                    stt.m0 = stt.m1 = -INFINITY;
                    stt.l0 = stt.l1 = 0.f;
                }
            }
            const MqStage inf = alive ? info[st] : MqStage{0, 0, 0, 0};
            if (inf.ok) {
                const int base = inf.j * kBlk + 64 * inf.sb;  // position of the stage's first token
                const uint32_t kb = smem_u32(dyn + (size_t)st * kMqStage);
                for (int ch = ts; ch < 4; ch += TS) {
                    const int tok0 = ch * 16;
                    if (tok0 >= inf.valid || base + tok0 >= lim_hi) break;  // beyond every row's horizon
                    mq_chunk16(stt, qa, kb, kb + 2 * kMqHalf, tok0, lim[0] - base, lim[1] - base, a.scale_log2,
                               lane);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        stt.l0 += __shfl_xor_sync(0xffffffffu, stt.l0, 1);
        stt.l0 += __shfl_xor_sync(0xffffffffu, stt.l0, 2);
        stt.l1 += __shfl_xor_sync(0xffffffffu, stt.l1, 1);
        stt.l1 += __shfl_xor_sync(0xffffffffu, stt.l1, 2);
    }
    __syncthreads();  // every consumer and the producer are done with the ring
    if (consumer) {
        // this warp's rows to shared memory (the ring) for the token-slot merge
        float* mo = reinterpret_cast<float*>(dyn) + warp * 16 * kHeadDim;
        const int rr = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            *reinterpret_cast<float2*>(mo + rr * kHeadDim + n * 8 + cq) = make_float2(stt.o[n][0], stt.o[n][1]);
            *reinterpret_cast<float2*>(mo + (rr + 8) * kHeadDim + n * 8 + cq) = make_float2(stt.o[n][2], stt.o[n][3]);
        }
        if ((lane & 3) == 0) {
            ml_s[warp][rr][0] = stt.m0;
            ml_s[warp][rr][1] = stt.l0;
            ml_s[warp][rr + 8][0] = stt.m1;
            ml_s[warp][rr + 8][1] = stt.l1;
        }
    }
    __syncthreads();
    // merge the TS token slots of every row and write the split's normalised O and LSE
    const float* mo_all = reinterpret_cast<const float*>(dyn);
    for (int e = tid; e < rows * kHeadDim; e += blockDim.x) {
        const int rl = e / kHeadDim, ch = e % kHeadDim;  // row within the CTA, channel
        const int rt = rl / 16, rr = rl % 16;
        float M = -INFINITY;
        for (int x = 0; x < TS; ++x) M = fmaxf(M, ml_s[rt * TS + x][rr][0]);
        float osum = 0.f, lsum = 0.f;
        if (M > -INFINITY)
            for (int x = 0; x < TS; ++x) {
                const int w = rt * TS + x;
                const float mw = ml_s[w][rr][0];
                const float fw = mw == -INFINITY ? 0.f : exp2f(mw - M);
                lsum += fw * ml_s[w][rr][1];
                osum += fw * mo_all[(w * 16 + rr) * kHeadDim + ch];
            }
        const int r = row0 + rl, ti = r / G, g = r % G;
        const int64_t orow = (((int64_t)s * a.M + ti) * c.H_q + h * G + g) * a.num_splits + sp;
        a.o_part[orow * kHeadDim + ch] = lsum > 0.f ? osum / lsum : 0.f;
        if (ch == 0) a.lse_part[orow] = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
    }
}

template <int kBlk>
int launch_mq_t(const sba_cache& c, const MqArgs& a, cudaStream_t stream) {
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)c.num_pages * c.H_kv * kBlk;
    if (!make_kv_tmap(&tk, c.k, rows, 64) || !make_kv_tmap(&tv, c.v, rows, 64)) return SBA_ERR_CUDA;
    if (allow_smem<mq_decode_kernel<kBlk>>(kMqSmem) != SBA_OK) return SBA_ERR_CUDA;
    dim3 grid(a.num_splits, c.H_kv * a.row_groups, c.B);
    return launch(mq_decode_kernel<kBlk>, grid, dim3(kMqThreads), kMqSmem, stream, tk, tv, a);
}

}  // namespace

int mq_row_groups(const sba_cache& c, int M) {
    const int R = M * (c.H_q / c.H_kv);
    return (R + kRowsPerCta - 1) / kRowsPerCta;
}

int launch_multi_query(const sba_cache& c, const void* q, int M, const int32_t* sel_idx, const int32_t* sel_cnt,
                       int n_max, float scale, int num_splits,
                       float* o_part, float* lse_part, cudaStream_t stream) {
    // from 64 query rows per group on, the tcgen05 pipeline (rect_tc.cu) takes the same call
    if (M * (c.H_q / c.H_kv) >= kTcRows)
        return launch_multi_query_tc(c, q, M, sel_idx, sel_cnt, n_max, scale, num_splits, o_part, lse_part, stream);
    MqArgs a{};
    a.c = c;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.M = M;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.n_max = n_max;
    a.scale_log2 = scale * kLog2e;
    a.num_splits = num_splits;
    a.row_groups = mq_row_groups(c, M);
    a.o_part = o_part;
    a.lse_part = lse_part;
    return c.b == 64 ? launch_mq_t<64>(c, a, stream) : launch_mq_t<128>(c, a, stream);
}

}  // namespace sba
