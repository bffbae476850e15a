// Per-block attention math of the sparse decode, shared by the split-KV
// decode kernel and the fused decode-step kernel.
//
// A consumer warp owns T = b/4 tokens of every K/V block staged in shared
// memory (128-byte TMA swizzle, two 64-channel halves per tensor).  The G query
// heads of the group are the 16 rows of bf16 tensor-core tiles (m16n8k16,
// fp32 accumulate, rows past G are zero): S = Q K^T, online base-2 softmax with
// the optional log-gate ("SAS ...", Method: softmax(q K^T + log g) V), then
// O += P V with P split into bf16 hi + lo parts (about 16 mantissa bits).
#pragma once

#include "common.cuh"

namespace sba {

constexpr int kDecodeConsumerWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int kBlk>
struct TileGeom {
    static constexpr int kHalf = kBlk * 128;   // one 64-channel half of a tile, bytes
    static constexpr int kStage = 4 * kHalf;   // K0 K1 V0 V1
    static constexpr int T = kBlk / kDecodeConsumerWarps;  // tokens per consumer warp
    static constexpr int NT = T / 8;                        // 8-token MMA n-tiles per warp
};

struct StageInfo {
    int j;      // logical block
    int valid;  // valid tokens in the block
    int ok;     // 1 if the tiles were loaded
    int pos;    // position of the block in the selection
};

__device__ __forceinline__ uint32_t swz(uint32_t half_base, int row, int chunk) {
    // 128-byte TMA swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7)
    return half_base + row * 128 + ((chunk ^ (row & 7)) << 4);
}

struct DecodeState {
    float o[16][4];
    float m0, m1;  // running max (log2 units) of rows r, r+8
    float l0, l1;  // this thread's partial sums of rows r, r+8
};

__device__ __forceinline__ void decode_state_init(DecodeState& st) {
#pragma unroll
    for (int n = 0; n < 16; ++n) st.o[n][0] = st.o[n][1] = st.o[n][2] = st.o[n][3] = 0.f;
    st.m0 = st.m1 = -INFINITY;
    st.l0 = st.l1 = 0.f;
}

// Q of the group (rows = query heads, zero past G) as m16n8k16 A fragments.
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[8][4], const __nv_bfloat16* qb, int G, int lane) {
    const int r = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const int c0 = ks * 16 + cq;
        qa[ks][0] = r < G ? *reinterpret_cast<const uint32_t*>(qb + r * kHeadDim + c0) : 0u;
        qa[ks][1] = r + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (r + 8) * kHeadDim + c0) : 0u;
        qa[ks][2] = r < G ? *reinterpret_cast<const uint32_t*>(qb + r * kHeadDim + c0 + 8) : 0u;
        qa[ks][3] = r + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (r + 8) * kHeadDim + c0 + 8) : 0u;
    }
}

// One staged block: the T tokens of token slot `slot` (0..3).  `stage` is the generic pointer of
// the stage, `valid` the block's valid token count, g0/g1 the log-gates of
// rows r and r+8 (already in log2 units): added to the logits, or with kOuter
// ("SAS ...", Method: the gate outside the softmax) left out of the logits and
// instead multiplied, as g = 2^g, into the weights of the values.
template <int kBlk, bool kOuter = false>
__device__ __forceinline__ void decode_block(DecodeState& st, const uint32_t (&qa)[8][4], uint8_t* stage, int valid,
                                             float g0, float g1, float scale_log2, int slot, int lane) {
    using TG = TileGeom<kBlk>;
    constexpr int T = TG::T, NT = TG::NT;
    const int tok0 = slot * T;  // this warp's tokens: slot 0..3 of the block
    if (tok0 >= valid) return;
    const int cq = (lane & 3) * 2;
    const uint32_t kb = smem_u32(stage);
    const uint32_t vb = kb + 2 * TG::kHalf;
    if (valid < tok0 + T) {
        // rows past len may hold anything: zero this warp's invalid V rows so 0*garbage cannot appear
        uint8_t* vrow = stage + 2 * TG::kHalf;
        for (int e = lane; e < (tok0 + T - valid) * 16; e += 32) {
            const int row = valid + e / 16, ch = e % 16;
            *reinterpret_cast<uint4*>(vrow + (ch >> 3) * TG::kHalf + row * 128 + ((ch & 7) << 4)) =
                make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
    }
    // ---- S = Q K^T (16 x T) ----
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int row = tok0 + nt * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
            const int chunk = 4 * kp + (lane >> 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(swz(kb + (chunk >> 3) * TG::kHalf, row, chunk & 7), b0, b1, b2, b3);
            mma_bf16_16816(sc[nt], qa[2 * kp], b0, b1);
            mma_bf16_16816(sc[nt], qa[2 * kp + 1], b2, b3);
        }
    }
    // ---- scale, log-gate, mask, online softmax (base 2) ----
    const float b0 = kOuter ? 0.f : g0, b1 = kOuter ? 0.f : g1;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t = tok0 + nt * 8 + cq;
        const bool v0 = t < valid, v1 = t + 1 < valid;
        sc[nt][0] = v0 ? fmaf(sc[nt][0], scale_log2, b0) : -INFINITY;
        sc[nt][1] = v1 ? fmaf(sc[nt][1], scale_log2, b0) : -INFINITY;
        sc[nt][2] = v0 ? fmaf(sc[nt][2], scale_log2, b1) : -INFINITY;
        sc[nt][3] = v1 ? fmaf(sc[nt][3], scale_log2, b1) : -INFINITY;
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
    for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = exp2f(sc[nt][0] - u0);
        sc[nt][1] = exp2f(sc[nt][1] - u0);
        sc[nt][2] = exp2f(sc[nt][2] - u1);
        sc[nt][3] = exp2f(sc[nt][3] - u1);
        st.l0 += sc[nt][0] + sc[nt][1];
        st.l1 += sc[nt][2] + sc[nt][3];
    }
    if (kOuter) {  // the block's gate weights its values, not its share of the normaliser
        const float gm0 = exp2f(g0), gm1 = exp2f(g1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sc[nt][0] *= gm0;
            sc[nt][1] *= gm0;
            sc[nt][2] *= gm1;
            sc[nt][3] *= gm1;
        }
    }
    // ---- O += P V (P as bf16 hi + lo) ----
#pragma unroll
    for (int kt = 0; kt < NT / 2; ++kt) {
        uint32_t ph[4], pl[4];
        const float* p0 = sc[2 * kt];
        const float* p1 = sc[2 * kt + 1];
        const float pv[8] = {p0[0], p0[1], p0[2], p0[3], p1[0], p1[1], p1[2], p1[3]};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 hi = __floats2bfloat162_rn(pv[2 * e], pv[2 * e + 1]);
            const float2 hf = __bfloat1622float2(hi);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(pv[2 * e] - hf.x, pv[2 * e + 1] - hf.y);
            ph[e] = *reinterpret_cast<const uint32_t*>(&hi);
            pl[e] = *reinterpret_cast<const uint32_t*>(&lo);
        }
        const int row = tok0 + kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            const int chunk = 2 * np + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(swz(vb + (chunk >> 3) * TG::kHalf, row, chunk & 7), b0, b1, b2, b3);
            mma_bf16_16816(st.o[2 * np], ph, b0, b1);
            mma_bf16_16816(st.o[2 * np], pl, b0, b1);
            mma_bf16_16816(st.o[2 * np + 1], ph, b2, b3);
            mma_bf16_16816(st.o[2 * np + 1], pl, b2, b3);
        }
    }
}

// This warp's (max, sum, O) rows to shared memory: merge_o [warps][16][128],
// merge_ml [warps][16][2].  Rows >= rows_used (zero query rows) are not stored.
__device__ __forceinline__ void decode_state_store(DecodeState& st, float* merge_o, float* merge_ml, int warp,
                                                   int lane, int rows_used = 16) {
    const int r = lane >> 2, cq = (lane & 3) * 2;
    st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 1);
    st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 2);
    st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 1);
    st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 2);
    float* mo = merge_o + warp * 16 * kHeadDim;
    if (r < rows_used) {
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<float2*>(mo + r * kHeadDim + n * 8 + cq) = make_float2(st.o[n][0], st.o[n][1]);
    }
    if (r + 8 < rows_used) {
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<float2*>(mo + (r + 8) * kHeadDim + n * 8 + cq) = make_float2(st.o[n][2], st.o[n][3]);
    }
    if ((lane & 3) == 0) {
        merge_ml[(warp * 16 + r) * 2] = st.m0;
        merge_ml[(warp * 16 + r) * 2 + 1] = st.l0;
        merge_ml[(warp * 16 + r + 8) * 2] = st.m1;
        merge_ml[(warp * 16 + r + 8) * 2 + 1] = st.l1;
    }
}

// Merge `nwarps` consumer warps' states for (row, channel): normalised O and the
// natural-log LSE of the row (-inf and O = 0 when the row saw no token).
__device__ __forceinline__ void merge_warps(const float* merge_o, const float* merge_ml, int row, int ch, float& o,
                                            float& lse, int nwarps = kDecodeConsumerWarps) {
    float M = -INFINITY;
    for (int w = 0; w < nwarps; ++w) M = fmaxf(M, merge_ml[(w * 16 + row) * 2]);
    float osum = 0.f, lsum = 0.f;
    if (M > -INFINITY) {
        for (int w = 0; w < nwarps; ++w) {
            const float mw = merge_ml[(w * 16 + row) * 2];
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            lsum += f * merge_ml[(w * 16 + row) * 2 + 1];
            osum += f * merge_o[(w * 16 + row) * kHeadDim + ch];
        }
    }
    o = lsum > 0.f ? osum / lsum : 0.f;
    lse = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
}


// ---------------------------------------------------------------------------
// Transposed tiles for at most 8*NH query heads (the fused step): the 16 tokens of a
// warp are the MMA rows and the heads the columns -- S^T = K Q^T and O^T += V^T P^T --
// so a group of G <= 8 heads fills one n8 tile instead of padding 16 rows, which halves
// the tensor-core work and the O registers.  Blocks are staged 64 tokens at a time
// (TileGeom<64>); P^T reaches the B-operand layout through movmatrix.
// ---------------------------------------------------------------------------
template <int NH>
struct DecodeStateT {
    float o[NH][8][4];  // O^T tile mt: c0,c1 = (channel 16mt + lane/4, heads 8nh + 2(lane%4) + 0/1); c2,c3 = channel + 8
    float m[NH][2];     // running max (log2 units) of heads 8nh + 2(lane%4) + x
    float l[NH][2];     // this lane's partial sums of those heads
};

template <int NH>
__device__ __forceinline__ void decode_state_init_t(DecodeStateT<NH>& st) {
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) st.o[nh][mt][0] = st.o[nh][mt][1] = st.o[nh][mt][2] = st.o[nh][mt][3] = 0.f;
        st.m[nh][0] = st.m[nh][1] = -INFINITY;
        st.l[nh][0] = st.l[nh][1] = 0.f;
    }
}

// Q of the group as B fragments of S^T = K Q^T: column = head 8nh + lane/4 (zero past G),
// rows = channel pairs 16ks + 2(lane%4) (+8).
template <int NH>
__device__ __forceinline__ void load_q_frags_t(uint32_t (&qb)[NH][8][2], const __nv_bfloat16* qg, int G, int lane) {
    const int c2 = (lane & 3) * 2;
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
        const int head = nh * 8 + (lane >> 2);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const __nv_bfloat16* p = qg + head * kHeadDim + ks * 16 + c2;
            qb[nh][ks][0] = head < G ? *reinterpret_cast<const uint32_t*>(p) : 0u;
            qb[nh][ks][1] = head < G ? *reinterpret_cast<const uint32_t*>(p + 8) : 0u;
        }
    }
}

// One 64-token stage: the 16 tokens of token slot `slot` (0..3).  gb[nh][x] is the log-gate
// (log2 units) of head 8nh + 2(lane%4) + x, added to the logits; with `outer` ("SAS ...",
// Method: the gate outside the softmax) it stays out of the logits and 2^gb instead weights
// the values.  `valid` counts the stage's valid tokens.
template <int NH>
__device__ __forceinline__ void decode_block_t(DecodeStateT<NH>& st, const uint32_t (&qb)[NH][8][2], uint8_t* stage,
                                               int valid, const float (&gb)[NH][2], float scale_log2, int slot,
                                               int lane, bool outer = false) {
    using TG = TileGeom<64>;
    const int tok0 = slot * 16;
    if (tok0 >= valid) return;
    const uint32_t kb = smem_u32(stage);
    const uint32_t vb = kb + 2 * TG::kHalf;
    if (valid < tok0 + 16) {
        // rows past len may hold anything: zero this warp's invalid V rows so 0*garbage cannot appear
        uint8_t* vrow = stage + 2 * TG::kHalf;
        for (int e = lane; e < (tok0 + 16 - valid) * 16; e += 32) {
            const int row = valid + e / 16, ch = e % 16;
            *reinterpret_cast<uint4*>(vrow + (ch >> 3) * TG::kHalf + row * 128 + ((ch & 7) << 4)) =
                make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
    }
    // ---- S^T = K Q^T (16 tokens x 8 heads per n-tile): two independent accumulator chains
    // (even and odd channel steps), summed once ----
    float s[NH][4], s2[NH][4];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) s[nh][0] = s[nh][1] = s[nh][2] = s[nh][3] = s2[nh][0] = s2[nh][1] = s2[nh][2] = s2[nh][3] = 0.f;
    {
        const int row = tok0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        uint32_t a[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int chunk = 2 * ks + (lane >> 4);
            ldmatrix_x4(swz(kb + (chunk >> 3) * TG::kHalf, row, chunk & 7), a[ks][0], a[ks][1], a[ks][2], a[ks][3]);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) mma_bf16_16816((ks & 1) ? s2[nh] : s[nh], a[ks], qb[nh][ks][0], qb[nh][ks][1]);
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
            for (int x = 0; x < 4; ++x) s[nh][x] += s2[nh][x];
    }
    // ---- scale, log-gate, mask; online softmax over the tokens of each head (base 2) ----
    const int tr = lane >> 2;  // this lane's tokens: tr and tr + 8
    const bool v0 = tok0 + tr < valid, v1 = tok0 + tr + 8 < valid;
    bool rescale = false;
    float alpha[NH][2], u[NH][2];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const float bias = outer ? 0.f : gb[nh][x];
            s[nh][x] = v0 ? fmaf(s[nh][x], scale_log2, bias) : -INFINITY;
            s[nh][2 + x] = v1 ? fmaf(s[nh][2 + x], scale_log2, bias) : -INFINITY;
            float mx = fmaxf(s[nh][x], s[nh][2 + x]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float n = fmaxf(st.m[nh][x], mx);
            u[nh][x] = n == -INFINITY ? 0.f : n;
            alpha[nh][x] = exp2f(st.m[nh][x] - u[nh][x]);
            rescale |= alpha[nh][x] != 1.f;
            st.m[nh][x] = n;
            st.l[nh][x] *= alpha[nh][x];
        }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                st.o[nh][mt][0] *= alpha[nh][0];
                st.o[nh][mt][1] *= alpha[nh][1];
                st.o[nh][mt][2] *= alpha[nh][0];
                st.o[nh][mt][3] *= alpha[nh][1];
            }
    }
    // ---- P^T as B fragments (bf16 hi + lo): the two 8x8 halves of the S^T tile transposed ----
    uint32_t bh[NH][2], bl[NH][2];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = exp2f(s[nh][e] - u[nh][e & 1]);
        st.l[nh][0] += p[0] + p[2];
        st.l[nh][1] += p[1] + p[3];
        if (outer) {  // the block's gate weights its values, not its share of the normaliser
            const float gm0 = exp2f(gb[nh][0]), gm1 = exp2f(gb[nh][1]);
            p[0] *= gm0;
            p[2] *= gm0;
            p[1] *= gm1;
            p[3] *= gm1;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // tokens tr (hh = 0) and tr + 8 (hh = 1)
            const __nv_bfloat162 hi = __floats2bfloat162_rn(p[2 * hh], p[2 * hh + 1]);
            const float2 hf = __bfloat1622float2(hi);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(p[2 * hh] - hf.x, p[2 * hh + 1] - hf.y);
            bh[nh][hh] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&hi));
            bl[nh][hh] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&lo));
        }
    }
    // ---- O^T += V^T P^T: eight 16-channel row tiles ----
    {
        const int q = lane >> 3;
        const int row = tok0 + (q >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int chunk = 2 * mt + (q & 1);
            uint32_t a[4];
            ldmatrix_x4_trans(swz(vb + (chunk >> 3) * TG::kHalf, row, chunk & 7), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
                mma_bf16_16816(st.o[nh][mt], a, bh[nh][0], bh[nh][1]);
                mma_bf16_16816(st.o[nh][mt], a, bl[nh][0], bl[nh][1]);
            }
        }
    }
}

// Row stride (floats) of merge_o for the transposed tiles: 4 words of padding put the eight
// lanes of one head (consecutive channels) and the lanes of the next heads in distinct banks.
constexpr int kMergeStride = kHeadDim + 4;

// This warp's (max, sum, O) of heads < G to shared memory: merge_o [warps][16][kMergeStride]
// (head rows, channels), merge_ml [warps][16][2].
template <int NH>
__device__ __forceinline__ void decode_state_store_t(DecodeStateT<NH>& st, float* merge_o, float* merge_ml, int warp,
                                                     int lane, int G) {
    const int t = lane & 3, tr = lane >> 2;
    float* mo = merge_o + warp * 16 * kMergeStride;
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            float l = st.l[nh][x];  // over the warp's tokens: lanes of equal lane%4 hold the same heads
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            const int hd = nh * 8 + 2 * t + x;
            if (hd < G) {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    mo[hd * kMergeStride + mt * 16 + tr] = st.o[nh][mt][x];
                    mo[hd * kMergeStride + mt * 16 + tr + 8] = st.o[nh][mt][2 + x];
                }
                if (tr == 0) {
                    merge_ml[(warp * 16 + hd) * 2] = st.m[nh][x];
                    merge_ml[(warp * 16 + hd) * 2 + 1] = l;
                }
            }
        }
}

}  // namespace sba
