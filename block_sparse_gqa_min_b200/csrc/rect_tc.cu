// The rectification pass on the fifth-generation tensor cores (tcgen05, TMEM).
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation", Summary:
// every f generated tokens are re-encoded in one parallel dense pass -- their
// keys and values rewritten, the block keys of the touched blocks refreshed --
// and each of the f tokens attends causally to the whole cache (Key points:
// f in {16, 32, 64, 128}).  With the M*G query rows of a group sharing every
// key and value tile, this is a dense contraction: 128 query rows against each
// 128-token tile, the shape the tensor cores take whole.
//
// The same pipeline serves several query tokens sharing one selection
// (sba_sparse_decode_multi at M*G >= 64 query rows, ReSA Key points: the
// self-speculative comparison checks several draft tokens with one sparse
// pass): the block list is then the group's selection, two 64-token blocks or
// one 128-token block per stage, and nothing is written to the cache.
//
// One CTA per (split, KV head x row group of 128 query rows, sequence): eight
// softmax warps, a producer warp and an MMA warp.
//  - the producer warp streams the CTA's share of the sequence in 128-token
//    stages (K0 K1 V0 V1 halves of 128 rows x 128 B, each filled by two 2-D
//    TMA loads of 64 rows, 128-byte swizzle, no multicast) into a ring of
//    three 64 KB stages (shared memory holds nothing else).  Before a block
//    the window touches is loaded, it writes the window's K/V rows of that
//    block into the cache (a proxy fence orders them ahead of the tile load);
//    rows past the share or past len are zeroed in the stage before anyone
//    reads it; after its last stage it recomputes the Quest min/max of the
//    touched blocks from their keys in global memory.
//  - the MMA warp allocates all 512 TMEM columns and, one thread issuing, runs
//    S = Q K^T for each stage (M 128 rows, N 128 tokens, K 128 channels:
//    eight tcgen05.mma kind::f16, bf16 in, fp32 accumulate; A = Q from TMEM,
//    B = the K tile) into one of two S/P buffers (TMEM columns 0-127,
//    128-255), so the next stage's S is computed while the softmax works on
//    this one; then, once P has replaced S in the buffer, O += P_hi V + P_lo V
//    (M 128, N 128 channels, K 128 tokens; A = P from TMEM, V read MN-major
//    straight from the TMA tile) into TMEM columns 256-383.  The S of stage
//    q + 2 overwrites the P that O += P V of stage q reads; the tensor core
//    runs one thread's MMAs in issue order, so no wait separates them.
//    tcgen05.commit signals S, O and the stage's release on mbarriers.  A 16-bit A operand in TMEM is row r = lane r with two
//    consecutive K elements per 32-bit column (the lower one in the low half):
//    Q takes columns 384-447 (128 channels); P the 128 columns of its buffer
//    (64 for the hi parts of the 128 tokens, then 64 for the lo).
//  - the softmax warps: query row r = TMEM lane r is shared by the warps w with
//    w % 4 = r / 32, each owning an equal share of the stage's 128 columns.  A
//    thread reads its columns of S (tcgen05.ld 32x32b), applies the causal
//    limit (t <= len - f + i for token i), agrees on the row maximum with the
//    row's other warps through shared memory, keeps an online softmax in base 2
//    (the scale folded into the exponent's FMA) whose offset moves only when
//    the row maximum grows by more than 2^8 (then O's row is rescaled in TMEM;
//    otherwise exponentials stay below 2^8), and writes its tokens of P as bf16
//    hi + lo parts (hi + lo within 2^-15 |p| of p) over S in the same buffer
//    (tcgen05.st).  At the end it reads its columns of O, normalises them and
//    writes the split's O and LSE ([B][f][H_q][S][d], [B][f][H_q][S]).
// Every wait is bounded: a wait that runs out reports SBA_DEV_TIMEOUT and the
// roles stop, and TMEM is released on every path.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "decode_tile.cuh"
#include "launch.cuh"

namespace sba {

bool make_kv_tmap(CUtensorMap* m, void* base, uint64_t rows, int blk);  // decode.cu

#ifndef SBA_RECT_SOFTMAX_WARPS
#define SBA_RECT_SOFTMAX_WARPS 8
#endif

namespace {

constexpr int kRtRows = 128;               // query rows per CTA: the MMA's M
constexpr int kStageTok = 128;             // tokens per ring stage: the N of S = Q K^T
constexpr int kRtStages = 3;               // 64 KB K/V stages: 192 KB, all the shared memory there is
constexpr int kRtStage = 65536;
constexpr int kRtHalf = 16384;             // 128 rows x 128 B (64 channels of K or V)
constexpr int kSmWarps = SBA_RECT_SOFTMAX_WARPS;  // softmax warps: kCq per TMEM lane quarter
constexpr int kCq = kSmWarps / 4;          // warps sharing a query row (column groups)
constexpr int kCols = kStageTok / kCq;     // S columns (tokens) of a stage per thread
constexpr int kOCols = 128 / kCq;          // O (and Q) channels per thread
constexpr int kRtThreads = (kSmWarps + 2) * 32;  // softmax warps, then the producer, then the MMA warp
constexpr int kProdWarp = kSmWarps, kMmaWarp = kSmWarps + 1;
static_assert(kSmWarps == 8 || kSmWarps == 16, "two or four warps per TMEM lane quarter");
static_assert(kCols % 32 == 0, "P is written 32 tokens at a time");
constexpr int kRtSmem = kRtStages * kRtStage + 1024;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S/P buffers 0-127 and 128-255 (S in fp32; then P as bf16 pairs: hi parts in the
// first 64, lo parts in the next 64); O 256-383 (fp32); Q 384-447 (bf16 pairs)
constexpr uint32_t kColS = 0, kColO = 256, kColQ = 384;

struct RtArgs {
    sba_cache c;
    const __nv_bfloat16* q;  // [B][f][H_q][d]
    int M;                   // f (the query tokens)
    const uint4* k_new;      // dense: [B][f][H_kv][d], keys and values of positions len-f .. len-1
    const uint4* v_new;
    const int32_t* sel_idx;  // sparse: [B][H_kv][n_max], the group's selected blocks
    const int32_t* sel_cnt;  // sparse: [B][H_kv]
    int n_max;
    float scale_log2;
    int num_splits;
    float* o_part;           // [B][f][H_q][S][d]
    float* lse_part;         // [B][f][H_q][S]
};

// ---- tcgen05 wrappers ----
// Shared-memory matrix descriptor: start address, leading / stride byte offsets (16-byte
// units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
// D (+)= A B with A read from TMEM (K-major: row = lane, two 16-bit K elements per column) and B
// from shared memory
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// consecutive TMEM columns of this thread's lane (warp w accesses lanes 32 (w % 4) ..)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 2^x by the special-function unit (flushes results below 2^-126 to zero, which no softmax
// weight here can reach with any effect)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// 8 / 16 / 32 consecutive 32-bit TMEM columns of this thread's lane, from registers; the caller
// waits (tcgen05.wait::st) before signalling
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// N consecutive fp32 columns (N = 16, 32 or 64) into / from registers
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float* v) {
    if constexpr (N == 16) {
        tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
    } else {
        static_assert(N % 32 == 0, "");
#pragma unroll
        for (int i = 0; i < N / 32; ++i) tmem_ld32(taddr + 32 * i, *reinterpret_cast<float(*)[32]>(v + 32 * i));
    }
}
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* v) {
    if constexpr (N == 8) {
        tmem_st8(taddr, *reinterpret_cast<const uint32_t(*)[8]>(v));
    } else if constexpr (N == 16) {
        tmem_st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(v));
    } else {
        static_assert(N % 32 == 0, "");
#pragma unroll
        for (int i = 0; i < N / 32; ++i) tmem_st32(taddr + 32 * i, *reinterpret_cast<const uint32_t(*)[32]>(v + 32 * i));
    }
}

__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int kBlk, bool kSparse>
__global__ void __launch_bounds__(kRtThreads, 1)
    rect_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ RtArgs a) {
    extern __shared__ uint8_t dyn_raw[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t kv_full[kRtStages], kv_empty[kRtStages], zbar, q_full, s_full[2], p_full[2], pv_done[2], fin;
    __shared__ uint32_t tmem_base;
    __shared__ float xmax[2][kCq][kRtRows];  // [stage parity][column group][row]: partial row maxima
    __shared__ float xl[kCq][kRtRows];       // [column group][row]: partial row sums at the end

    const sba_cache& c = a.c;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = blockIdx.x, h = blockIdx.y % c.H_kv, rg = blockIdx.y / c.H_kv, s = blockIdx.z;
    const int G = c.H_q / c.H_kv;
    const int R = a.M * G;
    const int row0 = rg * kRtRows;

    if (tid == 0) {
        for (int i = 0; i < kRtStages; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(&zbar, 1);
        mbar_init(&q_full, kSmWarps);  // one arrival per softmax warp
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], kSmWarps);
            mbar_init(&pv_done[b], 1);
        }
        mbar_init(&fin, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
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
    const bool appends = !kSparse && a.M > 0 && pos0 >= 0;
    if (!kSparse && !appends && tid == 0 && sp == 0 && blockIdx.y == 0) report(c.status, SBA_DEV_BAD_POSITION);
    const int tb0 = appends ? pos0 / kBlk : N;
    // dense: the blocks [0, N); sparse: the group's selection, in C-order of the list
    const int32_t* sel = kSparse ? a.sel_idx + ((int64_t)s * c.H_kv + h) * a.n_max : nullptr;
    int cnt = N;
    if (kSparse) {
        cnt = __ldg(a.sel_cnt + s * c.H_kv + h);
        if (cnt < 0 || cnt > a.n_max) {
            if (tid == 0 && sp == 0 && rg == 0) report(c.status, SBA_DEV_BAD_SELECTION);
            cnt = cnt < 0 ? 0 : a.n_max;
        }
    }
    const int i0 = (int)((int64_t)cnt * sp / a.num_splits), i1 = (int)((int64_t)cnt * (sp + 1) / a.num_splits);
    // dense: the share's tokens [t_begin, t_end) in 128-token stages (every stage holds at least
    // one); sparse: the share's blocks, two (b = 64) or one (b = 128) per stage
    const int t_begin = i0 * kBlk, t_end = min(len, i1 * kBlk);
    const int nproc = kSparse ? (kBlk == 64 ? (i1 - i0 + 1) / 2 : i1 - i0)
                              : (t_end > t_begin ? (t_end - t_begin + kStageTok - 1) / kStageTok : 0);
    // 64-token half h2 of stage q: its block j, the position of its first token, and its valid
    // tokens (0: no such half, or a selected index outside [0, N))
    auto stage_half = [&](int q, int h2, int& j, int& base) -> int {
        if (kSparse) {
            const int idx = kBlk == 64 ? i0 + 2 * q + h2 : i0 + q;
            if (idx >= i1) return 0;
            j = __ldg(sel + idx);
            if (j < 0 || j >= N) return 0;
            base = j * kBlk + (kBlk == 64 ? 0 : 64 * h2);
            return max(0, min(64, len - base));
        } else {
            base = t_begin + kStageTok * q + 64 * h2;
            j = base / kBlk;
            return max(0, min(64, t_end - base));
        }
    };

    // this thread's share of its query row (row = TMEM lane 32 (warp % 4) + lane, channels
    // kOCols (warp / 4) ..): zero past the group's rows
    uint32_t qv[kOCols / 2];
    if (warp < kSmWarps) {
        const int r = 32 * (warp & 3) + lane, cq = warp >> 2, gr = row0 + r;
        const __nv_bfloat16* qrow =
            gr < R ? a.q + (((int64_t)s * a.M + gr / G) * c.H_q + h * G + gr % G) * kHeadDim : nullptr;
#pragma unroll
        for (int cc = 0; cc < kOCols / 8; ++cc) {
            const uint4 v = qrow ? __ldg(reinterpret_cast<const uint4*>(qrow) + (kOCols / 8) * cq + cc)
                                 : make_uint4(0u, 0u, 0u, 0u);
            qv[4 * cc] = v.x, qv[4 * cc + 1] = v.y, qv[4 * cc + 2] = v.z, qv[4 * cc + 3] = v.w;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    if (warp < kSmWarps) {  // Q into its TMEM columns, then the MMA warp may read it
        tmem_st_n<kOCols / 2>(tm + ((uint32_t)(32 * (warp & 3)) << 16) + kColQ + (kOCols / 2) * (warp >> 2), qv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full);
    }

    bool alive = true;
    if (warp == kProdWarp) {
        // ------------------------------ producer ------------------------------
        uint32_t zpar = 0;
        for (int q = 0; q < nproc && alive; ++q) {
            const int st = q % kRtStages;
            if (q >= kRtStages) {
                if (lane == 0) alive = mbar_wait_sleep(&kv_empty[st], ((q / kRtStages) - 1) & 1, c.status);
                alive = __shfl_sync(0xffffffffu, alive, 0);
                if (!alive) break;
            }
            uint8_t* base = dyn + (size_t)st * kRtStage;
            // the stage's two 64-row halves: valid tokens and page of each (-1: not loaded), the
            // window's rows of a block written before its first half is loaded (dense)
            int pgs[2], vh[2], ys[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                int j = 0, t = 0;
                vh[h2] = stage_half(q, h2, j, t);
                pgs[h2] = -1;
                ys[h2] = 0;
                if (kSparse && lane == 0 && vh[h2] == 0) {
                    const int idx = kBlk == 64 ? i0 + 2 * q + h2 : i0 + q;
                    if (idx < i1 && (j < 0 || j >= N)) report(c.status, SBA_DEV_BAD_SELECTION);
                }
                if (vh[h2] == 0) continue;
                pgs[h2] = (int)page_of(c, s, j, lane == 0 ? c.status : nullptr);
                ys[h2] = (max(pgs[h2], 0) * c.H_kv + h) * kBlk + t % kBlk;
                if (pgs[h2] >= 0 && appends && t % kBlk == 0 && j >= tb0) {
                    const int w0 = max(pos0, j * kBlk), w1 = min(len, (j + 1) * kBlk);
                    for (int e = lane; e < (w1 - w0) * 32; e += 32) {
                        const int tt = w0 + (e >> 5), half = (e >> 4) & 1, l = e & 15;
                        const int64_t src = (((int64_t)s * a.M + (tt - pos0)) * c.H_kv + h) * 16 + l;
                        const uint4 v = __ldg((half ? a.v_new : a.k_new) + src);
                        reinterpret_cast<uint4*>(half ? c.v : c.k)[(((int64_t)pgs[h2] * c.H_kv + h) * kBlk + tt % kBlk) * 16 + l] = v;
                    }
                }
            }
            fence_proxy_async_global();  // this lane's window rows ahead of the tile loads
            __syncwarp();
            const int nload = (pgs[0] >= 0) + (pgs[1] >= 0);
            // a stage with rows to zero (past the share or len, a missing half, or a bad table entry,
            // reported) lands on the side barrier first
            const bool zero = vh[0] < 64 || vh[1] < 64 || nload < 2;
            uint64_t* bar = zero ? &zbar : &kv_full[st];
            if (lane == 0 && nload > 0) {
                mbar_arrive_expect_tx(bar, nload * (kRtStage / 2));
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    if (pgs[h2] < 0) continue;
                    const int y = ys[h2];
                    uint8_t* dst = base + 64 * 128 * h2;
                    tma_load_2d(dst, &tmK, bar, 0, y);
                    tma_load_2d(dst + kRtHalf, &tmK, bar, 64, y);
                    tma_load_2d(dst + 2 * kRtHalf, &tmV, bar, 0, y);
                    tma_load_2d(dst + 3 * kRtHalf, &tmV, bar, 64, y);
                }
            }
            if (zero) {
                // rows that are not the share's valid tokens may hold anything (NaN included, or a
                // previous stage): zero them before the tensor cores read the stage
                bool ok = true;
                if (nload > 0) {
                    if (lane == 0) ok = mbar_wait_sleep(&zbar, zpar, c.status);
                    zpar ^= 1u;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                }
                for (int e = lane; e < kStageTok * 32 && ok; e += 32) {
                    const int rr = e >> 5, part = (e >> 4) & 1, ch = e & 15;  // row, K or V, 16-byte chunk
                    if ((rr & 63) < vh[rr >> 6] && pgs[rr >> 6] >= 0) continue;
                    *reinterpret_cast<uint4*>(base + (2 * part + (ch >> 3)) * kRtHalf + rr * 128 + ((ch & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&kv_full[st]);
                if (!ok) alive = false;
            }
        }
        // the Quest descriptors of the blocks the window touched that lie in this share, recomputed
        // from all of each block's valid keys in global memory (the window's rows were written above
        // by this warp; at most three blocks per head)
        if (!kSparse && appends && c.desc && rg == 0 && alive) {
            __syncwarp();
            for (int j = max(tb0, i0); j < min(N, i1); ++j) {
                const int pg = (int)page_of(c, s, j, nullptr);
                if (pg < 0) continue;
                const int vb = min(kBlk, len - j * kBlk);
                const uint4* krows = reinterpret_cast<const uint4*>(c.k) + ((int64_t)pg * c.H_kv + h) * kBlk * 16;
                uint32_t mn[4], mx[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) mn[e] = 0x7f807f80u, mx[e] = 0xff80ff80u;
                const int ck = lane & 15;  // 16-byte chunk (8 channels) of a row; lanes 16-31 take odd rows
                for (int t = lane >> 4; t < vb; t += 2) {
                    const uint4 w = krows[t * 16 + ck];
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        mn[e] = bmin2(mn[e], ws[e]);
                        mx[e] = bmax2(mx[e], ws[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    mn[e] = bmin2(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], 16));
                    mx[e] = bmax2(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
                }
                if (lane < 16) {
                    uint8_t* d = reinterpret_cast<uint8_t*>(c.desc) + ((int64_t)pg * c.H_kv + h) * 2 * kHeadDim * 2;
                    *reinterpret_cast<uint4*>(d + lane * 16) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
                    *reinterpret_cast<uint4*>(d + 2 * kHeadDim + lane * 16) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------ MMA issue ------------------------------
        constexpr uint32_t kIdQK = umma_idesc(128, kStageTok, false);
        constexpr uint32_t kIdPV = umma_idesc(128, 128, true);
        // descriptors of ring stage 0 (K tile: K-major; V tile: MN-major, its two 64-channel halves
        // 16 KB apart); a stage or a K step adds its byte offset / 16 to the start-address field,
        // which stays below 2^14 for every shared-memory address
        const uint32_t ring = smem_u32(dyn);
        const uint64_t dK0 = umma_desc(ring, 16, 1024), dV0 = umma_desc(ring + 2 * kRtHalf, kRtHalf, 1024);
        bool issued = false;  // any MMA issued by this warp
        if (lane == 0) alive = mbar_wait_sleep(&q_full, 0, c.status);  // Q in TMEM
        alive = __shfl_sync(0xffffffffu, alive, 0);
        // S(q) = Q K(q)^T into buffer q % 2; K = 128 channels in eight steps of 16 (32 bytes along
        // the swizzled rows).  The buffer still holds P of stage q - 2, read by O += P V of that
        // stage, which this thread issued earlier: the tensor core runs one thread's MMAs in issue
        // order, so that read comes first without a wait.
        auto issue_qk = [&](int q) {
            const int st = q % kRtStages;
            if (lane == 0) alive = mbar_wait_sleep(&kv_full[st], (q / kRtStages) & 1, c.status);
            alive = __shfl_sync(0xffffffffu, alive, 0);
            if (!alive) return;
            tc_fence_after();
            const uint64_t dK = dK0 + (uint64_t)((st * kRtStage) >> 4);
            const uint32_t tS = tm + kColS + 128 * (q & 1);
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ts(tS, tm + kColQ + 8 * kk, dK + (uint64_t)((((kk >> 2) * kRtHalf) + (kk & 3) * 32) >> 4),
                                kIdQK, kk > 0);
                umma_commit(&s_full[q & 1]);
            }
            issued = true;
            __syncwarp();
        };
        if (nproc > 0 && alive) issue_qk(0);
        for (int q = 0; q < nproc && alive; ++q) {
            // the next stage's S overlaps this stage's softmax
            if (q + 1 < nproc) {
                issue_qk(q + 1);
                if (!alive) break;
            }
            if (lane == 0) alive = mbar_wait_sleep(&p_full[q & 1], (q >> 1) & 1, c.status);
            alive = __shfl_sync(0xffffffffu, alive, 0);
            if (!alive) break;
            tc_fence_after();
            const int st = q % kRtStages;
            const uint64_t dV = dV0 + (uint64_t)((st * kRtStage) >> 4);
            const uint32_t tP = tm + kColS + 128 * (q & 1);
            if (lane == 0) {
                // O += P V: K = 128 tokens in eight steps of 16 (two 8-token groups of the V tile, 2 KB)
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ts(tm + kColO, tP + 64 * part + 8 * kk, dV + (uint64_t)((kk * 2048) >> 4), kIdPV,
                                    (q > 0 || part > 0 || kk > 0));
                umma_commit(&pv_done[q & 1]);
                umma_commit(&kv_empty[st]);
            }
            __syncwarp();
        }
        // every MMA this warp issued has completed before TMEM can be released (also after a
        // wait that ran out)
        if (lane == 0 && issued) {
            umma_commit(&fin);
            mbar_wait_sleep(&fin, 0, c.status);
        }
        __syncwarp();
    } else {
        // ------------------------------ softmax ------------------------------
        const int qd = warp & 3, cq = warp >> 2;  // lane quarter, column group
        const int r = 32 * qd + lane;              // query row = TMEM lane
        const int gr = row0 + r;
        const int lim = gr < R ? pos0 + gr / G + 1 : 0;  // causal limit (exclusive)
        const uint32_t lane_base = tm + ((uint32_t)(qd * 32) << 16);
        const float sl2 = a.scale_log2;
        // m_used: the exponent offset in scaled base-2 units (-inf until the row has a valid token)
        float m_used = -INFINITY, l = 0.f;
        // (a wait that runs out turns this warp dead; a dead warp still takes every named barrier of the
        // loop, so the row's other warps never wait on it forever, and arrives on nothing)
        const int hh = (kCols * cq) >> 6, hoff = (kCols * cq) & 63;  // this group's half and offset in it
        for (int q = 0; q < nproc; ++q) {
            int jh = 0, bh = 0;
            const int vhalf = stage_half(q, hh, jh, bh);
            const int base = bh + hoff;  // position of this group's first token
            bool ok = alive;
            if (ok) {
                if (lane == 0) ok = mbar_wait_sleep(&s_full[q & 1], (q >> 1) & 1, c.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            float sv[kCols];
            float mx = -INFINITY;
            if (ok) {
                tc_fence_after();
                tmem_ld_n<kCols>(lane_base + kColS + 128 * (q & 1) + kCols * cq, sv);
                const int nval = min(kCols, min(vhalf - hoff, lim - base));  // valid columns of this group
                if (nval < kCols) {
#pragma unroll
                    for (int t = 0; t < kCols; ++t) sv[t] = t < nval ? sv[t] : -INFINITY;
                }
                float m4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    m4[u] = sv[u];
#pragma unroll
                    for (int t = u + 4; t < kCols; t += 4) m4[u] = fmaxf(m4[u], sv[t]);
                }
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;  // the scale is positive
            }
            // the row maximum agreed with the row's other warps
            xmax[q & 1][cq][r] = mx;
            named_bar(1 + qd, 32 * kCq);
#pragma unroll
            for (int x = 0; x < kCq; ++x) mx = fmaxf(mx, xmax[q & 1][x][r]);
            if (!ok) {
                alive = false;
                continue;
            }
            // the exponent offset moves only when the maximum grows by more than 2^8
            float alpha = 1.f;
            if (mx > -INFINITY && (m_used == -INFINITY || mx > m_used + 8.f)) {
                alpha = m_used == -INFINITY ? 0.f : ex2(m_used - mx);
                m_used = mx;
                l *= alpha;
            }
            const bool rescale = q > 0 && alpha != 1.f;
            // (a row still without a valid token has every score at -inf: offset 0 gives 0 for each)
            const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
            // O (to rescale) once O += P V of stage q - 1 has completed
            if (__any_sync(0xffffffffu, rescale)) {
                if (lane == 0) ok = mbar_wait_sleep(&pv_done[(q - 1) & 1], ((q - 1) >> 1) & 1, c.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    alive = false;
                    continue;
                }
                tc_fence_after();
                const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c0 = 0; c0 < kOCols; c0 += 16) {  // 16 columns at a time (few registers)
                    float ov[16];
                    tmem_ld16(lane_base + kColO + kOCols * cq + c0, ov);
                    uint32_t ou[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(ov[e] * f);
                    tmem_st16(lane_base + kColO + kOCols * cq + c0, ou);
                }
            }
            // P = hi + lo in bf16 by integer operations (no conversion instructions): hi = p with its
            // low 16 bits cleared (truncation), r = p - hi (exact in fp32, 0 <= r < 2^-7 p) rounded to
            // bf16 for lo by adding half a bf16 unit before its low 16 bits are dropped; the pair's
            // upper halves are packed by one byte permute.  |p - hi - lo| <= 2^-8 r < 2^-15 p while r
            // is a normal float (p >= 2^-100); below that the error is under 2^-130, nothing next to
            // a row sum >= 1.  Every warp of the row has read its S before the barrier above, so P may
            // replace S anywhere in the buffer: this group's tokens go to kCols / 2 columns of hi pairs
            // from (kCols / 2) cq and as many of lo pairs 64 columns further, 32 tokens at a time.
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t tP = lane_base + kColS + 128 * (q & 1) + (kCols / 2) * cq;
#pragma unroll
            for (int c0 = 0; c0 < kCols; c0 += 32) {
                uint32_t ph[16], pl[16];
#pragma unroll
                for (int t = 0; t < 32; t += 2) {
                    const float p0 = ex2(fmaf(sv[c0 + t], sl2, neg_m));
                    const float p1 = ex2(fmaf(sv[c0 + t + 1], sl2, neg_m));
                    ls[(t >> 1) & 3] += p0 + p1;
                    const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
                    const float r0 = p0 - __uint_as_float(u0 & 0xffff0000u);
                    const float r1 = p1 - __uint_as_float(u1 & 0xffff0000u);
                    ph[t / 2] = __byte_perm(u0, u1, 0x7632);
                    pl[t / 2] = __byte_perm(__float_as_uint(r0) + 0x8000u, __float_as_uint(r1) + 0x8000u, 0x7632);
                }
                tmem_st16(tP + c0 / 2, ph);
                tmem_st16(tP + 64 + c0 / 2, pl);
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[q & 1]);
        }
        // the split's normalised output of this row: this warp's kOCols channels
        xl[cq][r] = l;
        named_bar(1 + qd, 32 * kCq);
        float lt = 0.f;
#pragma unroll
        for (int x = 0; x < kCq; ++x) lt += xl[x][r];
        bool have = false;
        if (alive && nproc > 0) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait_sleep(&pv_done[(nproc - 1) & 1], ((nproc - 1) >> 1) & 1, c.status);
            have = __shfl_sync(0xffffffffu, ok, 0);
            if (have) tc_fence_after();
        }
        const int ti = gr / G, g = gr % G;
        const int64_t orow = (((int64_t)s * a.M + ti) * c.H_q + h * G + g) * a.num_splits + sp;
        const bool any = have && lt > 0.f;
        const float inv = any ? 1.f / lt : 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < kOCols; c0 += 32) {  // (the loads are warp-collective: every lane takes them)
            float ov[32];
            if (have) tmem_ld32(lane_base + kColO + kOCols * cq + c0, ov);
            if (gr < R) {
                float* dst = a.o_part + orow * kHeadDim + kOCols * cq + c0;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + e) =
                        any ? make_float4(ov[e] * inv, ov[e + 1] * inv, ov[e + 2] * inv, ov[e + 3] * inv)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        if (gr < R && cq == 0) a.lse_part[orow] = any ? (m_used + log2f(lt)) * kLn2 : -INFINITY;
    }
    // every role is done with TMEM: the allocating warp releases it
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(kTmemCols));
    }
}

template <int kBlk, bool kSparse>
int launch_rect_t(const sba_cache& c, const RtArgs& a, int row_groups, cudaStream_t stream) {
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)c.num_pages * c.H_kv * kBlk;
    if (!make_kv_tmap(&tk, c.k, rows, 64) || !make_kv_tmap(&tv, c.v, rows, 64)) return SBA_ERR_CUDA;
    if (allow_smem<rect_tc_kernel<kBlk, kSparse>>(kRtSmem) != SBA_OK) return SBA_ERR_CUDA;
    dim3 grid(a.num_splits, c.H_kv * row_groups, c.B);
    return launch(rect_tc_kernel<kBlk, kSparse>, grid, dim3(kRtThreads), kRtSmem, stream, tk, tv, a);
}

}  // namespace

int launch_rectify_tc(const sba_cache& c, const void* q, int f, const void* k_new, const void* v_new, float scale,
                      int num_splits, float* o_part, float* lse_part, cudaStream_t stream) {
    RtArgs a{};
    a.c = c;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.M = f;
    a.k_new = reinterpret_cast<const uint4*>(k_new);
    a.v_new = reinterpret_cast<const uint4*>(v_new);
    a.scale_log2 = scale * kLog2e;
    a.num_splits = num_splits;
    a.o_part = o_part;
    a.lse_part = lse_part;
    const int row_groups = (f * (c.H_q / c.H_kv) + kRtRows - 1) / kRtRows;
    return c.b == 64 ? launch_rect_t<64, false>(c, a, row_groups, stream)
                     : launch_rect_t<128, false>(c, a, row_groups, stream);
}

int launch_multi_query_tc(const sba_cache& c, const void* q, int M, const int32_t* sel_idx, const int32_t* sel_cnt,
                          int n_max, float scale, int num_splits, float* o_part, float* lse_part,
                          cudaStream_t stream) {
    RtArgs a{};
    a.c = c;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.M = M;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.n_max = n_max;
    a.scale_log2 = scale * kLog2e;
    a.num_splits = num_splits;
    a.o_part = o_part;
    a.lse_part = lse_part;
    const int row_groups = (M * (c.H_q / c.H_kv) + kRtRows - 1) / kRtRows;
    return c.b == 64 ? launch_rect_t<64, true>(c, a, row_groups, stream)
                     : launch_rect_t<128, true>(c, a, row_groups, stream);
}

}  // namespace sba
