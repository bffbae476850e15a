// The rectification pass on the fifth-generation tensor cores (tcgen05, TMEM).
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation", Summary:
// every f generated tokens are re-encoded in one parallel dense pass -- their
// keys and values rewritten, the block keys of the touched blocks refreshed --
// and each of the f tokens attends causally to the whole cache (Key points:
// f in {16, 32, 64, 128}).  With the M*G query rows of a group sharing every
// key and value tile, this is a dense contraction: 128 query rows against each
// 64-token tile, the shape the tensor cores take whole.
//
// One CTA per (split, KV head x row group of 128 query rows, sequence); 192
// threads:
//  - warp 4 (producer) streams each block in 64-token stages (K0 K1 V0 V1: four
//    2-D TMA loads of 64 rows x 128 B, 128-byte swizzle, no multicast) into a
//    ring of 32 KB stages.  Before a block the window touches is loaded, it
//    writes the window's K/V rows of that block into the cache (a proxy fence
//    orders them ahead of the tile load); after its last fill it recomputes the
//    Quest min/max of those blocks from the staged K rows.  Rows past len are
//    zeroed in the stage before anyone reads it.
//  - warp 5 (MMA) allocates 256 TMEM columns and, one thread issuing, runs per
//    stage S = Q K^T (M 128 rows, N 64 tokens, K 128 channels: eight
//    tcgen05.mma kind::f16, bf16 in, fp32 accumulate into TMEM columns 0-63),
//    then, once the softmax warps have written P, O += P_hi V + P_lo V (M 128,
//    N 128 channels, K 64 tokens; V read MN-major straight from the TMA tile)
//    into TMEM columns 128-255.  tcgen05.commit signals S, O and the stage's
//    release on mbarriers.
//  - warps 0-3 (softmax): thread r owns query row r = TMEM lane r.  It reads its
//    row of S (tcgen05.ld 32x32b.x64), applies the causal limit (t <= len - f + i
//    for token i) and the scale, keeps an online softmax whose exponent offset
//    moves only when the row maximum grows by more than 2^8 (then O's row is
//    rescaled in TMEM; otherwise exponentials stay below 2^8), and writes P as
//    bf16 hi + lo parts (about 16 mantissa bits) into the 128-byte-swizzled A
//    tile of the next MMA.  At the end it reads its O row, normalises it and
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

namespace {

constexpr int kRtRows = 128;               // query rows per CTA: the MMA's M
constexpr int kRtStages = 4;               // 64-token K/V stages
constexpr int kRtStage = 32768;
constexpr int kRtHalf = 8192;              // 64 rows x 128 B
constexpr int kRtThreads = 192;            // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kProdWarp = 4, kMmaWarp = 5;
constexpr int kOffQ = 0;                   // 2 x 16 KB: 128 rows x 64 channels, K-major, 128-B swizzle
constexpr int kOffP = 32768;               // P hi (16 KB) then P lo (16 KB): 128 rows x 64 tokens
constexpr int kOffRing = 65536;
constexpr int kRtSmem = kOffRing + kRtStages * kRtStage + 1024;
constexpr uint32_t kTmemCols = 256;        // S: columns 0-63; O: 128-255
constexpr uint32_t kColS = 0, kColO = 128;

struct RtArgs {
    sba_cache c;
    const __nv_bfloat16* q;  // [B][f][H_q][d]
    int M;                   // f
    const uint4* k_new;      // [B][f][H_kv][d]: keys and values of positions len-f .. len-1
    const uint4* v_new;
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
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 64 consecutive TMEM columns of this thread's lane (warp w reads lanes 32w..32w+31).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,"
        "%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float (&v)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,"
        "%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31])), "r"(__float_as_uint(v[32])),
        "r"(__float_as_uint(v[33])), "r"(__float_as_uint(v[34])), "r"(__float_as_uint(v[35])),
        "r"(__float_as_uint(v[36])), "r"(__float_as_uint(v[37])), "r"(__float_as_uint(v[38])),
        "r"(__float_as_uint(v[39])), "r"(__float_as_uint(v[40])), "r"(__float_as_uint(v[41])),
        "r"(__float_as_uint(v[42])), "r"(__float_as_uint(v[43])), "r"(__float_as_uint(v[44])),
        "r"(__float_as_uint(v[45])), "r"(__float_as_uint(v[46])), "r"(__float_as_uint(v[47])),
        "r"(__float_as_uint(v[48])), "r"(__float_as_uint(v[49])), "r"(__float_as_uint(v[50])),
        "r"(__float_as_uint(v[51])), "r"(__float_as_uint(v[52])), "r"(__float_as_uint(v[53])),
        "r"(__float_as_uint(v[54])), "r"(__float_as_uint(v[55])), "r"(__float_as_uint(v[56])),
        "r"(__float_as_uint(v[57])), "r"(__float_as_uint(v[58])), "r"(__float_as_uint(v[59])),
        "r"(__float_as_uint(v[60])), "r"(__float_as_uint(v[61])), "r"(__float_as_uint(v[62])),
        "r"(__float_as_uint(v[63]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

template <int kBlk>
__global__ void __launch_bounds__(kRtThreads, 1)
    rect_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ RtArgs a) {
    constexpr int kSub = kBlk / 64;
    extern __shared__ uint8_t dyn_raw[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t kv_full[kRtStages], kv_empty[kRtStages], zbar, s_full, p_full, pv_done, fin;
    __shared__ uint32_t tmem_base;

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
        mbar_init(&s_full, 1);
        mbar_init(&p_full, 4);
        mbar_init(&pv_done, 1);
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
    const int pos0 = len - a.M;  // first window token's position
    const bool appends = a.M > 0 && pos0 >= 0;
    if (!appends && tid == 0 && sp == 0 && blockIdx.y == 0) report(c.status, SBA_DEV_BAD_POSITION);
    const int tb0 = appends ? pos0 / kBlk : N;
    const int i0 = (int)((int64_t)N * sp / a.num_splits), i1 = (int)((int64_t)N * (sp + 1) / a.num_splits);
    const int nfill = (i1 - i0) * kSub;
    auto fill_valid = [&](int f) {  // tokens of fill f below len (0: the fill is skipped by every role)
        const int j = i0 + f / kSub, sb = f % kSub;
        return min(64, max(0, len - j * kBlk - 64 * sb));
    };

    // the query rows of this CTA into the K-major, 128-byte-swizzled A tile (zero past the group's rows)
    if (warp < 4) {
        const int r = tid, gr = row0 + r;
        const __nv_bfloat16* qrow =
            gr < R ? a.q + (((int64_t)s * a.M + gr / G) * c.H_q + h * G + gr % G) * kHeadDim : nullptr;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
            const uint4 v = qrow ? __ldg(reinterpret_cast<const uint4*>(qrow) + ch) : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(dyn + kOffQ + (ch >> 3) * 16384 + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;

    bool alive = true;
    if (warp == kProdWarp) {
        // ------------------------------ producer ------------------------------
        uint32_t zpar = 0;
        int q = 0;  // processed fills (ring slots)
        for (int f = 0; f < nfill && alive; ++f) {
            const int vf = fill_valid(f);
            if (vf == 0) continue;
            const int i = i0 + f / kSub, sb = f % kSub, j = i;
            const int st = q % kRtStages;
            if (q >= kRtStages) {
                if (lane == 0) alive = mbar_wait(&kv_empty[st], ((q / kRtStages) - 1) & 1, c.status);
                alive = __shfl_sync(0xffffffffu, alive, 0);
                if (!alive) break;
            }
            const int pg = (int)page_of(c, s, j, lane == 0 ? c.status : nullptr);
            uint8_t* base = dyn + kOffRing + (size_t)st * kRtStage;
            if (pg < 0) {
                // a bad table entry (reported): the stage is zeros, the roles stay in step
                for (int e = lane; e < kRtStage / 16; e += 32) reinterpret_cast<uint4*>(base)[e] = make_uint4(0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&kv_full[st]);
                ++q;
                continue;
            }
            if (appends && sb == 0 && j >= tb0) {
                // the window's rows of this block, each lane's stores ordered ahead of the tile load
                const int t0 = max(pos0, j * kBlk), t1 = min(len, (j + 1) * kBlk);
                for (int e = lane; e < (t1 - t0) * 32; e += 32) {
                    const int t = t0 + (e >> 5), half = (e >> 4) & 1, l = e & 15;
                    const int64_t src = (((int64_t)s * a.M + (t - pos0)) * c.H_kv + h) * 16 + l;
                    const uint4 v = __ldg((half ? a.v_new : a.k_new) + src);
                    reinterpret_cast<uint4*>(half ? c.v : c.k)[(((int64_t)pg * c.H_kv + h) * kBlk + t % kBlk) * 16 + l] = v;
                }
                fence_proxy_async_global();
                __syncwarp();
            }
            uint64_t* bar = vf == 64 ? &kv_full[st] : &zbar;
            if (lane == 0) {
                const int y = (pg * c.H_kv + h) * kBlk + 64 * sb;
                mbar_arrive_expect_tx(bar, kRtStage);
                tma_load_2d(base, &tmK, bar, 0, y);
                tma_load_2d(base + kRtHalf, &tmK, bar, 64, y);
                tma_load_2d(base + 2 * kRtHalf, &tmV, bar, 0, y);
                tma_load_2d(base + 3 * kRtHalf, &tmV, bar, 64, y);
            }
            if (vf < 64) {
                // rows past len may hold anything: zero them before the tensor cores read the stage
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&zbar, zpar, c.status);
                zpar ^= 1u;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                for (int e = lane; e < (64 - vf) * 32 && ok; e += 32) {
                    const int rr = vf + (e >> 5), part = (e >> 4) & 1, ch = e & 15;
                    *reinterpret_cast<uint4*>(base + (2 * part + (ch >> 3)) * kRtHalf + rr * 128 + ((ch & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&kv_full[st]);
                if (!ok) alive = false;
            }
            ++q;
        }
        // the Quest descriptors of the blocks the window touched, from their staged K rows (the
        // last fills of this share, still in the ring: nothing is loaded after them)
        const int nproc = q;
        if (appends && c.desc && rg == 0 && alive) {
            for (int pq = max(0, nproc - kRtStages); pq < nproc; ++pq) {
                // processed fill pq is fill pq (only the very last fill of a share can be skipped)
                const int i = i0 + pq / kSub, sb = pq % kSub, j = i;
                if (sb != 0 || j < tb0) continue;
                const int vb = min(kBlk, len - j * kBlk);
                uint32_t mn[4], mx[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) mn[e] = 0x7f807f80u, mx[e] = 0xff80ff80u;
                bool ok = true;
                for (int sub = 0; sub < kSub && ok; ++sub) {
                    const int ff = pq + sub, vs = min(64, vb - 64 * sub);
                    if (vs <= 0 || ff >= nproc) break;
                    if (lane == 0) ok = mbar_wait(&kv_full[ff % kRtStages], (ff / kRtStages) & 1, c.status);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const uint8_t* kt = dyn + kOffRing + (size_t)(ff % kRtStages) * kRtStage;
                    const int ck = lane & 15, cc = ck & 7;
                    for (int t = lane >> 4; t < vs; t += 2) {
                        const uint4 w = *reinterpret_cast<const uint4*>(kt + (ck >> 3) * kRtHalf + t * 128 + ((cc ^ (t & 7)) << 4));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            mn[e] = bmin2(mn[e], ws[e]);
                            mx[e] = bmax2(mx[e], ws[e]);
                        }
                    }
                }
                if (!ok) break;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    mn[e] = bmin2(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], 16));
                    mx[e] = bmax2(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
                }
                const int pg = (int)page_of(c, s, j, nullptr);
                if (lane < 16 && pg >= 0) {
                    uint8_t* d = reinterpret_cast<uint8_t*>(c.desc) + ((int64_t)pg * c.H_kv + h) * 2 * kHeadDim * 2;
                    *reinterpret_cast<uint4*>(d + lane * 16) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
                    *reinterpret_cast<uint4*>(d + 2 * kHeadDim + lane * 16) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------ MMA issue ------------------------------
        constexpr uint32_t kIdQK = umma_idesc(128, 64, false);
        constexpr uint32_t kIdPV = umma_idesc(128, 128, true);
        const uint32_t sQ = smem_u32(dyn + kOffQ), sP = smem_u32(dyn + kOffP);
        int q = 0;
        bool issued = false;  // any MMA issued by this warp
        for (int f = 0; f < nfill && alive; ++f) {
            if (fill_valid(f) == 0) continue;
            const int st = q % kRtStages;
            if (lane == 0) alive = mbar_wait(&kv_full[st], (q / kRtStages) & 1, c.status);
            alive = __shfl_sync(0xffffffffu, alive, 0);
            if (!alive) break;
            tc_fence_after();
            const uint32_t sK = smem_u32(dyn + kOffRing + (size_t)st * kRtStage);
            const uint32_t sV = sK + 2 * kRtHalf;
            if (lane == 0) {
                // S = Q K^T: K = 128 channels in eight steps of 16 (32 bytes along the swizzled rows)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tm + kColS, umma_desc(sQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             umma_desc(sK + (kk >> 2) * kRtHalf + (kk & 3) * 32, 16, 1024), kIdQK, kk > 0);
                umma_commit(&s_full);
            }
            issued = true;
            __syncwarp();
            if (lane == 0) alive = mbar_wait(&p_full, q & 1, c.status);
            alive = __shfl_sync(0xffffffffu, alive, 0);
            if (!alive) break;
            tc_fence_after();
            if (lane == 0) {
                // O += P V: K = 64 tokens in four steps of 16 (two 8-row groups of the V tile each);
                // V is MN-major: its two 64-channel halves are 8 KB apart
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tm + kColO, umma_desc(sP + part * 16384 + kk * 32, 16, 1024),
                                 umma_desc(sV + kk * 2048, kRtHalf, 1024), kIdPV, (q > 0 || part > 0 || kk > 0));
                umma_commit(&pv_done);
                umma_commit(&kv_empty[st]);
            }
            __syncwarp();
            ++q;
        }
        // every MMA this warp issued has completed before TMEM can be released (also after a
        // wait that ran out)
        if (lane == 0 && issued) {
            umma_commit(&fin);
            mbar_wait(&fin, 0, c.status);
        }
        __syncwarp();
    } else {
        // ------------------------------ softmax ------------------------------
        const int r = tid;  // query row = TMEM lane
        const int gr = row0 + r;
        const int lim = gr < R ? pos0 + gr / G + 1 : 0;  // causal limit (exclusive)
        const uint32_t lane_base = tm + ((uint32_t)(warp * 32) << 16);
        float m_used = -INFINITY, l = 0.f;
        int q = 0;
        for (int f = 0; f < nfill && alive; ++f) {
            const int vf = fill_valid(f);
            if (vf == 0) continue;
            const int j = i0 + f / kSub, sb = f % kSub;
            const int base = j * kBlk + 64 * sb;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&s_full, q & 1, c.status);
            alive = __shfl_sync(0xffffffffu, ok, 0);
            if (!alive) break;
            tc_fence_after();
            float sv[64];
            tmem_ld64(lane_base + kColS, sv);
            float mx = -INFINITY;
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                sv[t] = (t < vf && base + t < lim) ? sv[t] * a.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[t]);
            }
            // the exponent offset moves only when the maximum grows by more than 2^8
            float alpha = 1.f;
            if (mx > -INFINITY && (m_used == -INFINITY || mx > m_used + 8.f)) {
                alpha = m_used == -INFINITY ? 0.f : exp2f(m_used - mx);
                m_used = mx;
                l *= alpha;
            }
            const bool rescale = q > 0 && alpha != 1.f;
            float lsum = 0.f;
            uint32_t ph[32], pl[32];
#pragma unroll
            for (int t = 0; t < 64; t += 2) {
                const float p0 = m_used == -INFINITY ? 0.f : exp2f(sv[t] - m_used);
                const float p1 = m_used == -INFINITY ? 0.f : exp2f(sv[t + 1] - m_used);
                lsum += p0 + p1;
                const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
                const float2 hf = __bfloat1622float2(hi);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                ph[t / 2] = *reinterpret_cast<const uint32_t*>(&hi);
                pl[t / 2] = *reinterpret_cast<const uint32_t*>(&lo);
            }
            l += lsum;
            // P and O are free once the previous O += P V has completed
            if (q > 0) {
                if (lane == 0) ok = mbar_wait(&pv_done, (q - 1) & 1, c.status);
                alive = __shfl_sync(0xffffffffu, ok, 0);
                if (!alive) break;
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, rescale)) {
                float ov[64];
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    tmem_ld64(lane_base + kColO + 64 * hlf, ov);
#pragma unroll
                    for (int e = 0; e < 64; ++e) ov[e] *= rescale ? alpha : 1.f;
                    tmem_st64(lane_base + kColO + 64 * hlf, ov);
                }
            }
            uint8_t* prow = dyn + kOffP + r * 128;
#pragma unroll
            for (int cch = 0; cch < 8; ++cch) {
                const int off = ((cch ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(prow + off) = make_uint4(ph[4 * cch], ph[4 * cch + 1], ph[4 * cch + 2], ph[4 * cch + 3]);
                *reinterpret_cast<uint4*>(prow + 16384 + off) =
                    make_uint4(pl[4 * cch], pl[4 * cch + 1], pl[4 * cch + 2], pl[4 * cch + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full);
            ++q;
        }
        // the split's normalised output of this row
        float ov[2][64];
        bool have = false;
        if (alive && q > 0) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&pv_done, (q - 1) & 1, c.status);
            have = __shfl_sync(0xffffffffu, ok, 0);
            if (have) {
                tc_fence_after();
                tmem_ld64(lane_base + kColO, ov[0]);
                tmem_ld64(lane_base + kColO + 64, ov[1]);
            }
        }
        if (gr < R) {
            const int ti = gr / G, g = gr % G;
            const int64_t orow = (((int64_t)s * a.M + ti) * c.H_q + h * G + g) * a.num_splits + sp;
            float* dst = a.o_part + orow * kHeadDim;
            const bool any = have && l > 0.f;
            const float inv = any ? 1.f / l : 0.f;
#pragma unroll
            for (int e = 0; e < 128; e += 4)
                *reinterpret_cast<float4*>(dst + e) =
                    any ? make_float4(ov[e >> 6][e & 63] * inv, ov[e >> 6][(e & 63) + 1] * inv,
                                      ov[e >> 6][(e & 63) + 2] * inv, ov[e >> 6][(e & 63) + 3] * inv)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
            a.lse_part[orow] = any ? (m_used + log2f(l)) * kLn2 : -INFINITY;
        }
    }
    // every role is done with TMEM: the allocating warp releases it
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(kTmemCols));
    }
}

template <int kBlk>
int launch_rect_t(const sba_cache& c, const RtArgs& a, int row_groups, cudaStream_t stream) {
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)c.num_pages * c.H_kv * kBlk;
    if (!make_kv_tmap(&tk, c.k, rows, 64) || !make_kv_tmap(&tv, c.v, rows, 64)) return SBA_ERR_CUDA;
    if (allow_smem<rect_tc_kernel<kBlk>>(kRtSmem) != SBA_OK) return SBA_ERR_CUDA;
    dim3 grid(a.num_splits, c.H_kv * row_groups, c.B);
    return launch(rect_tc_kernel<kBlk>, grid, dim3(kRtThreads), kRtSmem, stream, tk, tv, a);
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
    return c.b == 64 ? launch_rect_t<64>(c, a, row_groups, stream) : launch_rect_t<128>(c, a, row_groups, stream);
}

}  // namespace sba
