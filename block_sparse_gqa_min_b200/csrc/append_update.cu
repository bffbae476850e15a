// KV append and block-descriptor maintenance.
//
// "Rectified Sparse Attention for Efficient Long-Sequence Generation", Summary:
// new tokens' KV entries and their block keys are written as decoding goes on,
// and a re-encoded window overwrites both.  Descriptors are RECOMPUTED from all
// valid tokens of every touched block, so an overwrite can lower a max or raise
// a min correctly.
//   Quest descriptor: per-channel min and max of the block's keys (exact bf16).
//   Gate key ("SAS: Simple Attention Sparsification ...", Limitations: pooled
//   block summaries; "SeerAttention-R ...", abstract: plug-in gate):
//   pooled = [max || min || avg] (3d), k' = Wk pooled, stored kg = Wq^T k' / sqrt(dg).
#include <math.h>

#include "common.cuh"
#include "launch.cuh"

namespace sba {

// One CTA per (token, sequence); each warp copies one KV head: lanes 0-15 move
// the 256-byte key row, lanes 16-31 the value row, 16 bytes per lane.
__global__ void __launch_bounds__(128) append_kv_kernel(sba_cache c, const uint4* __restrict__ k_new,
                                                        const uint4* __restrict__ v_new,
                                                        const int32_t* __restrict__ pos_start, int n_new) {
    pdl_wait();
    pdl_trigger();
    const int i = blockIdx.x, s = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pos = __ldg(pos_start + s) + i;
    if (pos < 0 || pos >= c.max_blocks * c.b) {
        if (threadIdx.x == 0) report(c.status, SBA_DEV_BAD_POSITION);
        return;
    }
    const int64_t page = page_of(c, s, pos / c.b, threadIdx.x == 0 ? c.status : nullptr);
    if (page < 0) return;
    const int row = pos % c.b;
    const int half = lane >> 4, l = lane & 15;
    for (int h = warp; h < c.H_kv; h += blockDim.x >> 5) {
        const uint4* src = (half ? v_new : k_new) + (((int64_t)s * n_new + i) * c.H_kv + h) * 16 + l;
        uint4* dst = reinterpret_cast<uint4*>(half ? c.v : c.k) + ((page * c.H_kv + h) * c.b + row) * 16 + l;
        *dst = __ldg(src);
    }
}

// One CTA (128 threads) per (touched block, KV head, sequence).  Thread t reads
// 16-byte chunk t%16 (8 channels) of rows t/16, t/16+8, ...; partial results
// of the 8 row groups are reduced through shared memory.
template <bool kQuest, bool kGate>
__global__ void __launch_bounds__(128) update_desc_kernel(sba_cache c, const int32_t* __restrict__ pos_start,
                                                          int n_new, sba_gate gate) {
    pdl_wait();
    pdl_trigger();
    __shared__ float red_mn[8][kHeadDim], red_mx[8][kHeadDim], red_sum[8][kHeadDim];
    __shared__ float pooled[3 * kHeadDim];
    __shared__ float kproj[256];

    const int s = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
    const int b = c.b;
    const int len = __ldg(c.seq_lens + s);
    const int N = blocks_of(len, b);
    const int p0 = __ldg(pos_start + s);
    if (p0 < 0 || (int64_t)p0 + n_new > (int64_t)c.max_blocks * b) {
        if (tid == 0 && blockIdx.x == 0 && h == 0) report(c.status, SBA_DEV_BAD_POSITION);
        return;
    }
    const int j = p0 / b + blockIdx.x;
    const int jlast = (p0 + n_new - 1) / b;
    if (j > jlast || j >= N) return;
    const int64_t page = page_of(c, s, j, tid == 0 ? c.status : nullptr);
    if (page < 0) return;
    const int cnt = min(b, len - j * b);

    const uint4* tile = reinterpret_cast<const uint4*>(c.k) + (page * c.H_kv + h) * (int64_t)b * 16;
    const int chunk = tid & 15, rg = tid >> 4;
    float mn[8], mx[8], sm[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        mn[e] = INFINITY;
        mx[e] = -INFINITY;
        sm[e] = 0.f;
    }
    for (int r = rg; r < cnt; r += 8) {
        const uint4 w = tile[r * 16 + chunk];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = bf16_lo(ws[e]), bb = bf16_hi(ws[e]);
            mn[2 * e] = fminf(mn[2 * e], a);
            mx[2 * e] = fmaxf(mx[2 * e], a);
            sm[2 * e] += a;
            mn[2 * e + 1] = fminf(mn[2 * e + 1], bb);
            mx[2 * e + 1] = fmaxf(mx[2 * e + 1], bb);
            sm[2 * e + 1] += bb;
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        red_mn[rg][chunk * 8 + e] = mn[e];
        red_mx[rg][chunk * 8 + e] = mx[e];
        red_sum[rg][chunk * 8 + e] = sm[e];
    }
    __syncthreads();
    // thread t now owns channel t
    float lo = red_mn[0][tid], hi = red_mx[0][tid], sum = red_sum[0][tid];
#pragma unroll
    for (int g = 1; g < 8; ++g) {
        lo = fminf(lo, red_mn[g][tid]);
        hi = fmaxf(hi, red_mx[g][tid]);
        sum += red_sum[g][tid];
    }
    if (kQuest) {
        __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(c.desc) + (page * c.H_kv + h) * 2 * kHeadDim;
        d[tid] = __float2bfloat16_rn(lo);  // exact: lo is one of the bf16 keys
        d[kHeadDim + tid] = __float2bfloat16_rn(hi);
    }
    if (kGate) {
        pooled[tid] = hi;
        pooled[kHeadDim + tid] = lo;
        pooled[2 * kHeadDim + tid] = sum / (float)cnt;
        __syncthreads();
        // k' = Wk . pooled : a warp takes four output rows at a time (their 3d inputs split over
        // the lanes, 48 loads in flight per lane), so the rows do not wait on each other
        const int warp = tid >> 5, lane = tid & 31;
        for (int r0 = 4 * warp; r0 < gate.dg; r0 += 16) {
            float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 3 * kHeadDim / 32; ++m) {
                const int i = lane + 32 * m;
                const float pv = pooled[i];
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    if (r0 + x < gate.dg) acc4[x] = fmaf(__ldg(gate.Wk + (int64_t)(r0 + x) * 3 * kHeadDim + i), pv, acc4[x]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                float acc = acc4[x];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (lane == 0 && r0 + x < gate.dg) kproj[r0 + x] = acc;
            }
        }
        __syncthreads();
        // kg = Wq^T k' / sqrt(dg): thread t reads column t of Wq (coalesced rows), four partial sums
        // with sixteen rows' loads in flight
        float accp[4] = {0.f, 0.f, 0.f, 0.f};
        int r = 0;
        for (; r + 16 <= gate.dg; r += 16) {
#pragma unroll
            for (int x = 0; x < 16; ++x)
                accp[x & 3] = fmaf(__ldg(gate.Wq + (int64_t)(r + x) * kHeadDim + tid), kproj[r + x], accp[x & 3]);
        }
        for (; r < gate.dg; ++r) accp[0] = fmaf(__ldg(gate.Wq + (int64_t)r * kHeadDim + tid), kproj[r], accp[0]);
        const float acc = (accp[0] + accp[1]) + (accp[2] + accp[3]);
        c.kg[(page * c.H_kv + h) * kHeadDim + tid] = acc * rsqrtf((float)gate.dg);
    }
}

int launch_append_kv(const sba_cache& c, const void* k_new, const void* v_new, const int32_t* pos_start, int n_new,
                     cudaStream_t stream) {
    dim3 grid(n_new, c.B);
    return launch(append_kv_kernel, grid, dim3(128), 0, stream, c, reinterpret_cast<const uint4*>(k_new),
                  reinterpret_cast<const uint4*>(v_new), pos_start, n_new);
}

int launch_update_descriptors(const sba_cache& c, const int32_t* pos_start, int n_new, const sba_gate* gate,
                              cudaStream_t stream) {
    const bool quest = c.desc != nullptr;
    const bool gated = gate != nullptr && c.kg != nullptr;
    if (!quest && !gated) return SBA_OK;
    const int touched = (n_new - 1) / c.b + 2;  // blocks a window of n_new positions can overlap
    dim3 grid(touched, c.H_kv, c.B);
    sba_gate g{};
    if (gate) g = *gate;
    if (quest && gated) return launch(update_desc_kernel<true, true>, grid, dim3(128), 0, stream, c, pos_start, n_new, g);
    if (quest) return launch(update_desc_kernel<true, false>, grid, dim3(128), 0, stream, c, pos_start, n_new, g);
    return launch(update_desc_kernel<false, true>, grid, dim3(128), 0, stream, c, pos_start, n_new, g);
}

}  // namespace sba
