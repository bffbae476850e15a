// Exact top-k selection with index-order tie-break over fp32 score keys in
// shared memory ("Rectified Sparse Attention ...", Key points: top-n of the
// non-local blocks; the locals are always kept).  Shared by the scoring kernel
// and the fused decode-step kernel.
#pragma once

#include "common.cuh"

namespace sba {

// Exclusive prefix of per-warp totals held in shared memory.
__device__ __forceinline__ int warp_prefix(const int* warp_tot, int warp) {
    int acc = 0;
    for (int w = 0; w < warp; ++w) acc += warp_tot[w];
    return acc;
}

// ---------------------------------------------------------------------------
// Selection over NC ranked candidates (keys in smem) plus the forced local
// blocks [NC, N).  Writes ascending indices to out[0..min(n_sel, n_max)).
// k = number of candidates to take.  Runs on all kNT threads of the CTA;
// hist needs 256 words, warp_tot kNT/32 ints, sh 2 words (shared memory).
// ---------------------------------------------------------------------------
template <int kNT>
__device__ void select_and_compact(const uint32_t* keys, int NC, int N, int k, int32_t* out, int n_max,
                                   uint32_t* hist, int* warp_tot, uint32_t* sh) {
    constexpr int kWarps = kNT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // mode: 0 = threshold (0 < k < NC), 1 = take all candidates, 2 = take none
    const int mode = k >= NC ? 1 : (k <= 0 ? 2 : 0);
    uint32_t T = 0;
    int rem = 0;
    if (mode == 0) {
        uint32_t prefix = 0, pmask = 0;
        rem = k;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += kNT) hist[i] = 0;
            __syncthreads();
            // warp-aggregated histogram: float keys crowd into few bins (the top byte is sign +
            // exponent), so lanes that share a bin add once, as a group
            for (int j0 = warp * 32; j0 < NC; j0 += kNT) {
                const int j = j0 + lane;
                bool in = false;
                uint32_t bin = 256u + lane;  // unique dummy bin for inactive lanes
                if (j < NC) {
                    const uint32_t kk = keys[j];
                    if ((kk & pmask) == prefix) {
                        in = true;
                        bin = (kk >> shift) & 255u;
                    }
                }
                const unsigned same = __match_any_sync(0xffffffffu, bin);
                if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(same));
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t cnt[8], lsum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cnt[e] = hist[255 - 8 * lane - e];
                    lsum += cnt[e];
                }
                uint32_t incl = lsum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                const uint32_t excl = incl - lsum;
                if (excl < (uint32_t)rem && (uint32_t)rem <= incl) {
                    uint32_t run = excl;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (run + cnt[e] >= (uint32_t)rem) {
                            sh[0] = prefix | ((uint32_t)(255 - 8 * lane - e) << shift);
                            sh[1] = (uint32_t)rem - run;
                            break;
                        }
                        run += cnt[e];
                    }
                }
            }
            __syncthreads();
            prefix = sh[0];
            rem = (int)sh[1];
            pmask |= 0xffu << shift;
        }
        T = prefix;  // exact key of the n-th candidate; `rem` equal keys are taken, lowest index first
    }
    // Per-warp contiguous segments, processed 32 consecutive indices at a time,
    // so that ranks among equal keys and output positions follow index order.
    const int seg = ((N + kWarps * 32 - 1) / (kWarps * 32)) * 32;
    const int jb = warp * seg, je = min(N, jb + seg);
    const unsigned lt = (1u << lane) - 1u;
    // pass A: ties per warp
    int eq_w = 0;
    if (mode == 0)
        for (int base = jb; base < je; base += 32) {
            const int j = base + lane;
            const bool is_eq = j < je && j < NC && keys[j] == T;
            eq_w += __popc(__ballot_sync(0xffffffffu, is_eq));
        }
    if (lane == 0) warp_tot[warp] = eq_w;
    __syncthreads();
    const int eq_before = warp_prefix(warp_tot, warp);
    __syncthreads();
    // pass B: selected per warp; pass C: write
    for (int pass = 0; pass < 2; ++pass) {
        int er = eq_before, sel_run = 0;
        int out_base = 0;
        if (pass == 1) out_base = warp_prefix(warp_tot, warp);
        for (int base = jb; base < je; base += 32) {
            const int j = base + lane;
            bool sel = false, is_eq = false;
            if (j < je) {
                if (j >= NC) {
                    sel = true;
                } else if (mode == 1) {
                    sel = true;
                } else if (mode == 0) {
                    const uint32_t kk = keys[j];
                    is_eq = kk == T;
                    sel = kk > T;
                }
            }
            const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
            if (is_eq) sel = (er + __popc(eqm & lt)) < rem;
            er += __popc(eqm);
            const unsigned sm = __ballot_sync(0xffffffffu, sel);
            if (pass == 1 && sel) {
                const int pos = out_base + sel_run + __popc(sm & lt);
                if (pos < n_max) out[pos] = j;
            }
            sel_run += __popc(sm);
        }
        if (pass == 0) {
            __syncthreads();
            if (lane == 0) warp_tot[warp] = sel_run;
            __syncthreads();
        }
    }
}


// ---------------------------------------------------------------------------
// Fast exact top-k for the same contract as select_and_compact.  Every step
// gives each thread independent work (four keys per 16-byte load, rank
// counting over broadcast reads) so that few warps still run at throughput:
// 1. group maxima over groups of gs consecutive candidates, gs the largest of
//    4..128 that still leaves >= 2k groups (every group maximum is a candidate);
// 2. T0 = the k-th largest group maximum, by counting for every group maximum
//    the ones above it.  The k largest group maxima are k distinct candidates
//    >= T0, so every top-k candidate is >= T0;
// 3. the candidates >= T0 go to a buffer; if more than `cap` pass,
//    select_and_compact is used instead;
// 4. every buffered candidate is ranked by counting the buffered candidates
//    that beat it (larger key, or equal key and lower index): the ranks are
//    unique, so rank < k is exactly the top-k;
// 5. winners are written in ascending index order (their rank by index among
//    the winners), then the locals.
// keys must be 16-byte aligned.  Scratch (shared memory): gmax [ceil(NC/4)]
// words, bkey/bidx/brank [cap] words each, misc [2] ints.
// ---------------------------------------------------------------------------
template <int kNT>
__device__ __noinline__ void select_fast(const uint32_t* keys, int NC, int N, int k, int32_t* out, int n_max, uint32_t* gmax,
                            uint32_t* bkey, int* bidx, int* brank, int cap, int* misc, uint32_t* hist, int* warp_tot,
                            uint32_t* sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || k >= NC) {
        // all candidates or none, then the locals: already ascending
        const int first = k <= 0 ? NC : 0;
        for (int i = tid; i < N - first; i += kNT)
            if (i < n_max) out[i] = first + i;
        return;
    }
    int gs = 128;
    while (gs > 4 && (NC + gs - 1) / gs < 2 * k) gs >>= 1;
    const int lpg = gs / 4;                  // lanes per group (1..32)
    const int ng = (NC + gs - 1) / gs;
    const int nv = (NC + 3) / 4;             // 16-byte key vectors
    const uint4* kv = reinterpret_cast<const uint4*>(keys);
    // 1. group maxima
    for (int v0 = warp * 32; v0 < nv; v0 += kNT) {
        const int v = v0 + lane;
        uint32_t m = 0;
        if (v < nv) {
            const uint4 q = kv[v];
            const int j = 4 * v;
            m = max(max(j < NC ? q.x : 0u, j + 1 < NC ? q.y : 0u), max(j + 2 < NC ? q.z : 0u, j + 3 < NC ? q.w : 0u));
        }
        for (int o = 1; o < lpg; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((lane & (lpg - 1)) == 0 && v < nv) gmax[v / lpg] = m;
    }
    if (tid == 0) {
        misc[0] = ng >= k ? -1 : 0;  // T0 (unsigned min over candidates); no bound from < k groups
        misc[1] = 0;                 // buffer count
    }
    __syncthreads();
    // 2. T0 = smallest group maximum with fewer than k group maxima above it
    for (int g0 = warp * 32; g0 < ng && ng >= k; g0 += kNT) {
        const int g = g0 + lane;
        uint32_t cand = 0xffffffffu;
        if (g < ng) {
            const uint32_t x = gmax[g];
            int above = 0;
#pragma unroll 4
            for (int t = 0; t < ng; ++t) above += gmax[t] > x;
            if (above < k) cand = x;
        }
        cand = __reduce_min_sync(0xffffffffu, cand);
        if (lane == 0 && cand != 0xffffffffu) atomicMin(reinterpret_cast<unsigned*>(&misc[0]), cand);
    }
    __syncthreads();
    const uint32_t T0 = (uint32_t)misc[0];
    // 3. filter the candidates >= T0 into the buffer (four keys per thread)
    for (int v0 = warp * 32; v0 < nv; v0 += kNT) {
        const int v = v0 + lane;
        uint32_t q[4] = {0u, 0u, 0u, 0u};
        int n = 0;
        if (v < nv) {
            const uint4 w = kv[v];
            q[0] = w.x;
            q[1] = w.y;
            q[2] = w.z;
            q[3] = w.w;
#pragma unroll
            for (int e = 0; e < 4; ++e) n += (4 * v + e < NC) && q[e] >= T0;
        }
        int incl = n;  // inclusive scan of the counts over the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        int base = 0;
        if (lane == 31 && incl) base = atomicAdd(&misc[1], incl);
        base = __shfl_sync(0xffffffffu, base, 31) + incl - n;
        if (n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 4 * v + e;
                if (j < NC && q[e] >= T0) {
                    if (base < cap) {
                        bkey[base] = q[e];
                        bidx[base] = j;
                    }
                    ++base;
                }
            }
        }
    }
    __syncthreads();
    const int m = misc[1];
    if (m > cap) {
        select_and_compact<kNT>(keys, NC, N, k, out, n_max, hist, warp_tot, sh);
        return;
    }
    // 4. unique ranks: (key desc, index asc)
    for (int i = tid; i < m; i += kNT) {
        const uint32_t ki = bkey[i];
        const int xi = bidx[i];
        int r = 0;
#pragma unroll 4
        for (int t = 0; t < m; ++t) {
            const uint32_t kt = bkey[t];
            r += (kt > ki) | ((kt == ki) & (bidx[t] < xi));
        }
        brank[i] = r;
    }
    __syncthreads();
    // 5. winners in ascending index order, then the locals
    for (int i = tid; i < m; i += kNT) {
        if (brank[i] >= k) continue;
        const int xi = bidx[i];
        int pos = 0;
#pragma unroll 4
        for (int t = 0; t < m; ++t) pos += (brank[t] < k) & (bidx[t] < xi);
        if (pos < n_max) out[pos] = xi;
    }
    for (int i = tid; i < N - NC; i += kNT)
        if (k + i < n_max) out[k + i] = NC + i;
}

}  // namespace sba
