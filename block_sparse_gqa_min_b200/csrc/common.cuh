// Device helpers shared by the libsba kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sba.h"

namespace sba {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 16;
constexpr int kMaxBlocksPerSeq = 32768;  // selection keys live in shared memory
constexpr int kMaxQueryTokens = 1024;   // query tokens per sequence of the multi-token calls
constexpr int kMaxRectifyTokens = 128;  // rectification window: the pages' largest f
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bounded waits give up after ~2 s

// ---------------------------------------------------------------------------
// Small arithmetic helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Order-preserving map fp32 -> u32 (larger float, larger key).  -0 is first
// turned into +0 so that the two compare equal.
__device__ __forceinline__ uint32_t orderable_key(float f) {
    f = f + 0.0f;
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// log g of a historical block from its gate logit u ("SAS ...", Method, and the activations
// of its ablations): softmax u - LSE; unnormalised u (pass lse = 0); sigmoid
// log(1 / (1 + exp(-u))), written without overflow on either side.
__device__ __forceinline__ float log_gate_of(float u, float lse, int act) {
    if (act != SBA_GATE_SIGMOID) return u - lse;
    return fminf(u, 0.f) - log1pf(expf(-fabsf(u)));
}

// The gate g itself, as the group's ranking sums it: exp(u - lse) (softmax, raw with lse = 0)
// or 1 / (1 + exp(-u)) (sigmoid).
__device__ __forceinline__ float gate_of(float u, float lse, int act) {
    return act == SBA_GATE_SIGMOID ? 1.f / (1.f + expf(-u)) : expf(u - lse);
}

__device__ __forceinline__ void report(int32_t* status, int bit) {
    if (status) atomicOr(status, bit);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Physical page of logical block j of sequence s, or -1 (and a status bit)
// when the table entry is out of range.
__device__ __forceinline__ int64_t page_of(const sba_cache& c, int s, int j, int32_t* status) {
    int64_t p = c.block_table ? (int64_t)__ldg(c.block_table + (int64_t)s * c.max_blocks + j)
                              : (int64_t)s * c.max_blocks + j;
    if (p < 0 || p >= c.num_pages) {
        report(status, SBA_DEV_BAD_PAGE);
        return -1;
    }
    return p;
}

__device__ __forceinline__ int blocks_of(int len, int b) { return len <= 0 ? 0 : (len + b - 1) / b; }

// Selection size for a sequence of N blocks (the rule documented in sba.h).
__host__ __device__ __forceinline__ int num_selected(int N, const sba_select_params& p) {
    if (N <= 0) return 0;
    int budget = p.n_budget;
    if (p.keep_den > 0) budget = (int)(((int64_t)N * p.keep_num + p.keep_den - 1) / p.keep_den);
    int L = p.n_local;
    if (p.scorer == SBA_SCORER_GATE && L < 1) L = 1;
    if (L > N) L = N;
    int n = budget;
    if (p.n_min > n) n = p.n_min;
    if (L > n) n = L;
    return n < N ? n : N;
}

__host__ __device__ __forceinline__ int num_local(int N, const sba_select_params& p) {
    int L = p.n_local;
    if (p.scorer == SBA_SCORER_GATE && L < 1) L = 1;
    return L < N ? L : (N > 0 ? N : 0);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PDL): wait for the grids this one depends on;
// let the next grid in the stream get scheduled.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// mbarrier + TMA (cp.async.bulk.tensor) wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase.  Returns false (and reports
// SBA_DEV_TIMEOUT) if the phase did not complete within `limit_ns`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status,
                                          uint64_t limit_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            report(status, SBA_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The same wait, each try suspending the thread until the phase completes or about
// `hint_ns` pass: a waiting warp then takes no issue slots from the working ones.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, int32_t* status,
                                                uint32_t hint_ns = 20000) {
    if (mbar_try_wait_hint(bar, parity, hint_ns)) return true;
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_hint(bar, parity, hint_ns)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
            report(status, SBA_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
// x is the innermost (element) coordinate, y the row coordinate.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 4-D tiled TMA load of one box (coordinates innermost first), completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// 16-byte asynchronous copy global -> this CTA's shared memory (cached in L2
// only).  Both addresses 16-byte aligned.  Many small scattered copies go
// through the load/store unit at full rate, unlike one bulk copy each.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

// Make `bar` track this thread's earlier cp.async copies: its pending count is
// raised now and lowered when they have landed, so the phase cannot complete
// before them (this is not an arrival of its own).
__device__ __forceinline__ void cp_async_mbar_track(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 16-byte global load that does not allocate in L1 (data read once per step).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// Generic-proxy global writes made visible to later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters and distributed shared memory
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}

// Every thread of every CTA of the cluster; release/acquire at cluster scope.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory variable in CTA `peer` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t peer) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(peer));
    return r;
}

__device__ __forceinline__ uint32_t ld_peer_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float ld_peer_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 ld_peer_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 );
    return v;
}

__device__ __forceinline__ uint32_t atom_add_peer_u32(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_peer_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_peer_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core helpers (bf16 inputs, fp32 accumulate)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
// An 8x8 matrix of 16-bit values transposed across the warp: lane l holds row l/4,
// columns 2(l%4) and 2(l%4)+1, before and after.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B on tensor cores, tf32 inputs, fp32 accumulate (m16n8k8).
__device__ __forceinline__ void mma_tf32_1688(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace sba
