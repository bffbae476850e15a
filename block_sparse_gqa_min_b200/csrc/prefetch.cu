// L2 prefetch of a layer's block descriptors, to overlap the step before it.
//
// Scoring reads every descriptor of a layer ("Rectified Sparse Attention ...",
// Key points: the 1/b term of the per-step memory; "SAS ...", Limitations: at
// very long contexts the block scan dominates decode), and those reads depend
// only on the cache, never on the query.  A decode step of a layer is a chain
// of dependent phases (scores -> selection -> sparse attention -> merge) whose
// later phases leave HBM mostly idle; this kernel asks the L2 to fetch the NEXT
// layer's descriptors during that time, so that the next step's scan reads
// them from L2.
//
// It is a hint: it writes nothing.  It is launched with programmatic dependent
// launch, so it runs while the kernel before it in the stream is still
// running; it then waits for that kernel (griddepcontrol.wait) before it
// exits, so every kernel after it still sees the one before it completed.
// The lengths it reads before that wait only size the prefetch.
#include "common.cuh"
#include "launch.cuh"

namespace sba {

namespace {

constexpr int kPfThreads = 32;
constexpr uint32_t kPfChunk = 16384;  // bytes per bulk prefetch instruction

__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

struct PfArgs {
    const uint8_t* desc;        // [num_pages][H_kv][512 B]
    const int32_t* seq_lens;
    const int32_t* block_table;
    int B, H_kv, b, max_blocks, num_pages;
};

__global__ void __launch_bounds__(kPfThreads) prefetch_desc_kernel(PfArgs a) {
    pdl_trigger();  // the next kernel may be scheduled at once
    const int lane = threadIdx.x;
    const uint32_t row = (uint32_t)a.H_kv * 512u;  // one page's descriptors
    for (int s = 0; s < a.B; ++s) {
        const int len = __ldg(a.seq_lens + s);
        const int N = min(len <= 0 ? 0 : (len + a.b - 1) / a.b, a.max_blocks);
        if (!a.block_table) {
            // contiguous pages: one range per sequence, split over the grid in chunks
            const uint8_t* base = a.desc + (int64_t)s * a.max_blocks * row;
            const uint64_t bytes = (uint64_t)N * row;
            const uint64_t nch = (bytes + kPfChunk - 1) / kPfChunk;
            for (uint64_t ch = (uint64_t)blockIdx.x * kPfThreads + lane; ch < nch; ch += (uint64_t)gridDim.x * kPfThreads) {
                const uint64_t off = ch * kPfChunk;
                const uint64_t n = bytes - off < kPfChunk ? bytes - off : kPfChunk;
                prefetch_l2_bulk(base + off, (uint32_t)n);
            }
        } else {
            // paged: each valid block's page row (entries outside [0, num_pages) are skipped)
            for (int j = blockIdx.x * kPfThreads + lane; j < N; j += gridDim.x * kPfThreads) {
                const int p = __ldg(a.block_table + (int64_t)s * a.max_blocks + j);
                if (p >= 0 && p < a.num_pages) prefetch_l2_bulk(a.desc + (int64_t)p * row, row);
            }
        }
    }
    pdl_wait();  // complete only after the kernel before this one: stream order is kept
}

}  // namespace

int launch_prefetch_descriptors(const sba_cache& c, int num_sms, cudaStream_t stream) {
    PfArgs a{};
    a.desc = reinterpret_cast<const uint8_t*>(c.desc ? c.desc : (void*)c.kg);
    a.seq_lens = c.seq_lens;
    a.block_table = c.block_table;
    a.B = c.B;
    a.H_kv = c.H_kv;
    a.b = c.b;
    a.max_blocks = c.max_blocks;
    a.num_pages = c.num_pages;
    return launch(prefetch_desc_kernel, dim3(num_sms), dim3(kPfThreads), 0, stream, a);
}

}  // namespace sba
