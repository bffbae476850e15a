// sba_score_select_static: sba_score_select for callers that cannot allocate.
//
// Some callers cannot allocate device memory at the point where they issue a
// decode step: an engine that records its step into a CUDA graph and forbids
// cudaMalloc while a stream is capturing, a plugin inside a serving framework
// whose enqueue callback must not allocate, or an embedded runtime that hands
// out a fixed device-memory budget once at start-up.  This entry point needs
// no workspace from them: the scoring scratch is one file-scope device array,
// reserved when the library is loaded and held by every GPU that loads the
// library until the process exits.
//
// Rules (also stated in include/sba.h):
//  - at most kStaticScratchBytes of scratch; a problem needing more is
//    rejected with SBA_ERR_WORKSPACE before anything is enqueued;
//  - the first call on a device looks up the array's device address
//    (cudaGetSymbolAddress, once per device, with that device current), so
//    make that first call before any stream capture; the address is kept with
//    the device's context and looked up again if the context changes (after a
//    cudaDeviceReset the module, and with it the array, is loaded anew);
//  - every call on a device shares the one array, which keeps the previous
//    call's contents: each call clears the completion counters first
//    (cudaMemsetAsync on the caller's stream); calls whose kernels can overlap
//    on the GPU (different streams with no ordering) race on the array;
//  - nothing here calls cudaMalloc, cudaFree or an allocating library routine.
// The scoring itself is the unchanged sba_score_select path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/sba.h"
#include "launch.cuh"

namespace sba {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device

// The scratch.  In host code this name is only a host-side stand-in, never a
// device address: kernels receive the address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_score_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
    CUcontext ctx;  // the context the address belongs to
    void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The current context (the driver's cuCtxGetCurrent through the runtime's entry point,
// so the library needs no libcuda link), or nullptr.
CUcontext current_context() {
    static PFN_cuCtxGetCurrent_v4000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    }();
    CUcontext ctx = nullptr;
    if (fn) fn(&ctx);
    return ctx;
}

// Device address of g_score_scratch on the current device, looked up once per device and
// context.
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        note_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return SBA_ERR_CUDA;
    }
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!ctx || !g_scratch[dev].ptr || g_scratch[dev].ctx != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_score_scratch);  // (makes the primary context current if none is)
        if (e != cudaSuccess || !p) {
            note_cuda_error(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
            return SBA_ERR_CUDA;
        }
        g_scratch[dev] = ScratchAddr{current_context(), p};
    }
    *out = g_scratch[dev].ptr;
    return SBA_OK;
}

}  // namespace
}  // namespace sba

extern "C" {

size_t sba_static_scratch_bytes(void) { return sba::kStaticScratchBytes; }

int sba_score_select_static(const sba_cache* c, const void* q, const sba_select_params* p, int32_t* sel_idx,
                            int32_t* sel_cnt, float* gate_bias, int32_t n_max, void* stream) {
    // every argument check of sba_score_select, done before anything is enqueued (a rejected
    // call leaves nothing on the stream)
    const int rc0 = sba::check_score_select(c, q, p, sel_idx, sel_cnt, n_max);
    if (rc0 != SBA_OK) return rc0;
    const size_t need = sba_workspace_size(c, p);
    if (need == 0) return SBA_ERR_INVALID_ARG;
    if (need > sba::kStaticScratchBytes) return SBA_ERR_WORKSPACE;
    void* ws = nullptr;
    int rc = sba::scratch_address(&ws);
    if (rc != SBA_OK) return rc;
    // the completion counters (the first region of the scratch) must start at zero
    const size_t counter_bytes = (sizeof(uint32_t) * (size_t)c->B * c->H_kv + 255) & ~size_t(255);
    const cudaError_t e = cudaMemsetAsync(ws, 0, counter_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        sba::note_cuda_error(e);
        return SBA_ERR_CUDA;
    }
    return sba_score_select(c, q, p, sel_idx, sel_cnt, gate_bias, n_max, ws, sba::kStaticScratchBytes, stream);
}

}  // extern "C"
