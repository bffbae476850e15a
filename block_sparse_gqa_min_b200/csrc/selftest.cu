// Self-test of the bounded waits every kernel of the library uses.
//
// One warp initialises an mbarrier that nothing ever arrives on and waits on its
// first phase with the library's own bounded wait (mbar_wait), limited to the
// caller's `limit_ns`: the wait runs out, reports SBA_DEV_TIMEOUT into the status
// word and the kernel returns, so the host sees the failure as data and the
// context stays usable.  No trap, no fault and no unbounded loop is involved.
#include "common.cuh"
#include "launch.cuh"

namespace sba {
namespace {

__global__ void wait_timeout_selftest_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    bool ok = true;
    if (threadIdx.x == 0) ok = mbar_wait(&bar, 0, status, limit_ns);  // nothing arrives: runs out
    ok = __shfl_sync(0xffffffffu, ok, 0);
    (void)ok;
}

}  // namespace

int launch_wait_timeout_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

}  // namespace sba
