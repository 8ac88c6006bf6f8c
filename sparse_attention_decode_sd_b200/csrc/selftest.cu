// selftest.cu -- the bounded-wait path, run on purpose: one warp waits on a shared-memory mbarrier that
// nothing arrives on, with the same helper every pipeline wait of the library uses.  The wait must give
// up after its limit and record SD_ERR_TIMEOUT; no copy is ever issued, so nothing is left in flight.
#include "common.cuh"

namespace sd {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint64_t limit_ns, int32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0u, limit_ns));
    if (!ok && threadIdx.x == 0) report(status, SD_ERR_TIMEOUT);
}

}  // namespace sd

extern "C" sd_status sd_selftest_wait_timeout(uint32_t wait_ms, int32_t* dev_status, void* stream) {
    if (dev_status == nullptr || wait_ms < 1 || wait_ms > 10000) return SD_ERR_INVALID_ARG;
    sd::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)wait_ms * 1000000ull, dev_status);
    return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}
