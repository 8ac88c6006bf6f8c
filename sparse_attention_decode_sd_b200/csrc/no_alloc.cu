// no_alloc.cu -- sd_topk_index_static: the exact top-k indexer for callers that cannot allocate
// device memory, so cannot provide the indexer's workspace themselves.  Examples: a plugin running
// inside a host engine that hands it only its inputs and outputs; a service whose device memory is
// planned once at start-up and may not grow; code that runs on the calling thread while that thread
// must not call cudaMalloc (which synchronises the device and is not a stream operation).
//
// The indexer's workspace (fp32 score rows or candidate pairs, thresholds, candidate counts) lives instead in one
// file-scope device array of kStaticScratchBytes (48 MiB).  Every GPU that loads this library holds
// that array until the process exits.  The call itself allocates nothing: no cudaMalloc, no
// cudaFree, no allocating library routine.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = 48u << 20;   // 48 MiB
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a host-side handle for the symbol, not a device
// address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) float sd_static_scratch[kStaticScratchBytes / sizeof(float)];

std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device (with that
// device current) on its first call and kept.  The address belongs to the device's context: after
// a cudaDeviceReset the library's device code is loaded again, so the entry point must not be
// called after a reset in the same process (documented in the header).
sd_status static_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, sd_static_scratch) != cudaSuccess || p == nullptr) return SD_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return SD_OK;
}

}  // namespace

extern "C" sd_status sd_topk_index_static(const sd_shape* shape, const void* q, const void* K,
                                          const int32_t* page_table, const int32_t* lens, const int32_t* k,
                                          int32_t* idx, int32_t* dev_status, void* stream) {
    size_t need = 0;
    sd_status st = sd_workspace_size(shape, SD_OP_TOPK, &need);
    if (st != SD_OK) return st;
    if (need > kStaticScratchBytes) return SD_ERR_WORKSPACE;   // the shape's indexer workspace exceeds 48 MiB
    void* scratch = nullptr;
    st = static_scratch(&scratch);
    if (st != SD_OK) return st;
    // Nothing in the scratch has to start at zero: each call resets the counters it accumulates and
    // writes every score and candidate its selection reads.  Successive calls reuse the same array.
    return sd_topk_index(shape, q, K, page_table, lens, k, idx, scratch, kStaticScratchBytes, dev_status, stream);
}
