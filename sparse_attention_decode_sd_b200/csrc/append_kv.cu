// append_kv.cu -- one decode step's K/V row per request written into its page (the growing cache
// of an agentic decode loop), plus the length and per-request k that the next step uses.
#include "common.cuh"
#include "kernels.h"

namespace sd {

__global__ void __launch_bounds__(128) append_kernel(AppendArgs a) {
    pdl_enter();
    const int b = blockIdx.x;
    __shared__ long s_row;
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        const int p = a.lens[b];
        int ok = 1;
        if (p < 0 || (long)p >= (long)a.max_pages * kPageSize) {
            report(a.status, SD_ERR_INVALID_ARG);
            ok = 0;
        } else {
            const int page = a.page_table[(long)b * a.max_pages + p / kPageSize];
            if (page < 0 || page >= a.num_pages) {
                report(a.status, SD_ERR_INDEX_OOB);
                ok = 0;
            } else {
                s_row = ((long)page * kPageSize + (p % kPageSize)) * a.Hkv;
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    if (!s_ok) return;
    for (int i = threadIdx.x; i < a.Hkv * 16; i += blockDim.x) {
        const int kvh = i >> 4, ch = i & 15;
        const long dst = (s_row + kvh) * kHeadDim + ch * 8;
        const long src = ((long)b * a.Hkv + kvh) * kHeadDim + ch * 8;
        *reinterpret_cast<uint4*>(a.K + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
        *reinterpret_cast<uint4*>(a.V + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int n = a.lens[b] + 1;
        a.lens[b] = n;
        if (a.k_sel != nullptr) a.k_sel[b] = max(1, (int)((2L * n + a.ratio) / (2L * a.ratio)));
    }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(append_kernel, dim3(a.B), dim3(128), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
