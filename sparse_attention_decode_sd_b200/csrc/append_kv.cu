// append_kv.cu -- one decode step's K/V row per request written into its page (the growing cache
// of an agentic decode loop), plus the length and per-request k that the next step uses.  With Quest
// boxes ("The Sparse Frontier" review, sec. 7.1: per page and KV head the per-dimension minimum and
// maximum of its keys) the box of the written page is brought up to date in the same pass: the new
// key row alone when it opens the page, else the elementwise min / max with the stored box (min and
// max are associative, so the result equals a summary of the page's rows).
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
    const bool opens_page = (a.lens[b] % kPageSize) == 0;   // read before the length is advanced below
    for (int i = threadIdx.x; i < a.Hkv * 16; i += blockDim.x) {
        const int kvh = i >> 4, ch = i & 15;
        const long dst = (s_row + kvh) * kHeadDim + ch * 8;
        const long src = ((long)b * a.Hkv + kvh) * kHeadDim + ch * 8;
        const uint4 kr = *reinterpret_cast<const uint4*>(a.k_new + src);
        *reinterpret_cast<uint4*>(a.K + dst) = kr;
        *reinterpret_cast<uint4*>(a.V + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
        if (a.boxes != nullptr) {
            const long page = s_row / ((long)kPageSize * a.Hkv);
            uint4* bmin = reinterpret_cast<uint4*>(a.boxes + ((page * a.Hkv + kvh) * 2) * kHeadDim + ch * 8);
            uint4* bmax = reinterpret_cast<uint4*>(a.boxes + ((page * a.Hkv + kvh) * 2 + 1) * kHeadDim + ch * 8);
            if (opens_page) {
                *bmin = kr;
                *bmax = kr;
            } else {
                uint4 lo = *bmin, hi = *bmax;
                uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
                uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
                const uint32_t* k = reinterpret_cast<const uint32_t*>(&kr);
#pragma unroll
                for (int t = 0; t < 4; ++t) {   // bf16 pairs: min and max are exact
                    const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162*>(&k[t]);
                    const __nv_bfloat162 mn = __hmin2(*reinterpret_cast<const __nv_bfloat162*>(&l[t]), kv);
                    const __nv_bfloat162 mx = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&h[t]), kv);
                    l[t] = *reinterpret_cast<const uint32_t*>(&mn);
                    h[t] = *reinterpret_cast<const uint32_t*>(&mx);
                }
                *bmin = lo;
                *bmax = hi;
            }
        }
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
