// quest.cu -- the Quest page-level approximate indexer ("The Sparse Frontier" review (xllm),
// sec. 7.1 "Quest", Table 1, memory model Eq. 10): the KV cache is cut into pages of 16 positions;
// each page is represented, per KV head, by the per-dimension minimum and maximum of its keys; for
// every decode query and query head the most relevant pages are kept, always including the page of
// the current (last) position.  Relevance of page j (the pages do not spell it out; this is the
// largest q.k any key inside the page's [min, max] box can reach):
//     r_j = sum_d max(q_d * min_d, q_d * max_d) = q+ . max + q- . min,   q+ = max(q, 0), q- = min(q, 0).
// The output is the same idx rows as the exact indexer (every position of the kept pages, ascending,
// then -1), so sd_sparse_decode consumes it unchanged.
//
//   quest_summarize_kernel  boxes of every logical page of every request (or only of each request's
//                           last page, after an append), from the rows that exist (positions < N_b)
//   quest_score_kernel      r for every page of every (b, h): 16 pages x G heads per tensor-core tile,
//                           the 256-wide contraction [max | min] . [q+ ; q-] (mma.sync m16n8k16)
//   quest_select_kernel     per (b, h): the current page plus the ceil(k_b / 16) - 1 most relevant other
//                           pages (exact radix select, ties to the lower page), expanded to positions
#include "common.cuh"
#include "kernels.h"
#include "radix_select.cuh"

namespace sd {

// ---------------------------------------------------------------------------------------------
// summarize: one warp per (request, logical page, kv head); lane l owns dims 4l .. 4l + 3
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quest_summarize_kernel(QuestArgs a, long units) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long u = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (u >= units) return;
    // unit u = (b, page slot, kvh); with last_only one page slot per request
    const int kvh = (int)(u % a.Hkv);
    const long bj = u / a.Hkv;
    const int pages_per_req = a.last_only ? 1 : a.max_pages;
    const int b = (int)(bj / pages_per_req);
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int np = (n + kPageSize - 1) / kPageSize;
    const int j = a.last_only ? np - 1 : (int)(bj % pages_per_req);
    if (j < 0 || j >= np) return;
    const int page = a.page_table[(long)b * a.max_pages + j];
    if (page < 0 || page >= a.num_pages) {
        if (lane == 0) report(a.status, SD_ERR_INDEX_OOB);
        return;
    }
    const int rows = min(kPageSize, n - j * kPageSize);
    // all 16 row loads in flight together (rows past N_b repeat row 0, which leaves min and max unchanged)
    uint2 v[kPageSize];
#pragma unroll
    for (int r = 0; r < kPageSize; ++r)
        v[r] = *reinterpret_cast<const uint2*>(a.K + (((long)page * kPageSize + (r < rows ? r : 0)) * a.Hkv + kvh) *
                                                   kHeadDim + 4 * lane);
    float mn[4], mx[4];
#pragma unroll
    for (int r = 0; r < kPageSize; ++r) {
        const float f[4] = {bf16_lo(v[r].x), bf16_hi(v[r].x), bf16_lo(v[r].y), bf16_hi(v[r].y)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            mn[e] = r ? fminf(mn[e], f[e]) : f[e];
            mx[e] = r ? fmaxf(mx[e], f[e]) : f[e];
        }
    }
    // min and max of bf16 values are bf16 values: the conversions below are exact
    __nv_bfloat16* box = a.boxes + ((long)page * a.Hkv + kvh) * 2 * kHeadDim;
    *reinterpret_cast<uint2*>(box + 4 * lane) = make_uint2(pack_bf16x2(mn[0], mn[1]), pack_bf16x2(mn[2], mn[3]));
    *reinterpret_cast<uint2*>(box + kHeadDim + 4 * lane) = make_uint2(pack_bf16x2(mx[0], mx[1]), pack_bf16x2(mx[2], mx[3]));
}

// ---------------------------------------------------------------------------------------------
// score: one warp per (request, kv head, 16 pages)
// ---------------------------------------------------------------------------------------------
// Fragments of one 256-byte row (global memory) in the A-operand word order of the tile below: thread
// c = lane & 3 holds 16-byte chunks c, c + 4, c + 8, c + 12 (the contraction index is permuted the
// same way in q, which leaves every dot product unchanged).
__device__ __forceinline__ void load_row_frags(const __nv_bfloat16* row, int c, uint32_t (&R)[16]) {
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(r4 + c + 4 * i);
        R[4 * i + 0] = v.x;
        R[4 * i + 1] = v.y;
        R[4 * i + 2] = v.z;
        R[4 * i + 3] = v.w;
    }
}

// q+ (sign 0) or q- (sign 1) fragments (B operand, 8 heads) in the same permuted word order.
template <int NT>
__device__ __forceinline__ void load_q_signed(const QuestArgs& a, int b, int kvh, bool neg, uint32_t (&qf)[NT][16]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const __nv_bfloat162 zero = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + g;
        const bool ok = hh < a.G;
        const uint4* qp = reinterpret_cast<const uint4*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + (ok ? hh : 0)) * kHeadDim);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = ok ? __ldg(qp + c + 4 * i) : make_uint4(0, 0, 0, 0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&w[t]);
                x = neg ? __hmin2(x, zero) : __hmax2(x, zero);
                qf[nt][4 * i + t] = *reinterpret_cast<uint32_t*>(&x);
            }
        }
    }
}

constexpr int kQuestTilesPerWarp = 8;   // 16-page tiles a warp scores, with the next tile's loads in flight

// Box fragments of tile j0 (pages j0 + g and j0 + g + 8; pages past the request read page 0's box).
__device__ __forceinline__ void load_box_tile(const QuestArgs& a, int b, int kvh, int np, int j0, uint32_t (&Rmx)[2][16],
                                              uint32_t (&Rmn)[2][16]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int j = j0 + g + 8 * half;
        int page = j < np ? a.page_table[(long)b * a.max_pages + j] : 0;
        if (page < 0 || page >= a.num_pages) page = 0;   // reported by the summarize kernel
        const __nv_bfloat16* box = a.boxes + ((long)page * a.Hkv + kvh) * 2 * kHeadDim;
        load_row_frags(box + kHeadDim, c, Rmx[half]);
        load_row_frags(box, c, Rmn[half]);
    }
}

// One warp per (request, kv head, kQuestTilesPerWarp consecutive 16-page tiles).
template <int NT>
__global__ void __launch_bounds__(256) quest_score_kernel(QuestArgs a, long units) {
    pdl_enter();
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const long u = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (u >= units) return;
    const int chunks = (a.max_pages + 16 * kQuestTilesPerWarp - 1) / (16 * kQuestTilesPerWarp);
    const int chunk = (int)(u % chunks);
    const long grp = u / chunks;
    const int b = (int)(grp / a.Hkv), kvh = (int)(grp % a.Hkv);
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int np = (n + kPageSize - 1) / kPageSize;
    const int jbeg = chunk * 16 * kQuestTilesPerWarp, jend = min(np, jbeg + 16 * kQuestTilesPerWarp);
    if (jbeg >= jend) return;
    uint32_t qp[NT][16], qn[NT][16];
    load_q_signed<NT>(a, b, kvh, false, qp);
    load_q_signed<NT>(a, b, kvh, true, qn);
    uint32_t Rmx[2][16], Rmn[2][16];
    load_box_tile(a, b, kvh, np, jbeg, Rmx, Rmn);
    for (int j0 = jbeg; j0 < jend; j0 += 16) {
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[nt], Rmx[0][2 * s], Rmx[1][2 * s], Rmx[0][2 * s + 1], Rmx[1][2 * s + 1],
                               qp[nt][2 * s], qp[nt][2 * s + 1]);
                mma_bf16_16816(acc[nt], Rmn[0][2 * s], Rmn[1][2 * s], Rmn[0][2 * s + 1], Rmn[1][2 * s + 1],
                               qn[nt][2 * s], qn[nt][2 * s + 1]);
            }
        // the next tile's loads go out before this tile's results are written
        if (j0 + 16 < jend) load_box_tile(a, b, kvh, np, j0 + 16, Rmx, Rmn);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + 2 * c + e;
                if (col >= a.G) continue;
                float* rrow = a.rel + ((long)b * a.Hq + (long)kvh * a.G + col) * a.max_pages;
                if (j0 + g < np) rrow[j0 + g] = acc[nt][e];
                if (j0 + g + 8 < np) rrow[j0 + g + 8] = acc[nt][2 + e];
            }
    }
}

// ---------------------------------------------------------------------------------------------
// select: one CTA per (b, h)
// ---------------------------------------------------------------------------------------------
constexpr int kQuestSelectThreads = 512;
constexpr int kQuestLoads = 16;   // relevance loads in flight per thread (8192 pages per round)

// Keys of the pages 0 .. n - 1 in shared memory; an element's position is its page index.
struct PageKeys {
    const uint32_t* k;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int j) const { return k[j]; }
    __device__ __forceinline__ int pos(int j) const { return j; }
};

size_t quest_select_smem(const QuestArgs& a) {
    return sizeof(int) * (4096 + 40 + 8) + (size_t)a.max_pages * 8;
}

__global__ void __launch_bounds__(kQuestSelectThreads) quest_select_kernel(QuestArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    int* hist = reinterpret_cast<int*>(smem);                   // [4096]
    int* scratch = hist + 4096;                                  // [40]
    int* s_sel = scratch + 40;                                   // [8]
    uint32_t* lkey = reinterpret_cast<uint32_t*>(s_sel + 8);     // [max_pages]: relevance keys
    int* kept = reinterpret_cast<int*>(lkey + a.max_pages);      // [max_pages]: kept pages, ascending
    pdl_enter();
    const int tid = threadIdx.x, nthr = blockDim.x;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hq);
    int32_t* row = a.idx + bh * a.k_max;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int kb = a.k[b];
    const int np = (n + kPageSize - 1) / kPageSize;
    const int kp = min(np, (int)(((long)kb + kPageSize - 1) / kPageSize));
    if (kb < 1 || (long)kp * kPageSize > a.k_max && kp < np) {
        if (tid == 0) report(a.status, SD_ERR_INVALID_ARG);
        for (int i = tid; i < a.k_max; i += nthr) row[i] = -1;
        return;
    }
    if (kp >= np) {   // every page is kept (includes N_b == 0)
        if (n > a.k_max) {
            if (tid == 0) report(a.status, SD_ERR_INVALID_ARG);
            for (int i = tid; i < a.k_max; i += nthr) row[i] = -1;
            return;
        }
        for (int i = tid; i < a.k_max; i += nthr) row[i] = (i < n) ? i : -1;
        return;
    }
    // the kp - 1 most relevant pages among 0 .. np - 2 (np - 1, the current page, is always kept):
    // their keys, kQuestLoads relevance loads in flight per thread, and the keys' range
    const float* rrow = a.rel + bh * a.max_pages;
    reset_key_range(s_sel);
    __syncthreads();
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j0 = tid; j0 < np - 1; j0 += kQuestLoads * nthr) {
        float v[kQuestLoads];
#pragma unroll
        for (int u = 0; u < kQuestLoads; ++u) {
            const int j = j0 + u * nthr;
            v[u] = j < np - 1 ? __ldcg(rrow + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kQuestLoads; ++u) {
            const int j = j0 + u * nthr;
            if (j < np - 1) {
                const uint32_t key = float_key(v[u]);
                lkey[j] = key;
                kmin = min(kmin, key);
                kmax = max(kmax, key);
            }
        }
    }
    add_key_range(s_sel, kmin, kmax);
    __syncthreads();
    if (kp > 1) select_exact(PageKeys{lkey, np - 1}, kp - 1, kept, hist, scratch, s_sel, true);
    __syncthreads();
    // positions of the kept pages, ascending: kp - 1 full pages, then the (possibly partial) current page
    for (int i = tid; i < a.k_max; i += nthr) {
        const int r = i / kPageSize, s = i - r * kPageSize;
        int pos = -1;
        if (r < kp) {
            const int j = r < kp - 1 ? kept[r] : np - 1;
            const int p = j * kPageSize + s;
            pos = p < n ? p : -1;
        }
        row[i] = pos;
    }
}

// ---------------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------------
cudaError_t launch_quest_summarize(const QuestArgs& a, cudaStream_t stream) {
    const long units = (long)a.B * (a.last_only ? 1 : a.max_pages) * a.Hkv;
    const long grid = (units + 7) / 8;
    cudaError_t e = launch_pdl(quest_summarize_kernel, dim3((unsigned)grid), dim3(256), 0, stream, a, units);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quest_score(const QuestArgs& a, cudaStream_t stream) {
    const long units = (long)a.B * a.Hkv * ((a.max_pages + 16 * kQuestTilesPerWarp - 1) / (16 * kQuestTilesPerWarp));
    const long grid = (units + 7) / 8;
    cudaError_t e = a.G <= 8 ? launch_pdl(quest_score_kernel<1>, dim3((unsigned)grid), dim3(256), 0, stream, a, units)
                             : launch_pdl(quest_score_kernel<2>, dim3((unsigned)grid), dim3(256), 0, stream, a, units);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quest_select(const QuestArgs& a, cudaStream_t stream) {
    const size_t smem = quest_select_smem(a);
    cudaError_t e = cudaFuncSetAttribute(quest_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(quest_select_kernel, dim3(a.B * a.Hq), dim3(kQuestSelectThreads), smem, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
