// topk_select.cu -- selection step of the exact top-k indexer ("Oracle Top-K", gist.science
// summary sec. 2): per (request, query head), the k highest scores of the row the score pass wrote,
// ties at the k-th score going to the lower position, emitted as ascending positions.
//
// select_kernel, one CTA per (b, h), reads the row's candidates as the score pass left them (a
// 16-bit mask per page and head, scores in the score-pass warps' streams).  If the threshold
// admitted fewer than k candidates (rare), it selects from scores recomputed on the fly.  Usual case: the
// candidates are compacted in position order into shared memory, where an exact radix select over
// order-preserving 32-bit keys (12 + 12 + 8 bits) finds the k-th key and an ordered compaction
// writes the ascending positions.  If they do not fit, the same select runs on the masked row in
// global memory (L2), with block scans putting the output in order.
#include "common.cuh"
#include "kernels.h"
#include "radix_select.cuh"

namespace sd {

constexpr int kSelectThreads = 512;


// The candidates of row (b, h) as the score pass left them: per page p, the record
// rec[p] = {start, mask}, mask bit i marking position p*16 + i as a candidate, whose scores sit in
// position order from cand[start] on.  The row's pages are taken in chunks of 16 * blockDim.x: in a
// chunk, warp w owns 512 consecutive pages, read in 8 rounds of 64 with lane l holding pages
// 2l and 2l + 1 of the round (one 16-byte load, coalesced across the warp).  Position order is
// (warp, round, lane, record), which warp scans per round and a block scan over warps reproduce.
constexpr int kRecsPerThread = 16;
constexpr int kRounds = kRecsPerThread / 2;
struct StreamRow {
    const float* cand;
    const uint2* rec;
    uint32_t limit;   // floats in the stream buffer: a record pointing past it is skipped (it can only
                      // come from a score pass that stopped early, which reported that)
    int np;           // pages of the row
    __device__ StreamRow(const TopkArgs& a, long bh, int n) {
        cand = a.cand;
        rec = a.prec + bh * a.mstride;
        limit = (uint32_t)((long)a.B * a.Hq * a.n_cap);
        np = (n + kPageSize - 1) / kPageSize;
    }
    __device__ __forceinline__ int chunks() const {
        const int cp = kRecsPerThread * (int)blockDim.x;
        return (np + cp - 1) / cp;
    }
    // first page of this lane's pair in round i of chunk ci
    __device__ __forceinline__ int page_of(int ci, int i) const {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        return ci * kRecsPerThread * (int)blockDim.x + warp * 32 * kRecsPerThread + i * 64 + 2 * lane;
    }
    // This lane's records of chunk ci, all loads in flight together (pages past the row read as empty).
    __device__ __forceinline__ void load(int ci, uint2 (&r)[kRecsPerThread]) const {
        uint4 v[kRounds];
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            // the page index is even, and a row holds mstride >= np records with mstride a multiple of
            // 8, so the pair lies in the row whenever its first page does; past the row read pair 0
            const int p = page_of(ci, i);
            v[i] = __ldg(reinterpret_cast<const uint4*>(rec + (p < np ? p : 0)));
        }
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int p = page_of(ci, i);
            r[2 * i] = p < np ? make_uint2(v[i].x, v[i].y) : make_uint2(0u, 0u);
            r[2 * i + 1] = p + 1 < np ? make_uint2(v[i].z, v[i].w) : make_uint2(0u, 0u);
        }
    }
    // Writes the candidates of records r (this lane's pages of chunk ci) in position order, the warp
    // starting at slot `wbase`: the position to pos[] and the candidate's index in the stream buffer to
    // idx[] (0xffffffff for a record that points past the buffer).  Every lane of the warp must call.
    __device__ __forceinline__ void stage(int ci, const uint2 (&r)[kRecsPerThread], int wbase, uint32_t* idx,
                                          int* pos) const {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int c = __popc(r[2 * i].y) + __popc(r[2 * i + 1].y);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int off = wbase + incl - c;
            wbase += __shfl_sync(0xffffffffu, incl, 31);
            const int p = page_of(ci, i);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t mm = r[2 * i + h].y;
                const uint32_t start = r[2 * i + h].x;
                const bool inside = (unsigned long)start + __popc(mm) <= limit;
                for (uint32_t k = 0; mm; ++k) {
                    const int bit = __ffs(mm) - 1;
                    mm &= mm - 1u;
                    idx[off] = inside ? start + k : 0xffffffffu;
                    pos[off] = (p + h) * kPageSize + bit;
                    ++off;
                }
            }
        }
    }
    // Candidates of a thread-contiguous partition of the row (thread t: pages [t*per, (t+1)*per)), in
    // position order, so that block scans over per-thread counts order the row -- for the passes that
    // read the candidates from global memory.
    template <class F>
    __device__ __forceinline__ void for_each(F f) const {
        const int per = (np + (int)blockDim.x - 1) / (int)blockDim.x;
        const int p0 = min(np, (int)threadIdx.x * per), p1 = min(np, p0 + per);
        for (int p = p0; p < p1; ++p) {
            uint32_t m = rec[p].y;
            if (m == 0u) continue;
            const uint32_t base = rec[p].x;
            if ((unsigned long)base + __popc(m) > limit) continue;
            const float* sp = cand + base;
            for (int k = 0; m; ++k) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                f(float_key(sp[k]), p * kPageSize + bit);
            }
        }
    }
};

// Rare fallback, when the threshold admitted fewer candidates than k: every score of row (b, h)
// recomputed on the fly from q and K in each pass (a fixed order of fp32 operations, so every pass
// sees the same values).  Thread t owns the positions [t*per, (t+1)*per).  q (fp32, in shared memory
// at qs) and the inputs are the ones the score pass recorded in the workspace.
struct RecomputedRow {
    const __nv_bfloat16* K;
    const int32_t* ptrow;
    const float* qs;
    int Hkv, kvh, num_pages;
    int i0, i1;
    __device__ RecomputedRow(const TopkArgs& a, long bh, int n, const float* q_smem) {
        const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
        K = static_cast<const __nv_bfloat16*>(a.inputs[1]);
        ptrow = static_cast<const int32_t*>(a.inputs[2]) + (long)b * a.max_pages;
        qs = q_smem;
        Hkv = a.Hkv;
        kvh = h / a.G;
        num_pages = a.num_pages;
        const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
        i0 = min(n, (int)threadIdx.x * per);
        i1 = min(n, i0 + per);
    }
    template <class F>
    __device__ __forceinline__ void for_each(F f) const {
        for (int i = i0; i < i1; ++i) {
            int page = __ldg(ptrow + i / kPageSize);
            if (page < 0 || page >= num_pages) page = 0;   // reported by the score pass
            const uint4* row =
                reinterpret_cast<const uint4*>(K + (((long)page * kPageSize + (i % kPageSize)) * Hkv + kvh) * kHeadDim);
            float d = 0.f;
#pragma unroll 4
            for (int ch = 0; ch < kHeadDim / 8; ++ch) {
                const uint4 v = __ldg(row + ch);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    d = fmaf(bf16_hi(w[t]), qs[ch * 8 + 2 * t + 1], fmaf(bf16_lo(w[t]), qs[ch * 8 + 2 * t], d));
            }
            f(float_key(d), i);
        }
    }
};

// Selection straight from a source visited with for_each in thread-ordered position order (any
// number of candidates): radix select, then the ascending positions through two block scans (ties
// first, then the selected).
// (Not inlined: these paths are rare, and their registers stay out of the usual path's budget.)
template <class Src>
__device__ __noinline__ void select_masked(const Src& src, int take, int32_t* row, int* hist, int* scratch,
                                          int* s_sel) {
    uint32_t T;
    int greater;
    radix_select([&](auto f) { src.for_each([&](uint32_t key, int) { f(key); }); }, take, hist, scratch, s_sel, &T,
                 &greater);
    const int quota = take - greater;
    int tc = 0;
    src.for_each([&](uint32_t key, int) { tc += key == T; });
    int ttot;
    const int tie_before = block_exclusive_scan(tc, scratch, &ttot);
    int sc = 0;
    {
        int tb = tie_before;
        src.for_each([&](uint32_t key, int) {
            if (key > T) ++sc;
            else if (key == T) sc += (tb++ < quota);
        });
    }
    int stot;
    int out = block_exclusive_scan(sc, scratch, &stot);
    int tb = tie_before;
    src.for_each([&](uint32_t key, int pos) {
        const bool keep = key > T || (key == T && tb++ < quota);
        if (keep) {
            if (out < take) row[out] = pos;
            ++out;
        }
    });
}

__global__ void __launch_bounds__(kSelectThreads, 2) select_kernel(TopkArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int* hist = reinterpret_cast<int*>(smem);   // [4096]
    int* scratch = hist + 4096;                  // [40]
    int* s_sel = scratch + 40;                   // [8]
    uint32_t* lkey = reinterpret_cast<uint32_t*>(s_sel + 8);   // [cap]
    int* lpos = reinterpret_cast<int*>(lkey + a.cap);           // [cap]
    pdl_enter();

    const int tid = threadIdx.x, nthr = blockDim.x;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hq);
    int32_t* row = a.idx + bh * a.k_max;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int kb = a.k[b];
    const int take = min(kb, n);
    if (kb < 1 || take > a.k_max) {
        if (tid == 0) report(a.status, SD_ERR_INVALID_ARG);
        for (int i = tid; i < a.k_max; i += nthr) row[i] = -1;
        return;
    }
    if (take == n) {   // everything is selected (includes N_b == 0)
        for (int i = tid; i < a.k_max; i += nthr) row[i] = (i < n) ? i : -1;
        return;
    }
    StreamRow src(a, bh, n);
    // Candidates chunk by chunk (one chunk up to 131072 positions): counted, and staged into shared
    // memory in position order -- positions and stream indices -- while they fit.
    int total = 0;
    for (int ci = 0; ci < src.chunks(); ++ci) {
        int cnt;
        {
            uint2 r[kRecsPerThread];
            src.load(ci, r);
            cnt = 0;
#pragma unroll
            for (int i = 0; i < kRecsPerThread; ++i) cnt += __popc(r[i].y);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);   // the warp's count
        int ctot;
        const int wb = block_exclusive_scan((tid & 31) == 0 ? cnt : 0, scratch, &ctot);
        const int wbase = total + __shfl_sync(0xffffffffu, wb, 0);   // candidates of the earlier warps
        if (total + ctot <= a.cap) {
            uint2 r[kRecsPerThread];
            src.load(ci, r);   // again, from L1: cheaper than keeping 32 registers across the scan
            src.stage(ci, r, wbase, lkey, lpos);
        }
        total += ctot;
    }
    if (total < take) {
        // the threshold admitted fewer candidates than k: select from scores recomputed on the fly
        float* qs = reinterpret_cast<float*>(lkey);
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.inputs[0]) + bh * kHeadDim;
        for (int i = tid; i < kHeadDim; i += nthr) qs[i] = __bfloat162float(q[i]);
        __syncthreads();
        select_masked(RecomputedRow(a, bh, n, qs), take, row, hist, scratch, s_sel);
    } else if (total <= a.cap) {
        // the usual case: every thread gathers scores for the staged stream indices, four loads in flight
        __syncthreads();
        for (int j0 = tid; j0 < total; j0 += 4 * nthr) {
            uint32_t ix[4];
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * nthr;
                ix[u] = j < total ? lkey[j] : 0xffffffffu;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = ix[u] < src.limit ? __ldg(a.cand + ix[u]) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * nthr;
                if (j < total) lkey[j] = ix[u] < src.limit ? float_key(v[u]) : 0u;
            }
        }
        __syncthreads();
        select_exact(SharedKeys{lkey, lpos, total}, take, row, hist, scratch, s_sel);
    } else {
        select_masked(src, take, row, hist, scratch, s_sel);
    }
    for (int i = take + tid; i < a.k_max; i += nthr) row[i] = -1;
    // The row's records are dead now: their L2 lines are dropped without being written back (only
    // lines that lie wholly inside this row's records), so that they cost no DRAM write bandwidth
    // in the kernels that follow.  The next score pass rewrites every record it reads.
    __syncthreads();
    {
        const uintptr_t lo = reinterpret_cast<uintptr_t>(src.rec), hi = lo + (uintptr_t)src.np * sizeof(uint2);
        const uintptr_t first = (lo + 127) & ~(uintptr_t)127, end = hi & ~(uintptr_t)127;
        for (uintptr_t ad = first + (uintptr_t)tid * 128; ad < end; ad += (uintptr_t)nthr * 128)
            asm volatile("discard.global.L2 [%0], 128;" ::"l"(ad) : "memory");
    }
}

// ---------------------------------------------------------------------------------------------
// host launcher
// ---------------------------------------------------------------------------------------------
size_t select_smem(const TopkArgs& a) { return sizeof(int) * (4096 + 40 + 8) + (size_t)a.cap * 8; }

cudaError_t launch_select(const TopkArgs& a, cudaStream_t stream) {
    const size_t smem = select_smem(a);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(select_kernel, dim3(a.B * a.Hq), dim3(kSelectThreads), smem, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
