// radix_select.cuh -- exact block-wide selection of the k largest order-preserving 32-bit keys
// (the selection step of exact top-k: "Technische Zusammenfassung: Kontextsparsitaet bei der
// Inferenzzeit", sec. 2, Oracle Top-K), shared by the token-level select kernel and the Quest page
// select kernel.  Ties at the k-th key go to the lower position; the output is ascending.
#pragma once

#include "common.cuh"

namespace sd {

struct SharedKeys {   // (key, position) list in shared memory, ascending positions
    const uint32_t* k;
    const int* p;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int j) const { return k[j]; }
    __device__ __forceinline__ int pos(int j) const { return p[j]; }
};

// Finds the bin t holding the target-th largest element (1 <= target <= total, counted from the top
// bin) and the number of elements in bins above t.  Every thread must call; results in s_out[0..1].
__device__ __forceinline__ void select_bin(const int* hist, int nbins, int target, int* scratch, int* s_out) {
    const int tid = threadIdx.x;
    const int bpt = max(1, nbins / (int)blockDim.x);
    const int hi = nbins - tid * bpt;   // this thread covers bins [hi - bpt, hi), top first
    if (tid == 0) {                     // defined result even if no bin qualifies
        s_out[0] = 0;
        s_out[1] = 0;
    }
    int s = 0;
    if (hi > 0)
        for (int i = 1; i <= bpt; ++i) s += hist[hi - i];
    int tot;
    const int ex = block_exclusive_scan(s, scratch, &tot);
    if (hi > 0 && ex < target && ex + s >= target) {
        int cum = ex;
        for (int i = 1; i <= bpt; ++i) {
            const int bin = hi - i;
            if (cum + hist[bin] >= target) {
                s_out[0] = bin;
                s_out[1] = cum;
                break;
            }
            cum += hist[bin];
        }
    }
    __syncthreads();
}

// Exact radix select over the keys a thread visits with visit(f) (f(key) per element): the key T
// of the target-th largest element (1 <= target <= count) and the number of elements with a key
// greater than T.  The keys' range is found first and the digits (up to 12 bits each) start at the
// highest bit in which the smallest and largest key differ: candidates cluster just above a
// threshold, so a fixed top digit would pile them into a few contended histogram bins.
// When the bin holding the target after a digit has at most kSmallBin elements, they are collected and
// ranked directly by one warp instead of running the next digit's histogram.
constexpr int kSmallBin = 64;

// The block's key range, for a caller that writes the keys: reset_key_range before the pass (and a
// barrier), add_key_range with each thread's (min, max) after it, then a barrier; key_range reads it.
__device__ __forceinline__ void reset_key_range(int* s_sel) {
    if (threadIdx.x == 0) {
        reinterpret_cast<unsigned int*>(s_sel)[2] = 0xffffffffu;
        reinterpret_cast<unsigned int*>(s_sel)[3] = 0u;
    }
}
__device__ __forceinline__ void add_key_range(int* s_sel, uint32_t kmin, uint32_t kmax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMin(reinterpret_cast<unsigned int*>(s_sel) + 2, kmin);
        atomicMax(reinterpret_cast<unsigned int*>(s_sel) + 3, kmax);
    }
}

// have_range: the caller filled the key range (reset_key_range / add_key_range and a barrier).
template <class Visit>
__device__ void radix_select(Visit visit, int target, int* hist, int* scratch, int* s_sel, uint32_t* T_out,
                             int* greater_out, bool have_range = false) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31;
    unsigned int* range = reinterpret_cast<unsigned int*>(s_sel + 2);
    if (!have_range) {
        uint32_t kmin = 0xffffffffu, kmax = 0u;
        visit([&](uint32_t key) {
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        });
        reset_key_range(s_sel);
        __syncthreads();
        add_key_range(s_sel, kmin, kmax);
        __syncthreads();
    }
    uint32_t kmin = range[0];
    uint32_t kmax = range[1];
    __syncthreads();
    const uint32_t diff = kmin ^ kmax;
    int top = diff ? 31 - __clz(diff) : -1;   // highest bit that differs; above it every key is kmin's
    uint32_t prefix = top >= 31 ? 0u : (kmin >> (top + 1)) << (top + 1);
    int greater = 0;
    while (top >= 0) {
        const int w = min(12, top + 1), sh = top + 1 - w;
        const int nb = 1 << w;
        for (int i = tid; i < nb; i += nthr) hist[i] = 0;
        __syncthreads();
        visit([&](uint32_t key) {
            if (top >= 31 || (key >> (top + 1)) == (prefix >> (top + 1)))
                atomicAdd(&hist[(key >> sh) & (uint32_t)(nb - 1)], 1);
        });
        __syncthreads();
        select_bin(hist, nb, target - greater, scratch, s_sel);
        const int bin = s_sel[0];
        const int in_bin = hist[bin];
        prefix |= (uint32_t)bin << sh;
        greater += s_sel[1];
        top = sh - 1;
        __syncthreads();
        if (top >= 0 && in_bin <= kSmallBin) {
            // the few keys of the bin (their bits above `top` equal prefix's): collect and rank them
            uint32_t* list = reinterpret_cast<uint32_t*>(hist);   // [kSmallBin]
            int* count = hist + kSmallBin;
            if (tid == 0) *count = 0;
            __syncthreads();
            visit([&](uint32_t key) {
                if ((key >> (top + 1)) == (prefix >> (top + 1))) list[atomicAdd(count, 1)] = key;
            });
            __syncthreads();
            if (tid < 32) {
                const int m = *count, r = target - greater;   // r-th largest of the m keys, 1 <= r <= m
                uint32_t found = 0u;
                int above = 0;
                bool hit = false;
                for (int i = lane; i < m; i += 32) {
                    const uint32_t e = list[i];
                    int gt = 0, eq = 0;
                    for (int t = 0; t < m; ++t) {
                        gt += list[t] > e;
                        eq += list[t] == e;
                    }
                    if (gt < r && r <= gt + eq) {
                        found = e;
                        above = gt;
                        hit = true;
                    }
                }
                const uint32_t who = __ballot_sync(0xffffffffu, hit);
                const int src = who ? __ffs(who) - 1 : 0;
                found = __shfl_sync(0xffffffffu, found, src);
                above = __shfl_sync(0xffffffffu, above, src);
                if (lane == 0) {
                    s_sel[0] = (int)found;
                    s_sel[1] = above;
                }
            }
            __syncthreads();
            prefix = (uint32_t)s_sel[0];
            greater += s_sel[1];
            __syncthreads();
            break;
        }
    }
    *T_out = prefix;       // all keys equal: T is that key, none greater
    *greater_out = greater;
}

template <class Src>
__device__ __forceinline__ void radix_find(const Src& src, int target, int* hist, int* scratch, int* s_sel,
                                           uint32_t* T_out, int* greater_out, bool have_range) {
    const int n = src.size();
    radix_select(
        [&](auto f) {
            for (int j = threadIdx.x; j < n; j += blockDim.x) f(src.key(j));
        },
        target, hist, scratch, s_sel, T_out, greater_out, have_range);
}

// Writes the selected positions of src in ascending order to row[0..take): keys above T, plus the
// first `quota` keys equal to T (ties go to the lower position).  Thread t takes a contiguous segment
// of src; one block scan of its (greater, equal) counts, packed in one int, places its output.
template <class Src>
__device__ void emit_selected(const Src& src, uint32_t T, int quota, int take, int32_t* row, int* scratch) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int n = src.size();
    const int per = (n + nthr - 1) / nthr;
    const int j0 = min(n, tid * per), j1 = min(n, j0 + per);
    int gt = 0, eq = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = src.key(j);
        gt += key > T;
        eq += key == T;
    }
    int tot;
    const int before = block_exclusive_scan((eq << 16) | gt, scratch, &tot);   // counts < 2^15 each
    int eq_before = before >> 16;
    int w = (before & 0xffff) + min(eq_before, quota);
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = src.key(j);
        const bool keep = key > T || (key == T && eq_before++ < quota);
        if (keep) {
            if (w < take) row[w] = src.pos(j);
            ++w;
        }
    }
}

template <class Src>
__device__ void select_exact(const Src& src, int take, int32_t* row, int* hist, int* scratch, int* s_sel,
                             bool have_range = false) {
    uint32_t T;
    int greater;
    radix_find(src, take, hist, scratch, s_sel, &T, &greater, have_range);
    emit_selected(src, T, take - greater, take, row, scratch);
}

}  // namespace sd
