// topk_select.cu -- selection step of the exact top-k indexer ("Oracle Top-K", gist.science
// summary sec. 2): per (request, query head), the k highest scores of the row the score pass wrote,
// ties at the k-th score going to the lower position, emitted as ascending positions.
//
// select_kernel, one CTA per (b, h): a strided sample of the scores places a candidate threshold;
// one pass over the row compacts every key at or above it, in position order, into shared memory;
// an exact radix select over order-preserving 32-bit keys (12 + 12 + 8 bits) finds the k-th key
// there, and an ordered compaction writes the ascending positions.  If the sample misplaced the
// threshold, the exact select runs over the whole row in global memory instead.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kSelectThreads = 512;
constexpr int kSelectItems = 4;   // consecutive elements per thread per tile of the exact emit

// ---------------------------------------------------------------------------------------------
// select
// ---------------------------------------------------------------------------------------------
struct GlobalKeys {   // the fp32 scores of one (b, h), read from the workspace
    const float* sc;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int j) const { return float_key(sc[j]); }
    __device__ __forceinline__ int pos(int j) const { return j; }
};
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

// Exact radix select: the key T of the target-th largest element of src (12 + 12 + 8 bit digits)
// and the number of elements with a key greater than T.
template <class Src>
__device__ void radix_find(const Src& src, int target, int* hist, int* scratch, int* s_sel, uint32_t* T_out,
                           int* greater_out) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int n = src.size();
    uint32_t prefix = 0;
    int greater = 0;
    // digits: key bits 31..20, then 19..8, then 7..0
    const int shifts[3] = {20, 8, 0};
    const int widths[3] = {12, 12, 8};
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        const int nb = 1 << widths[d];
        for (int i = tid; i < nb; i += nthr) hist[i] = 0;
        __syncthreads();
        const int hs = shifts[d] + widths[d];   // bits above this digit must equal the prefix
        for (int j = tid; j < n; j += nthr) {
            const uint32_t key = src.key(j);
            if (hs >= 32 || (key >> hs) == prefix) atomicAdd(&hist[(key >> shifts[d]) & (uint32_t)(nb - 1)], 1);
        }
        __syncthreads();
        select_bin(hist, nb, target - greater, scratch, s_sel);
        prefix = (prefix << widths[d]) | (uint32_t)s_sel[0];
        greater += s_sel[1];
        __syncthreads();
    }
    *T_out = prefix;
    *greater_out = greater;
}

// Writes the selected positions of src in ascending order to row[0..take): keys above T, plus the
// first `quota` keys equal to T (ties go to the lower position).
template <class Src>
__device__ void emit_selected(const Src& src, uint32_t T, int quota, int take, int32_t* row, int* scratch) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int n = src.size();
    int out_base = 0, eq_base = 0;
    for (int j0 = 0; j0 < n; j0 += nthr * kSelectItems) {
        const int j = j0 + tid * kSelectItems;
        uint32_t key[kSelectItems];
        int eqc = 0;
#pragma unroll
        for (int e = 0; e < kSelectItems; ++e) {
            key[e] = (j + e < n) ? src.key(j + e) : 0u;
            eqc += (j + e < n && key[e] == T);
        }
        int eq_tot;
        int eq_rank = eq_base + block_exclusive_scan(eqc, scratch, &eq_tot);
        bool keep[kSelectItems];
        int kc = 0;
#pragma unroll
        for (int e = 0; e < kSelectItems; ++e) {
            const bool valid = j + e < n;
            const bool eq = valid && key[e] == T;
            keep[e] = valid && (key[e] > T || (eq && eq_rank < quota));
            eq_rank += eq;
            kc += keep[e];
        }
        int k_tot;
        int w = out_base + block_exclusive_scan(kc, scratch, &k_tot);
#pragma unroll
        for (int e = 0; e < kSelectItems; ++e)
            if (keep[e]) {
                if (w < take) row[w] = src.pos(j + e);
                ++w;
            }
        out_base += k_tot;
        eq_base += eq_tot;
    }
}

template <class Src>
__device__ void select_exact(const Src& src, int take, int32_t* row, int* hist, int* scratch, int* s_sel) {
    uint32_t T;
    int greater;
    radix_find(src, take, hist, scratch, s_sel, &T, &greater);
    emit_selected(src, T, take - greater, take, row, scratch);
}

constexpr int kSample = 2048;   // strided sample of the scores used to place the candidate threshold

__global__ void __launch_bounds__(kSelectThreads) select_kernel(TopkArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int* hist = reinterpret_cast<int*>(smem);   // [4096]
    int* scratch = hist + 4096;                  // [40]
    int* s_sel = scratch + 40;                   // [8]
    int* s_cnt = s_sel + 8;                      // [2][32] per-warp counts, double buffered
    pdl_enter();
    uint32_t* lkey = reinterpret_cast<uint32_t*>(s_cnt + 64);
    int* lpos = reinterpret_cast<int*>(lkey + a.cap);

    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
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
    const float* sc = a.scores + bh * a.n_cap;

    // Candidate threshold tau: the j-th largest key of a strided sample, j chosen so that the keys
    // >= tau are expected to number about 1.25 take + 16 sample strides (many standard deviations
    // above take, well below the shared-memory capacity).  Small rows take every key.
    uint32_t tau = 0u;
    if (n > a.cap) {
        const int stride = n / kSample;
        uint32_t* skey = lkey;   // the sample lives in the candidate buffer until the pass below
        for (int i = tid; i < kSample; i += nthr) skey[i] = float_key(sc[(long)i * stride]);
        __syncthreads();
        const long want = ((long)take * kSample + n - 1) / n;
        const int j = (int)min((long)kSample, want + want / 4 + 16);
        int greater;
        radix_find(SharedKeys{skey, nullptr, kSample}, j, hist, scratch, s_sel, &tau, &greater);
    }

    // One pass: ordered compaction of every key >= tau into shared memory.  A tile is nthr * 16
    // consecutive keys; thread t owns 16 consecutive keys of it (four 16-byte loads in flight).
    constexpr int kPerThread = 16;
    int base = 0;
    int buf = 0;
    for (int i0 = 0; i0 < n; i0 += nthr * kPerThread) {
        const int i = i0 + tid * kPerThread;
        uint32_t key[kPerThread];
        if (i + kPerThread <= n) {
            float4 v[kPerThread / 4];
#pragma unroll
            for (int u = 0; u < kPerThread / 4; ++u) v[u] = *reinterpret_cast<const float4*>(sc + i + 4 * u);
#pragma unroll
            for (int u = 0; u < kPerThread / 4; ++u) {
                key[4 * u + 0] = float_key(v[u].x);
                key[4 * u + 1] = float_key(v[u].y);
                key[4 * u + 2] = float_key(v[u].z);
                key[4 * u + 3] = float_key(v[u].w);
            }
        } else {
#pragma unroll
            for (int e = 0; e < kPerThread; ++e) key[e] = (i + e < n) ? float_key(sc[i + e]) : 0u;
        }
        int cnt = 0;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) cnt += (i + e < n) && key[e] >= tau;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) s_cnt[buf * 32 + warp] = incl;
        __syncthreads();
        const int wc = (lane < nwarps) ? s_cnt[buf * 32 + lane] : 0;
        int wincl = wc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wincl, o);
            if (lane >= o) wincl += t;
        }
        const int wbase = __shfl_sync(0xffffffffu, wincl - wc, warp);
        const int tile_tot = __shfl_sync(0xffffffffu, wincl, 31);
        if (cnt > 0) {
            int w = base + wbase + incl - cnt;
#pragma unroll
            for (int e = 0; e < kPerThread; ++e)
                if ((i + e < n) && key[e] >= tau) {
                    if (w < a.cap) {
                        lkey[w] = key[e];
                        lpos[w] = i + e;
                    }
                    ++w;
                }
        }
        base += tile_tot;
        buf ^= 1;
    }
    __syncthreads();
    if (base >= take && base <= a.cap) {
        select_exact(SharedKeys{lkey, lpos, base}, take, row, hist, scratch, s_sel);
    } else {
        // the sample misplaced tau (too few or too many candidates): exact select on the full row
        select_exact(GlobalKeys{sc, n}, take, row, hist, scratch, s_sel);
    }
    for (int i = take + tid; i < a.k_max; i += nthr) row[i] = -1;
}

// ---------------------------------------------------------------------------------------------
// host launcher
// ---------------------------------------------------------------------------------------------
size_t select_smem(const TopkArgs& a) { return sizeof(int) * (4096 + 40 + 8 + 64) + (size_t)a.cap * 8; }

cudaError_t launch_select(const TopkArgs& a, cudaStream_t stream) {
    const size_t smem = select_smem(a);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(select_kernel, dim3(a.B * a.Hq), dim3(kSelectThreads), smem, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
