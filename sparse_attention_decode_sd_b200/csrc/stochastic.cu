// stochastic.cu -- the sampled half of stochastic index selection (the vAttention-style selection
// of "Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2 "Stochastische
// Indexierung" and sec. 3A).  The pages name the method, not its estimator; the reading here: per
// (request, query head) row, the exact top-k_det rows S_d (written by the exact indexer) plus
// m = min(k_samp, |R|) rows drawn uniformly without replacement from the rest R = [0, N_b) \ S_d,
// each drawn row standing for |R| / m rows of R.  The draw is reproducible from (seed, step): row r
// = b * Hq + h gives position p the key u(p) = top 32 bits of SM(SM(SM(seed + step) + r) + p), where
// SM(x) is one output of the SplitMix64 generator from state x (Steele, Lea and Flood, "Fast
// splittable pseudorandom number generators", 2014), and the drawn rows are the m positions of R
// with the smallest (u, p).
//
// sample_kernel   one CTA per row: marks S_d in a shared-memory bitmap, keeps the positions of R
//                 whose key falls below a threshold set for about m + 6 sqrt(m) + 32 of them (moved
//                 by bisection if fewer than m or more than fit survive), selects the m smallest
//                 keys exactly (radix select on the complemented keys, ties to the lower position)
//                 and rewrites the row as S_d and the drawn rows together in ascending position,
//                 the drawn ones carrying kSampledFlag (bit 30).
#include "common.cuh"
#include "kernels.h"
#include "radix_select.cuh"

namespace sd {

// One SplitMix64 output from state x: the state advances by the golden-ratio increment, then is
// mixed by two xor-shift-multiply rounds and a final xor-shift.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

constexpr int kSampleThreads = 512;
constexpr int kSampleHistBins = 4096;   // radix select digits of up to 12 bits

size_t sample_smem(const SampleArgs& a) {
    return (size_t)2 * a.words * sizeof(uint32_t) + (size_t)a.cap * (sizeof(uint32_t) + 2 * sizeof(int)) +
           (size_t)(kSampleHistBins + kMaxSelectScratch) * sizeof(int);
}

// Positions [p0, p1) of this thread: a contiguous slice of [0, n), slices in thread order.
__device__ __forceinline__ void thread_slice(int n, int* p0, int* p1) {
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    *p0 = min(n, (int)threadIdx.x * per);
    *p1 = min(n, *p0 + per);
}

__device__ __forceinline__ bool in_bitmap(const uint32_t* bits, int p) { return (bits[p >> 5] >> (p & 31)) & 1u; }

__global__ void __launch_bounds__(kSampleThreads) sample_kernel(SampleArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* det_bits = reinterpret_cast<uint32_t*>(smem);
    uint32_t* samp_bits = det_bits + a.words;
    uint32_t* ckey = samp_bits + a.words;                       // complemented keys of the candidates
    int* cpos = reinterpret_cast<int*>(ckey + a.cap);           // their positions, ascending
    int* chosen = cpos + a.cap;                                  // the drawn positions, ascending
    int* hist = chosen + a.cap;
    int* scratch = hist + kSampleHistBins;                       // block scan (33) + selection state (4)
    int* s_sel = scratch + 36;
    pdl_enter();

    const int tid = threadIdx.x;
    const int r = blockIdx.x;
    const int b = r / a.Hq;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int kd = a.k_det[b], ks = a.k_samp[b];
    if (kd < 1 || ks < 0) {   // k_det < 1 is also reported by the exact selection
        if (tid == 0) report(a.status, SD_ERR_INVALID_ARG);
        return;
    }
    int32_t* row = a.idx + (long)r * a.k_max;
    const int ndet = min(kd, n);   // the exact selection wrote min(k_det, N_b) rows
    const int rest = n - ndet;
    const int m = min(ks, rest);
    if (m <= 0) return;
    if (ndet + m > a.k_max) {
        if (tid == 0) report(a.status, SD_ERR_INVALID_ARG);
        return;
    }
    const int nw = (n + 31) >> 5;
    for (int i = tid; i < nw; i += blockDim.x) det_bits[i] = samp_bits[i] = 0u;
    __syncthreads();
    for (int j = tid; j < ndet; j += blockDim.x) {
        const int p = row[j];
        if (p >= 0 && p < n) atomicOr(&det_bits[p >> 5], 1u << (p & 31));
    }
    __syncthreads();

    const uint64_t c1 = splitmix64(splitmix64(a.seed + (uint64_t)a.step) + (uint64_t)r);
    int p0, p1;
    thread_slice(n, &p0, &p1);
    // threshold on the 32-bit keys (2^32: every position of R), moved by bisection until between m
    // and cap positions of R fall below it
    uint64_t lo = 0, hi = 1ull << 32;
    const double expect = (double)m + 6.0 * sqrt((double)m) + 32.0;
    uint64_t tau = expect >= (double)rest ? hi : (uint64_t)(expect / (double)rest * 4294967296.0) + 1;
    int total = 0, before = 0;
    for (int it = 0; it < 70; ++it) {
        int cnt = 0;
        for (int p = p0; p < p1; ++p)
            if (!in_bitmap(det_bits, p) && (splitmix64(c1 + (uint64_t)p) >> 32) < tau) ++cnt;
        before = block_exclusive_scan(cnt, scratch, &total);
        if (total < m) {
            lo = tau;
            tau = (tau >= hi / 2) ? hi : max(tau * 2, tau + 1);
            if (lo >= hi) break;
        } else if (total > a.cap) {
            hi = tau;
            tau = lo + (hi - lo) / 2;
            if (tau <= lo) break;
        } else {
            break;
        }
    }
    if (total < m || total > a.cap) {   // not reached for keys that are not massively tied
        if (tid == 0) report(a.status, SD_ERR_UNSUPPORTED);
        return;
    }
    {
        int w = before;
        for (int p = p0; p < p1; ++p) {
            if (in_bitmap(det_bits, p)) continue;
            const uint32_t key = (uint32_t)(splitmix64(c1 + (uint64_t)p) >> 32);
            if ((uint64_t)key < tau) {
                ckey[w] = ~key;   // the largest complemented keys are the smallest keys
                cpos[w] = p;
                ++w;
            }
        }
    }
    __syncthreads();
    const SharedKeys src{ckey, cpos, total};
    select_exact(src, m, chosen, hist, scratch, s_sel);
    __syncthreads();
    for (int j = tid; j < m; j += blockDim.x) {
        const int p = chosen[j];
        atomicOr(&samp_bits[p >> 5], 1u << (p & 31));
    }
    __syncthreads();
    // the row: S_d and the drawn rows in ascending position, drawn ones flagged
    const int wpt = (nw + (int)blockDim.x - 1) / (int)blockDim.x;
    const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
    int cnt = 0;
    for (int i = w0; i < w1; ++i) cnt += __popc(det_bits[i] | samp_bits[i]);
    int tot;
    int o = block_exclusive_scan(cnt, scratch, &tot);
    for (int i = w0; i < w1; ++i) {
        uint32_t bits = det_bits[i] | samp_bits[i];
        while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1;
            const int p = (i << 5) + bit;
            if (o < a.k_max) row[o] = ((samp_bits[i] >> bit) & 1u) ? (p | (int)kSampledFlag) : p;
            ++o;
        }
    }
}

cudaError_t launch_sample(const SampleArgs& a, cudaStream_t stream) {
    const size_t smem = sample_smem(a);
    cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(sample_kernel, dim3((unsigned)((long)a.B * a.Hq)), dim3(kSampleThreads), smem, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
