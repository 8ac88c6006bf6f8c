// topk_index.cu -- exact top-k indexer ("Oracle Top-K": exact selection of the k highest-scoring
// tokens; "Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2, and the
// indexer of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?").
//
// Two kernels:
//   score_pass_kernel   streams every K page of the requests that need selection exactly once
//                       (1-D bulk copies on the TMA engine into a shared-memory ring, one producer
//                       warp, eight consumer warps), scores 16 positions x G heads per MMA group
//                       on the tensor cores (mma.sync m16n8k16, bf16 x bf16 -> fp32) and writes
//                       fp32 scores [B][Hq][n_cap] to the workspace.  The grid is persistent and
//                       the pages of all requests are split evenly across CTAs, so ragged batches
//                       stay balanced.
//   select_kernel       one CTA per (b, h): exact radix select over order-preserving 32-bit keys
//                       (12 + 12 + 8 bits), ties at the k-th key to the lower position, then an
//                       ordered compaction that writes ascending positions.  The candidate set
//                       of the first digit normally fits in shared memory (one extra pass over
//                       the scores); otherwise the refinement streams the scores again.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kScoreConsumerWarps = 8;
constexpr int kScoreThreads = (kScoreConsumerWarps + 1) * 32;
constexpr int kSelectThreads = 512;
constexpr int kSelectItems = 4;   // consecutive elements per thread per tile

// Pages request b contributes to the score pass: every page of N_b, unless no selection is needed
// (N_b == 0 or k_b >= N_b: the select kernel then writes 0..N_b-1 directly; k_b < 1 is an error
// that the select kernel reports).
__device__ __forceinline__ int score_pages_of(const TopkArgs& a, int b) {
    const int n = a.lens[b];
    if (n <= 0 || (long)n > a.n_cap) return 0;
    const int kb = a.k[b];
    if (kb < 1 || kb >= n) return 0;
    return (n + kPageSize - 1) / kPageSize;
}

// Largest b with prefix[b] <= t (prefix is non-decreasing, prefix[B] > t).
__device__ __forceinline__ int locate_request(const int* prefix, int B, long t) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

// q fragments (B operand of the score MMA, k = head dim, n = 8 heads) for query heads
// kvh*G + nt*8 + (lane>>2).  Thread c = lane&3 holds 16-byte chunks c, c+4, c+8, c+12 of its head
// row: the contraction index is permuted identically for q and K, which leaves q.K unchanged and
// lets every thread read whole 16-byte chunks.
template <int NT>
__device__ __forceinline__ void load_q_frags(const TopkArgs& a, int b, int kvh, uint32_t (&qf)[NT][16]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + g;
        const bool ok = hh < a.G;
        const uint4* qp = reinterpret_cast<const uint4*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + (ok ? hh : 0)) * kHeadDim);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v = ok ? __ldg(qp + c + 4 * i) : make_uint4(0, 0, 0, 0);
            qf[nt][4 * i + 0] = v.x;
            qf[nt][4 * i + 1] = v.y;
            qf[nt][4 * i + 2] = v.z;
            qf[nt][4 * i + 3] = v.w;
        }
    }
}

// Loads K row `row` (shared memory, 256 B) into the A-fragment word order used with load_q_frags.
// Odd rows read their chunk pairs in swapped order so that the 8 lanes of a shared-memory phase
// (rows 2p and 2p+1) hit disjoint banks; the swap is undone with selects.
__device__ __forceinline__ void load_k_row(const uint8_t* row, int c, int sw, uint32_t (&R)[16]) {
    uint4 t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) t[i] = *reinterpret_cast<const uint4*>(row + 16 * (c + 4 * (i ^ sw)));
#pragma unroll
    for (int li = 0; li < 4; ++li) {
        const uint4 e = t[li], o = t[li ^ 1];
        R[4 * li + 0] = sw ? o.x : e.x;
        R[4 * li + 1] = sw ? o.y : e.y;
        R[4 * li + 2] = sw ? o.z : e.z;
        R[4 * li + 3] = sw ? o.w : e.w;
    }
}

template <int NT>
__global__ void __launch_bounds__(kScoreThreads, 1) score_pass_kernel(TopkArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int page_bytes = kPageSize * a.Hkv * kRowBytes;
    const int stage_bytes = a.spp * page_bytes;
    const int S = a.stages;
    uint8_t* data = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
    uint64_t* empty = full + S;
    int* prefix = reinterpret_cast<int*>(empty + S);   // [B + 1]
    int* scratch = prefix + a.B + 1;                    // [40]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Pages of all requests that need scoring, as one flattened sequence.
    int carry = 0;
    for (int base = 0; base < a.B; base += blockDim.x) {
        const int b = base + tid;
        const int v = (b < a.B) ? score_pages_of(a, b) : 0;
        int tot;
        const int ex = block_exclusive_scan(v, scratch, &tot);
        if (b < a.B) prefix[b] = carry + ex;
        carry += tot;
    }
    if (tid == 0) {
        prefix[a.B] = carry;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kScoreConsumerWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    const long T = carry;
    const long t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
    if (t0 >= t1) return;
    const long nst = (t1 - t0 + a.spp - 1) / a.spp;
    const long page_elems = (long)kPageSize * a.Hkv * kHeadDim;

    if (warp == kScoreConsumerWarps) {
        // ---------------- producer: one thread issues the bulk copies ----------------
        if (lane != 0) return;
        int b = locate_request(prefix, a.B, t0);
        long issued = 0;
        for (long st = 0; st < nst; ++st) {
            const int slot = (int)(st % S);
            if (st >= S && !mbar_wait(&empty[slot], (uint32_t)((st / S - 1) & 1))) {
                report(a.status, SD_ERR_TIMEOUT);
                break;
            }
            const long tb = t0 + st * a.spp;
            const int np = (int)min((long)a.spp, t1 - tb);
            mbar_arrive_expect_tx(&full[slot], (uint32_t)(np * page_bytes));
            for (int i = 0; i < np; ++i) {
                const long t = tb + i;
                while (t >= prefix[b + 1]) ++b;
                const int p = (int)(t - prefix[b]);
                int page = a.page_table[(long)b * a.max_pages + p];
                if (page < 0 || page >= a.num_pages) {
                    report(a.status, SD_ERR_INDEX_OOB);
                    page = 0;   // keep the transaction count whole; the scores of this page are void
                }
                bulk_copy_g2s(data + (size_t)slot * stage_bytes + (size_t)i * page_bytes, a.K + (long)page * page_elems,
                              (uint32_t)page_bytes, &full[slot]);
            }
            issued = st + 1;
        }
        // Never leave while a copy into this CTA's shared memory may still be in flight.
        for (long st = (issued > S ? issued - S : 0); st < issued; ++st)
            if (!mbar_wait(&full[st % S], (uint32_t)((st / S) & 1))) report(a.status, SD_ERR_TIMEOUT);
        return;
    }

    // ---------------- consumers: 8 warps, one (page, kv head) unit at a time ----------------
    const int g = lane >> 2, c = lane & 3, sw = g & 1;
    const int row_stride = a.Hkv * kRowBytes;
    uint32_t qf[NT][16];
    int cur_b = -1, cur_kvh = -1;
    int b = locate_request(prefix, a.B, t0);
    for (long st = 0; st < nst; ++st) {
        const int slot = (int)(st % S);
        if (!mbar_wait(&full[slot], (uint32_t)((st / S) & 1))) {
            report(a.status, SD_ERR_TIMEOUT);
            break;
        }
        const long tb = t0 + st * a.spp;
        const int np = (int)min((long)a.spp, t1 - tb);
        const uint8_t* sdata = data + (size_t)slot * stage_bytes;
        for (int u = warp; u < np * a.Hkv; u += kScoreConsumerWarps) {
            const int pi = u / a.Hkv, kvh = u - pi * a.Hkv;
            const long t = tb + pi;
            while (t >= prefix[b + 1]) ++b;
            const int p = (int)(t - prefix[b]);
            if (b != cur_b || kvh != cur_kvh) {
                load_q_frags<NT>(a, b, kvh, qf);
                cur_b = b;
                cur_kvh = kvh;
            }
            const uint8_t* rows = sdata + (size_t)pi * page_bytes + (size_t)kvh * kRowBytes;
            uint32_t Ra[16], Rb[16];
            load_k_row(rows + (size_t)g * row_stride, c, sw, Ra);
            load_k_row(rows + (size_t)(g + 8) * row_stride, c, sw, Rb);
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_bf16_16816(acc[nt], Ra[2 * j], Rb[2 * j], Ra[2 * j + 1], Rb[2 * j + 1], qf[nt][2 * j],
                                   qf[nt][2 * j + 1]);
            }
            const int n = a.lens[b];
            const int pa = p * kPageSize + g, pb = pa + 8;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + 2 * c + e;
                    if (col < a.G) {
                        float* srow = a.scores + ((long)b * a.Hq + (long)kvh * a.G + col) * a.n_cap;
                        if (pa < n) srow[pa] = acc[nt][e];
                        if (pb < n) srow[pb] = acc[nt][2 + e];
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
}

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
struct SharedKeys {   // candidate list in shared memory, ascending positions
    const uint32_t* k;
    const int* p;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int j) const { return k[j]; }
    __device__ __forceinline__ int pos(int j) const { return p[j]; }
};

// Finds the bin t holding the target-th largest element (target >= 1, counted from the top bin)
// and the number of elements in bins above t.  Every thread must call; results via shared memory.
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

// Refines the k-th key inside bin t (the top 12 bits), then writes the selected positions of src in
// ascending order: keys above the threshold key T, plus the first `quota` keys equal to T.
template <class Src>
__device__ void refine_and_emit(const Src& src, uint32_t t, int above, int take, int32_t* row, int* hist,
                                int* scratch, int* s_sel) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int n = src.size();
    // digit 2: key bits 19..8 among keys whose top 12 bits equal t
    for (int i = tid; i < 4096; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += nthr) {
        const uint32_t key = src.key(j);
        if ((key >> 20) == t) atomicAdd(&hist[(key >> 8) & 0xfffu], 1);
    }
    __syncthreads();
    const int need = take - above;
    select_bin(hist, 4096, need, scratch, s_sel);
    const uint32_t t2 = (uint32_t)s_sel[0];
    const int above2 = s_sel[1];
    __syncthreads();
    // digit 3: key bits 7..0 among keys whose top 24 bits equal (t, t2)
    const uint32_t pre24 = (t << 12) | t2;
    for (int i = tid; i < 256; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += nthr) {
        const uint32_t key = src.key(j);
        if ((key >> 8) == pre24) atomicAdd(&hist[key & 0xffu], 1);
    }
    __syncthreads();
    const int need2 = need - above2;
    select_bin(hist, 256, need2, scratch, s_sel);
    const uint32_t T = (pre24 << 8) | (uint32_t)s_sel[0];
    const int quota = need2 - s_sel[1];   // how many keys equal to T are taken, lowest positions first
    __syncthreads();

    // ordered compaction: tiles of nthr * kSelectItems consecutive entries
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

__global__ void __launch_bounds__(kSelectThreads) select_kernel(TopkArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int* hist = reinterpret_cast<int*>(smem);   // [4096]
    int* scratch = hist + 4096;                  // [40]
    int* s_sel = scratch + 40;                   // [8]
    uint32_t* lkey = reinterpret_cast<uint32_t*>(s_sel + 8);
    int* lpos = reinterpret_cast<int*>(lkey + a.cap);

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
    const float* sc = a.scores + bh * a.n_cap;

    // pass 1: histogram of the top 12 key bits
    for (int i = tid; i < 4096; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int i = tid * 4; i < n; i += nthr * 4) {
        if (i + 3 < n) {
            const float4 v = *reinterpret_cast<const float4*>(sc + i);
            atomicAdd(&hist[float_key(v.x) >> 20], 1);
            atomicAdd(&hist[float_key(v.y) >> 20], 1);
            atomicAdd(&hist[float_key(v.z) >> 20], 1);
            atomicAdd(&hist[float_key(v.w) >> 20], 1);
        } else {
            for (int e = i; e < n; ++e) atomicAdd(&hist[float_key(sc[e]) >> 20], 1);
        }
    }
    __syncthreads();
    select_bin(hist, 4096, take, scratch, s_sel);
    const uint32_t t = (uint32_t)s_sel[0];
    const int above = s_sel[1];
    const int m = above + hist[t];
    __syncthreads();

    if (m <= a.cap) {
        // pass 2: ordered compaction of every key in bins >= t into shared memory
        int base = 0;
        for (int i0 = 0; i0 < n; i0 += nthr * kSelectItems) {
            const int i = i0 + tid * kSelectItems;
            uint32_t key[kSelectItems];
            int cnt = 0;
#pragma unroll
            for (int e = 0; e < kSelectItems; ++e) {
                key[e] = (i + e < n) ? float_key(sc[i + e]) : 0u;
                cnt += (i + e < n) && ((key[e] >> 20) >= t);
            }
            int tot;
            int w = base + block_exclusive_scan(cnt, scratch, &tot);
#pragma unroll
            for (int e = 0; e < kSelectItems; ++e)
                if (i + e < n && (key[e] >> 20) >= t) {
                    if (w < a.cap) {
                        lkey[w] = key[e];
                        lpos[w] = i + e;
                    }
                    ++w;
                }
            base += tot;
        }
        __syncthreads();
        refine_and_emit(SharedKeys{lkey, lpos, min(base, a.cap)}, t, above, take, row, hist, scratch, s_sel);
    } else {
        refine_and_emit(GlobalKeys{sc, n}, t, above, take, row, hist, scratch, s_sel);
    }
    for (int i = take + tid; i < a.k_max; i += nthr) row[i] = -1;
}

// ---------------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------------
size_t score_pass_smem(const TopkArgs& a) {
    const size_t page_bytes = (size_t)kPageSize * a.Hkv * kRowBytes;
    return (size_t)a.stages * a.spp * page_bytes + 2 * sizeof(uint64_t) * a.stages + sizeof(int) * (a.B + 1 + 40);
}

size_t select_smem(const TopkArgs& a) { return sizeof(int) * (4096 + 40 + 8) + (size_t)a.cap * 8; }

cudaError_t launch_score_pass(const TopkArgs& a, int grid, cudaStream_t stream) {
    const size_t smem = score_pass_smem(a);
    if (a.G <= 8) {
        cudaError_t e = cudaFuncSetAttribute(score_pass_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        score_pass_kernel<1><<<grid, kScoreThreads, smem, stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(score_pass_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        score_pass_kernel<2><<<grid, kScoreThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_select(const TopkArgs& a, cudaStream_t stream) {
    const size_t smem = select_smem(a);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<<<a.B * a.Hq, kSelectThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace sd
