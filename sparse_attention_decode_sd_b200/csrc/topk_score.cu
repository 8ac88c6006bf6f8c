// topk_score.cu -- score pass of the exact top-k indexer ("Oracle Top-K": exact selection of the k
// highest-scoring tokens; "Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit",
// sec. 2, and the indexer of Fig. 1(a) of "Inference-time context sparsity: illusion or
// opportunity?").
//
// score_pass_kernel streams every K page of the requests that need selection exactly once (1-D bulk
// copies on the TMA engine into a shared-memory ring, one producer warp, eight consumer warps),
// scores 16 positions x G heads per MMA group on the tensor cores (mma.sync m16n8k16, bf16 x bf16
// -> fp32) and writes fp32 scores [B][Hq][n_cap] to the workspace.  The grid is persistent and the
// pages of all requests are split evenly across CTAs, so ragged batches stay balanced.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kScoreConsumerWarps = 8;
constexpr int kScoreThreads = (kScoreConsumerWarps + 1) * 32;

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
    pdl_enter();
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
// host launcher
// ---------------------------------------------------------------------------------------------
size_t score_pass_smem(const TopkArgs& a) {
    const size_t page_bytes = (size_t)kPageSize * a.Hkv * kRowBytes;
    return (size_t)a.stages * a.spp * page_bytes + 2 * sizeof(uint64_t) * a.stages + sizeof(int) * (a.B + 1 + 40);
}

cudaError_t launch_score_pass(const TopkArgs& a, int grid, cudaStream_t stream) {
    const size_t smem = score_pass_smem(a);
    if (a.G <= 8) {
        cudaError_t e = cudaFuncSetAttribute(score_pass_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(score_pass_kernel<1>, dim3(grid), dim3(kScoreThreads), smem, stream, a);
        if (e != cudaSuccess) return e;
    } else {
        cudaError_t e = cudaFuncSetAttribute(score_pass_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(score_pass_kernel<2>, dim3(grid), dim3(kScoreThreads), smem, stream, a);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace sd
