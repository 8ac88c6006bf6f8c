// topk_score.cu -- scoring side of the exact top-k indexer ("Oracle Top-K": exact selection of the
// k highest-scoring tokens; "Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit",
// sec. 2, and the indexer of Fig. 1(a) of "Inference-time context sparsity: illusion or
// opportunity?").
//
// threshold_kernel   one cluster of 8 CTAs per (request, KV head) group: the CTAs score kSample
//                    evenly spaced positions for the group's G heads on the tensor cores and
//                    gather the top 16 bits of each score's order-preserving key, head by head, in
//                    distributed shared memory; each CTA then sets the candidate threshold tau of
//                    its heads just below the j-th largest sampled score (a block radix select), j
//                    chosen so that about 1.25 k scores are expected at or above it.
// score_pass_kernel  streams every K page of the requests that need selection exactly once (tiled
//                    TMA tensor copies with 128-byte swizzle into a shared-memory ring, one
//                    producer warp, eight consumer warps) and scores 16 positions x G heads per MMA group
//                    (ldmatrix + mma.sync m16n8k16, bf16 x bf16 -> fp32).  Per page and head it writes a 16-bit mask of
//                    the candidates (scores >= tau) and packs their scores at the start of the
//                    page's 16 slots of the row: no counters, no atomics.  Rows short enough
//                    (tau = -inf) keep every position.  The grid is persistent and the pages of all
//                    requests are split evenly across CTAs, so ragged batches stay balanced.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kScoreConsumerWarps = 8;   // plus one producer warp that issues the copies
constexpr int kThresholdWarps = 4;   // 4 warps: a threshold CTA fits beside a score-pass CTA
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

// q fragments in the natural head-dimension order (for K fragments read with ldmatrix): for k-step
// j, thread (g, c) holds q[head nt*8 + g][16j + 2c, +1] and q[...][16j + 8 + 2c, +1].
template <int NT>
__device__ __forceinline__ void load_q_frags_nat(const TopkArgs& a, int b, int kvh, uint32_t (&qf)[NT][16]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + g;
        const bool ok = hh < a.G;
        const uint32_t* qp =
            reinterpret_cast<const uint32_t*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + (ok ? hh : 0)) * kHeadDim);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            qf[nt][2 * j] = ok ? __ldg(qp + 8 * j + c) : 0u;
            qf[nt][2 * j + 1] = ok ? __ldg(qp + 8 * j + 4 + c) : 0u;
        }
    }
}

// Loads a K row in global memory into the A-fragment word order used with load_q_frags.
__device__ __forceinline__ void load_k_row_global(const __nv_bfloat16* row, int c, uint32_t (&R)[16]) {
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

// Scores of 16 K rows (A fragments Ra: rows g, Rb: rows g + 8) against the q fragments, in two
// independent accumulation chains over the head dimension that are summed at the end.
template <int NT>
__device__ __forceinline__ void score_tile(const uint32_t (&Ra)[16], const uint32_t (&Rb)[16],
                                           const uint32_t (&qf)[NT][16], float (&acc)[NT][4]) {
    float acc2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = acc2[nt][i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mma_bf16_16816(acc[nt], Ra[2 * j], Rb[2 * j], Ra[2 * j + 1], Rb[2 * j + 1], qf[nt][2 * j], qf[nt][2 * j + 1]);
            mma_bf16_16816(acc2[nt], Ra[2 * j + 2], Rb[2 * j + 2], Ra[2 * j + 3], Rb[2 * j + 3], qf[nt][2 * j + 2],
                           qf[nt][2 * j + 3]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] += acc2[nt][i];
}

// Bits 0, 4, 8, ..., 28 of x gathered into bits 0..7.
__device__ __forceinline__ uint32_t gather_nibble_bits(uint32_t x) {
    x &= 0x11111111u;
    x = (x | (x >> 3)) & 0x03030303u;
    x = (x | (x >> 6)) & 0x000f000fu;
    return (x | (x >> 12)) & 0xffu;
}

// ---------------------------------------------------------------------------------------------
// threshold_kernel
// ---------------------------------------------------------------------------------------------
// Rank j in the sample whose score becomes the threshold: about 1.25 take + 16 sample strides lie
// above it -- several standard deviations above take.
__device__ __forceinline__ int sample_rank(int take, int n) {
    const long want = ((long)take * kSample + n - 1) / n;
    return (int)min((long)kSample, want + want / 4 + 16);
}

// The kth largest of kSample 16-bit keys in shared memory (1 <= kth <= kSample), by the whole CTA:
// radix select with two 8-bit digits; per-warp histograms keep atomic contention within a warp.
// hist holds kThresholdWarps * 256 ints; every thread must call.
__device__ uint32_t block_kth_largest16(const uint16_t* keys, int kth, int* hist, int* s_res) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0;
    int remaining = kth;
#pragma unroll 1
    for (int shift = 8; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256 * kThresholdWarps; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        int* wh = hist + 256 * warp;
        for (int i = tid; i < kSample; i += blockDim.x) {
            const uint32_t key = keys[i];
            if (shift == 8 || (key >> 8) == (prefix >> 8)) atomicAdd(&wh[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns bins 255 - 8l - 7 .. 255 - 8l (the highest bins first), summed over warps
            int cnt[8];
            int s = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                int v = 0;
                for (int w = 0; w < kThresholdWarps; ++w) v += hist[256 * w + 255 - 8 * lane - t];
                cnt[t] = v;
                s += v;
            }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int bin = -1, above = 0;
            if (incl - s < remaining && incl >= remaining) {
                int cum = incl - s;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (bin < 0 && cum + cnt[t] >= remaining) {
                        bin = 255 - 8 * lane - t;
                        above = cum;
                    }
                    cum += cnt[t];
                }
            }
            const uint32_t who = __ballot_sync(0xffffffffu, bin >= 0);
            const int src = who ? __ffs(who) - 1 : 0;
            bin = __shfl_sync(0xffffffffu, bin, src);
            above = __shfl_sync(0xffffffffu, above, src);
            if (lane == 0) {
                s_res[0] = bin < 0 ? 0 : bin;   // bin < 0 cannot happen for 1 <= kth <= kSample
                s_res[1] = above;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_res[0] << shift;
        remaining -= s_res[1];
        __syncthreads();
    }
    return prefix;
}

size_t threshold_smem(const TopkArgs& a) {
    const int nt = a.G <= 8 ? 1 : 2;
    return sizeof(uint16_t) * (size_t)nt * kSample + sizeof(int) * (256 * kThresholdWarps + 8);
}

// Cluster of 8 CTAs per (b, kv head) group.  CTA r scores sample tiles r*16 .. r*16 + 15 (16
// positions each) for all G heads and sends the top 16 key bits of head column col to CTA col % 8,
// which holds the keys of columns r and r + 8 and selects their thresholds.
template <int NT>
__global__ void __cluster_dims__(kThresholdCluster, 1, 1) __launch_bounds__(kThresholdWarps * 32)
    threshold_kernel(TopkArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint16_t* skey = reinterpret_cast<uint16_t*>(smem);                // [NT][kSample]: columns r, r + 8
    int* hist = reinterpret_cast<int*>(skey + NT * kSample);           // [warps][256]
    int* s_res = hist + 256 * kThresholdWarps;                         // [8]
    // Wait for the work before this kernel first, then let the score pass launch: the score pass starts
    // streaming K at once, which is safe only once everything before this kernel has completed.
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, c = lane & 3;
    const uint32_t rank = cluster_ctarank();
    const int grp = blockIdx.x / kThresholdCluster;
    const int b = grp / a.Hkv, kvh = grp - b * a.Hkv;
    const long bh0 = (long)b * a.Hq + (long)kvh * a.G;
    const int n = a.lens[b];
    const int kb = a.k[b];
    const bool valid = n > 0 && (long)n <= a.n_cap && kb >= 1;
    if (!valid || kb >= n || n <= a.ccap) {   // the same decision in every CTA of the cluster
        if (rank == 0) {
            const float t = (valid && kb < n) ? -INFINITY : INFINITY;
            for (int col = threadIdx.x; col < a.G; col += blockDim.x) a.tau[bh0 + col] = t;
        }
        return;
    }
    cluster_sync_all();   // every CTA of the cluster runs before any of them writes another's memory
    uint32_t qf[NT][16];
    load_q_frags<NT>(a, b, kvh, qf);
    const int32_t* ptrow = a.page_table + (long)b * a.max_pages;
    const uint32_t skey_s = smem_addr(skey);
    // kTilesPerWarp tiles per warp, two at a time with all four K-row loads of a pair in flight together
    constexpr int kTilesPerCta = kSample / 16 / kThresholdCluster;
    constexpr int kTilesPerWarp = kTilesPerCta / kThresholdWarps;
    static_assert(kTilesPerWarp % 2 == 0, "tiles go in pairs");
#pragma unroll 1
    for (int t0 = 0; t0 < kTilesPerWarp; t0 += 2) {
        uint32_t R[2][2][16];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int tile = (int)rank * kTilesPerCta + warp + kThresholdWarps * (t0 + t);
                const int i = tile * 16 + g + 8 * half;
                const int p = (int)(((long)i * n) / kSample);
                int page = __ldg(ptrow + p / kPageSize);
                if (page < 0 || page >= a.num_pages) page = 0;   // reported by the score pass
                load_k_row_global(a.K + (((long)page * kPageSize + (p % kPageSize)) * a.Hkv + kvh) * kHeadDim, c,
                                  R[t][half]);
            }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int tile = (int)rank * kTilesPerCta + warp + kThresholdWarps * (t0 + t);
            float acc[NT][4];
            score_tile<NT>(R[t][0], R[t][1], qf, acc);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + 2 * c + e;
                    if (col < a.G) {
                        const uint32_t dst = map_shared_rank(skey_s, (uint32_t)(col & 7)) +
                                             (uint32_t)(((col >> 3) * kSample + tile * 16 + g) * 2);
                        st_cluster_u16(dst, (uint16_t)(float_key(acc[nt][e]) >> 16));
                        st_cluster_u16(dst + 16u, (uint16_t)(float_key(acc[nt][2 + e]) >> 16));
                    }
                }
        }
    }
    cluster_sync_all();   // every sample key is in place
    const int kth = sample_rank(kb, n);
    for (int col = (int)rank; col < a.G; col += kThresholdCluster) {
        // the smallest score whose key has the j-th largest top 16 bits: a threshold at most the
        // j-th largest sampled score (a few more candidates, never fewer)
        const uint32_t key16 = block_kth_largest16(skey + (col >> 3) * kSample, kth, hist, s_res);
        float t = key_float(key16 << 16);
        if (t != t) t = -INFINITY;   // the bin of -inf also holds NaN encodings
        if (threadIdx.x == 0) a.tau[bh0 + col] = t;
    }
}

// ---------------------------------------------------------------------------------------------
// score_pass_kernel
// ---------------------------------------------------------------------------------------------
// The producer thread issues the copies of pipeline stage `st` into its slot: per page,
// two tiled TMA loads (head dims 0-63 and 64-127) of box {64 dims, 16 slots, Hkv heads}.  In shared
// memory a page is [half][kv head][slot][64 dims], 128-byte rows swizzled in 1024-byte groups, so
// the 16 rows of one KV head are consecutive and ldmatrix reads them without bank conflicts.
struct StageIssuer {
    const TopkArgs* a;
    const CUtensorMap* tmap;
    const int* prefix;
    uint8_t* data;
    uint64_t* full;
    long t0, t1;
    int stage_bytes, page_bytes;
    int b;   // request cursor (stages are issued in order)
    uint64_t stream_policy;   // K is read once here: its lines go first from L2
    __device__ void issue(long st, int slot) {
        const long tb = t0 + st * a->spp;
        const int np = (int)min((long)a->spp, t1 - tb);
        mbar_arrive_expect_tx(&full[slot], (uint32_t)(np * page_bytes));
        for (int i = 0; i < np; ++i) {
            const long t = tb + i;
            while (t >= prefix[b + 1]) ++b;
            const int p = (int)(t - prefix[b]);
            int page = a->page_table[(long)b * a->max_pages + p];
            if (page < 0 || page >= a->num_pages) {
                report(a->status, SD_ERR_INDEX_OOB);
                page = 0;   // keep the transaction count whole; the scores of this page are void
            }
            uint8_t* dst = data + (size_t)slot * stage_bytes + (size_t)i * page_bytes;
            tma_load_4d_hint(dst, tmap, 0, 0, 0, page, &full[slot], stream_policy);
            tma_load_4d_hint(dst + page_bytes / 2, tmap, 64, 0, 0, page, &full[slot], stream_policy);
        }
    }
};

// (request, kv head) context of the units a consumer warp scores.
template <int NT>
struct GroupCtx {
    int b = -1, kvh = -1, n = 0;
    uint32_t qf[NT][16];
    float tau[NT][2];       // candidate thresholds of head columns nt*8 + 2c + e (+inf past G)
    uint2* prec0;           // record row of head column 0 (the rows of the group's heads follow)
    __device__ __forceinline__ void load(const TopkArgs& a, int b_, int kvh_) {
        const int c = threadIdx.x & 3;
        pdl_wait();   // the thresholds come from the kernel before this one (returns at once after the first)
        load_q_frags_nat<NT>(a, b_, kvh_, qf);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + 2 * c + e;
                tau[nt][e] = (col < a.G) ? __ldg(a.tau + (long)b_ * a.Hq + (long)kvh_ * a.G + col) : INFINITY;
            }
        prec0 = a.prec + ((long)b_ * a.Hq + (long)kvh_ * a.G) * a.mstride;
        n = a.lens[b_];
        b = b_;
        kvh = kvh_;
    }
};

// K fragments of one unit (16 positions x 128 dims) from the swizzled stage by ldmatrix; gbase is
// this lane's row in the unit's 16-row group.
__device__ __forceinline__ void load_unit(uint32_t gbase, const uint32_t (&xo)[4], int half_bytes, uint32_t (&A)[8][4]) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        ldmatrix_x4(gbase + (uint32_t)((j >> 2) * half_bytes) + xo[j & 3], A[j][0], A[j][1], A[j][2], A[j][3]);
}

// Scores NU units of one (request, kv head) group from their K fragments: 16 positions x G heads
// each, two accumulation chains per unit.  Then appends each unit's candidates (scores >= tau) to the
// warp's stream at `so` -- head by head, each head's in position order -- and records per head where
// they start and the page's 16-bit candidate mask.
template <int NT, int NU>
__device__ __forceinline__ void score_units(const TopkArgs& a, const GroupCtx<NT>& x, const uint32_t (&A)[NU][8][4],
                                            const int (&p)[NU], uint32_t& so) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint64_t keep = l2_policy_evict_last();   // the select step reads candidates and records next
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t mc = 0x11111111u << c;                // lanes holding this lane's two head columns
    const uint32_t mlt = 0x11111111u * ((1u << c) - 1u);  // lanes holding the columns before them
    float acc[NU][NT][4], acc2[NU][NT][4];
#pragma unroll
    for (int u = 0; u < NU; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[u][nt][i] = acc2[u][nt][i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; j += 2)
#pragma unroll
        for (int u = 0; u < NU; ++u)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[u][nt], A[u][j][0], A[u][j][1], A[u][j][2], A[u][j][3], x.qf[nt][2 * j],
                               x.qf[nt][2 * j + 1]);
                mma_bf16_16816(acc2[u][nt], A[u][j + 1][0], A[u][j + 1][1], A[u][j + 1][2], A[u][j + 1][3],
                               x.qf[nt][2 * j + 2], x.qf[nt][2 * j + 3]);
            }
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        const int pa = p[u] * kPageSize + g, pb = pa + 8;
        float sc[NT][2][2];
        uint32_t m0[NT][2], m1[NT][2];   // candidate ballots: bit 4g + c = row g (resp. g + 8), columns 2c + e
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                sc[nt][e][0] = acc[u][nt][e] + acc2[u][nt][e];
                sc[nt][e][1] = acc[u][nt][2 + e] + acc2[u][nt][2 + e];
                const float th = x.tau[nt][e];   // +inf past G: such columns have no candidates
                m0[nt][e] = __ballot_sync(0xffffffffu, pa < x.n && sc[nt][e][0] >= th);
                m1[nt][e] = __ballot_sync(0xffffffffu, pb < x.n && sc[nt][e][1] >= th);
            }
        uint32_t pre_nt = 0;   // candidates of the head tiles before nt
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t before = __popc(m0[nt][0] & mlt) + __popc(m1[nt][0] & mlt) + __popc(m0[nt][1] & mlt) +
                                    __popc(m1[nt][1] & mlt);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + 2 * c + e;
                const uint32_t c0 = m0[nt][e] & mc, c1 = m1[nt][e] & mc;
                const uint32_t start = so + pre_nt + before + (e ? __popc(m0[nt][0] & mc) + __popc(m1[nt][0] & mc) : 0u);
                if (c0 & (1u << lane)) st_hint(a.cand + start + __popc(c0 & lt), sc[nt][e][0], keep);
                if (c1 & (1u << lane)) st_hint(a.cand + start + __popc(c0) + __popc(c1 & lt), sc[nt][e][1], keep);
                if (g == 0 && col < a.G)
                    st_hint(x.prec0 + (long)col * a.mstride + p[u],
                            make_uint2(start, gather_nibble_bits(m0[nt][e] >> c) | (gather_nibble_bits(m1[nt][e] >> c) << 8)),
                            keep);
            }
            pre_nt += __popc(m0[nt][0]) + __popc(m1[nt][0]) + __popc(m0[nt][1]) + __popc(m1[nt][1]);
        }
        so += pre_nt;
    }
}

template <int NT>
__device__ __forceinline__ void consume(const TopkArgs& a, const uint8_t* data, uint64_t* full, uint64_t* empty,
                                        const int* prefix, long t0, long t1, long nst, int half_bytes,
                                        int stage_bytes, int page_bytes) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int S = a.stages;
    // ldmatrix source of this lane: row (lane>>3 & 1)*8 + (lane&7) of the 16-row group, 16-byte
    // chunk 2*(j&3) + (lane>>4) of the half holding k-step j, swizzled by the row's low 3 bits.
    const uint32_t row_off = (uint32_t)((((lane >> 3) & 1) * 8 + (lane & 7)) * 128);
    uint32_t xo[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) xo[jj] = (uint32_t)(((2 * jj + (lane >> 4)) ^ (lane & 7)) << 4);
    const uint32_t data_s = smem_addr(data);
    GroupCtx<NT> x;
    int b = locate_request(prefix, a.B, t0);   // request cursor (units come in position order)
    // This warp's candidate stream: 16 G floats reserved per unit it scores, after the units of the
    // earlier CTAs (whose ranges hold t0 pages) and of the earlier warps of this CTA.
    uint32_t so;
    {
        const long nl = (t1 - t0) * a.Hkv;
        long ub = t0 * a.Hkv;
        for (int k = 0; k < warp; ++k) ub += nl > k ? (nl - k + kScoreConsumerWarps - 1) / kScoreConsumerWarps : 0;
        so = (uint32_t)(ub * kPageSize * a.G);
    }
    bool ok = true;
    // 32-bit, incrementally advanced indexing (no 64-bit division on the per-stage path).
    // pi = u / Hkv for u < 16 by multiply and shift: exact since 16 * (hmag - 65536 / Hkv) < 65536 / Hkv.
    const uint32_t hmag = (65536u + a.Hkv - 1) / a.Hkv;
    const int npages = (int)(t1 - t0);
    int slot = 0, page_off = 0;   // stage slot and first page (relative to t0) of the current stage
    uint32_t phase = 0;
    const int ups = a.spp * a.Hkv;   // <= 16: stages hold at most 64 KB of 4 KB-per-head pages
    int ustart = warp;               // this warp's first unit in the current stage: (warp - st*ups) mod 8
    const int ustep = ups & (kScoreConsumerWarps - 1);
    // shared-memory address of this lane's row for unit u of the current stage; sets the request,
    // position page and kv head
    auto locate = [&](int u, int& ub, int& up, int& ukvh) -> uint32_t {
        const int pi = (int)(((uint32_t)u * hmag) >> 16);
        ukvh = u - pi * a.Hkv;
        const long t = t0 + page_off + pi;
        while (t >= prefix[b + 1]) ++b;
        ub = b;
        up = (int)(t - prefix[b]);
        return data_s + (uint32_t)(slot * stage_bytes + pi * page_bytes + ukvh * 2048) + row_off;
    };
    // Stage by stage: wait for it, copy this warp's (at most two) units of it into registers,
    // release it at once (so that the producer can refill the slot while this warp computes), then
    // score them -- together when they share a (request, kv head) context.
    for (long st = 0; st < nst; ++st) {
        // warp-uniform outcome: the ballots need every lane
        if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], phase))) {
            ok = false;
            break;
        }
        const int nu = min(ups, (npages - page_off) * a.Hkv);   // units in this stage
        const int u = ustart;
        const bool one = u < nu, two = u + kScoreConsumerWarps < nu;
        int b1 = 0, p1 = 0, k1 = 0, b2 = 0, p2 = 0, k2 = 0;
        uint32_t A[2][8][4];
        if (one) load_unit(locate(u, b1, p1, k1), xo, half_bytes, A[0]);
        if (two) load_unit(locate(u + kScoreConsumerWarps, b2, p2, k2), xo, half_bytes, A[1]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }
        page_off += a.spp;
        ustart = (ustart - ustep) & (kScoreConsumerWarps - 1);
        if (!one) continue;
        if (b1 != x.b || k1 != x.kvh) x.load(a, b1, k1);
        if (two && b2 == b1 && k2 == k1) {
            const int pp[2] = {p1, p2};
            score_units<NT, 2>(a, x, A, pp, so);
        } else {
            const int pp[1] = {p1};
            score_units<NT, 1>(a, x, reinterpret_cast<const uint32_t(&)[1][8][4]>(A[0]), pp, so);
            if (two) {
                x.load(a, b2, k2);
                const int pp2[1] = {p2};
                score_units<NT, 1>(a, x, reinterpret_cast<const uint32_t(&)[1][8][4]>(A[1]), pp2, so);
            }
        }
    }
    if (!ok) report(a.status, SD_ERR_TIMEOUT);
}

template <int NT>
__device__ __forceinline__ void score_pass(const TopkArgs& a, const CUtensorMap& tmap) {
    extern __shared__ __align__(1024) uint8_t smem[];
    // No wait here: the threshold kernel launched this grid only after the work before it had completed,
    // so the inputs can be read at once and the K stream overlaps the threshold kernel.  Its output, the
    // thresholds, is read after griddepcontrol.wait (GroupCtx::load).
    pdl_launch_dependents();
    const int page_bytes = kPageSize * a.Hkv * kRowBytes;
    const int half_bytes = page_bytes / 2;
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
        if (blockIdx.x == 0) {   // for a row the select step has to recompute
            a.inputs[0] = a.q;
            a.inputs[1] = a.K;
            a.inputs[2] = a.page_table;
        }
    }
    __syncthreads();

    const long T = carry;
    const long t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
    if (t0 >= t1) return;
    const long nst = (t1 - t0 + a.spp - 1) / a.spp;

    if (warp == kScoreConsumerWarps) {
        // ---------------- producer: one thread issues the tensor copies ----------------
        if (lane != 0) return;
        StageIssuer is{&a, &tmap, prefix, data, full, t0, t1, stage_bytes, page_bytes, locate_request(prefix, a.B, t0),
                       l2_policy_evict_first()};
        long issued = 0;
        int slot = 0;
        uint32_t phase = 0;   // parity of the release the slot's next refill waits for
        for (long st = 0; st < nst; ++st) {
            if (st >= S && !mbar_wait(&empty[slot], phase)) {
                report(a.status, SD_ERR_TIMEOUT);
                break;
            }
            is.issue(st, slot);
            issued = st + 1;
            if (++slot == S) {
                slot = 0;
                if (st >= S) phase ^= 1u;
            }
        }
        // Never leave while a copy into this CTA's shared memory may still be in flight.
        for (long st = (issued > S ? issued - S : 0); st < issued; ++st)
            if (!mbar_wait(&full[st % S], (uint32_t)((st / S) & 1))) report(a.status, SD_ERR_TIMEOUT);
        return;
    }

    // ---------------- consumers ----------------
    // Unit U = (page offset U / Hkv, kv head U % Hkv) of this CTA's range; warp w takes
    // U = w, w + 8, w + 16, ...  Every warp waits for and releases every stage in order, whether or
    // not it has a unit there, which keeps the arrival count of each release barrier fixed.  With
    // Hkv dividing 8, a warp always meets the same KV head.
    consume<NT>(a, data, full, empty, prefix, t0, t1, nst, half_bytes, stage_bytes, page_bytes);
}

// G <= 8.  At most 144 registers per thread: a threshold CTA (4 warps, <= 80 registers) then fits on
// an SM beside a score-pass CTA -- also within each SM sub-partition's register file, which holds three
// of the score pass's nine warps plus one threshold warp -- so the score pass starts streaming K while
// the threshold kernel finishes.
__global__ void __maxnreg__(144) score_pass_kernel_g8(TopkArgs a, const __grid_constant__ CUtensorMap tmap) {
    score_pass<1>(a, tmap);
}
// 8 < G <= 16.
__global__ void __launch_bounds__(kScoreThreads, 1) score_pass_kernel_g16(TopkArgs a,
                                                                          const __grid_constant__ CUtensorMap tmap) {
    score_pass<2>(a, tmap);
}

// ---------------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------------
size_t score_pass_smem(const TopkArgs& a) {
    const size_t page_bytes = (size_t)kPageSize * a.Hkv * kRowBytes;
    return (size_t)a.stages * a.spp * page_bytes + 2 * sizeof(uint64_t) * a.stages + sizeof(int) * (a.B + 1 + 40);
}

cudaError_t launch_threshold(const TopkArgs& a, cudaStream_t stream) {
    const size_t smem = threshold_smem(a);
    cudaError_t e;
    if (a.G <= 8) {
        e = cudaFuncSetAttribute(threshold_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(threshold_kernel<1>, dim3(a.B * a.Hkv * kThresholdCluster), dim3(kThresholdWarps * 32), smem,
                       stream, a);
    } else {
        e = cudaFuncSetAttribute(threshold_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(threshold_kernel<2>, dim3(a.B * a.Hkv * kThresholdCluster), dim3(kThresholdWarps * 32), smem,
                       stream, a);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

namespace {

// The K cache as a 4-D tensor for TMA: {head dim 128, slot 16, kv head Hkv, page num_pages} with
// byte strides {2, Hkv*256, 256, 16*Hkv*256}; box {64, 16, Hkv, 1}; 128-byte swizzle.  Encoded on
// the host through the driver entry point, and kept for the last (device, K, num_pages, Hkv).
struct KMapCache {
    std::mutex mu;
    PFN_cuTensorMapEncodeTiled encode = nullptr;
    int dev = -1;
    const void* K = nullptr;
    int num_pages = 0, Hkv = 0;
    CUtensorMap map;
};
KMapCache g_kmap;

cudaError_t k_tensor_map(const TopkArgs& a, CUtensorMap* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_kmap.mu);
    if (g_kmap.encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
        g_kmap.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
    }
    if (g_kmap.dev != dev || g_kmap.K != a.K || g_kmap.num_pages != a.num_pages || g_kmap.Hkv != a.Hkv) {
        const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)kPageSize, (cuuint64_t)a.Hkv,
                                    (cuuint64_t)a.num_pages};
        const cuuint64_t strides[3] = {(cuuint64_t)a.Hkv * kRowBytes, (cuuint64_t)kRowBytes,
                                       (cuuint64_t)kPageSize * a.Hkv * kRowBytes};
        const cuuint32_t box[4] = {64, (cuuint32_t)kPageSize, (cuuint32_t)a.Hkv, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        const CUresult r = g_kmap.encode(&g_kmap.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(
                                         static_cast<const void*>(a.K)), dims, strides, box, estr,
                                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            g_kmap.dev = -1;
            return cudaErrorInvalidValue;
        }
        g_kmap.dev = dev;
        g_kmap.K = a.K;
        g_kmap.num_pages = a.num_pages;
        g_kmap.Hkv = a.Hkv;
    }
    *out = g_kmap.map;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_score_pass(const TopkArgs& a, int grid, cudaStream_t stream) {
    CUtensorMap tmap;
    cudaError_t e = k_tensor_map(a, &tmap);
    if (e != cudaSuccess) return e;
    const size_t smem = score_pass_smem(a);
    if (a.G <= 8) {
        e = cudaFuncSetAttribute(score_pass_kernel_g8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(score_pass_kernel_g8, dim3(grid), dim3(kScoreThreads), smem, stream, a, tmap);
    } else {
        e = cudaFuncSetAttribute(score_pass_kernel_g16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(score_pass_kernel_g16, dim3(grid), dim3(kScoreThreads), smem, stream, a, tmap);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
