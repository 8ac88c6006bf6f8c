// sparse_decode.cu -- exact attention over the selected rows of a paged GQA KV cache ("Sparse" mode
// of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?"; SDPA of the xllm
// survey sec. 1.1 restricted to the selected set), and the dense comparator over every row
// ("Dense" mode of the same figure).
//
// Sparse decode, two kernels per call (per-head walk):
//   rows_kernel           one group of threads per (request, query head) row of idx: checks the row
//                         (ascending positions below N_b, then negative padding only), finds its length
//                         (the index of the first negative entry), zeroes the output of empty rows and
//                         the row's arrival counter, and writes per-CTA length sums.  Rows of a
//                         stochastic selection (weighted mode) also get the log2 weight of their drawn
//                         entries.  It releases the decode grid as soon as it starts.
//   sparse_decode_kernel  one warp per CTA, a persistent grid of one wave (12 warps per SM).  The
//                         selected entries of all rows are cut evenly across the warps and each warp
//                         streams its entries in tiles of 16 rows.  The walk starts before rows_kernel
//                         ends, on the split that holds when every row has k_max entries (the
//                         indexer's rows); after the wait, the entry count confirms that split or the
//                         walk restarts on the row lengths.  Full rows are visited in the order of
//                         their start offset inside a warp's share, so that the G heads of a GQA
//                         group read the positions they share at the same time (the second read comes
//                         from L2).  Per tile, in a software pipeline that waits for no load but the
//                         gather itself: positions loaded four tiles ahead, mapped through the page
//                         table two tiles ahead, and the 256-byte K and V rows gathered one tile ahead
//                         by TMA four-row gathers (tile::gather4, 64-dim halves with the 128-byte
//                         swizzle) into a two-stage shared-memory ring.  On the tensor cores
//                         (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//                             S   = K_tile (16 rows x 128) . q              8 MMAs (q: column 0 of B)
//                             o  += V_tile^T (128 x 16 rows) . [p_hi, p_lo] 8 MMAs (columns 0 and 1 of B)
//                         with an fp32 online softmax in between; the weights p enter as a bf16 high
//                         part and a bf16 residual, and the head's output is the sum of the two
//                         accumulator columns.  A warp's part of one row is a "segment": each warp
//                         stores its (max, sum, output) partial and the last of the row's warps to
//                         arrive (a counter per row) merges the partials by log-sum-exp; a row held
//                         by one warp is written out directly.
//
// Sparse decode over GQA groups (chosen by the host when the heads of a group are expected to
// share many rows), four kernels: validate_kernel checks idx in chunks of 16 entries over the whole
// grid (every rule is on adjacent entries, and no row lengths are needed); union_masks_kernel sets,
// per (group, 16384-position range), a byte (two for G > 8) per position whose bits are the heads
// that selected it; dense_decode_kernel<., true> walks the masked positions of every group -- only
// those, or whole tiles with their masks where the union covers nearly every position -- one
// gathered tile serving every head that selected its rows; merge_kernel combines the partials.
//
// Dense decode (the comparator), three kernels: ranges_kernel counts the positions of each
// kRange-position range of every (request, KV head) group; dense_decode_kernel walks all rows of every
// group with the same tile pipeline, one 16-row tile serving all G heads of the group (S = K_tile . Q^T
// with the G heads as columns), its first range found from the counts; merge_kernel (four warps per
// (b, h)) combines the segment partials.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kStages = 3;                  // tiles in flight per dense decode warp
constexpr int kSparseStages = 2;            // tiles in flight per sparse decode warp
constexpr int kTileRows = 16;
constexpr int kRowPitch = kRowBytes + 16;   // padded shared-memory row: ldmatrix phases hit 8 distinct bank groups
constexpr int kTileBytes = kTileRows * kRowPitch;
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;
constexpr uint32_t kNoRow = 0xffffffffu;    // cache row of a position that maps to none (dense decode)
constexpr int kPrologue = 8;                // length sums per lane loaded together by a decode warp

// ---------------------------------------------------------------------------------------------
// the tile pipeline shared by both decodes
// ---------------------------------------------------------------------------------------------
struct __align__(128) DecodeSmem {
    uint8_t kv[kStages][2][kTileBytes];       // K tile, V tile: 16 rows x 272 B
    uint32_t meta_mask[kStages][kTileRows];   // head bitmask of each tile row (0: no row)
    int info[kStages][8];                     // rows, flags, owner, segment slot, segments of the owner
};

size_t decode_smem() { return sizeof(DecodeSmem); }

// A tile fetched one iteration ahead: row descriptors live in lanes 0..15.  Dense walk: the cache row
// is worked out at the prefetch (the page-table entry comes from L2).  Group walk: the page entry and
// the head mask (which comes from DRAM) are loads that the prefetch only issues; they are first
// examined when the tile is issued, an iteration later, so that the warp computes the tile in between
// without waiting for them.
struct TileDesc {
    int rows, flags;
    int owner;          // dense: group b * Hkv + kvh; sparse: row b * Hq + h
    int seg_j, nseg;    // segment slot of this warp in the owner, and the owner's segment count (sparse)
    uint32_t row_idx;   // dense walk: this lane's cache row (lanes < rows); kNoRow: none (skipped)
    int page;           // group walk: this lane's page-table entry (lanes < rows)
    uint32_t sub;       // group walk: this lane's row within the page block, slot * Hkv + kvh
    uint32_t mask;      // heads (columns) that attend to it (group walk, 0: none, the row is not gathered)
};

__device__ __forceinline__ TileDesc empty_tile() {
    TileDesc d;
    d.rows = 0;
    d.flags = 0;
    d.owner = d.seg_j = d.nseg = 0;
    d.row_idx = 0;
    d.page = 0;
    d.sub = 0;
    d.mask = 0;
    return d;
}

// Writes the tile's metadata to `stage` and issues its row gathers: 16-byte cp.async chunks, lane l
// copying chunk l % 16 of rows l / 16, l / 16 + 2, ...; missing rows are zero-filled.  One
// cp.async group per tile.  This is the first use of the row indices loaded by the prefetch one
// iteration earlier, so that load stays in flight while the warp computes the previous tile.
template <bool kUnion>
__device__ __forceinline__ void issue_tile(const DecodeArgs& a, DecodeSmem& ws, int stage, const TileDesc& d) {
    const int lane = threadIdx.x & 31;
    uint32_t row_idx = d.row_idx;
    if (kUnion) {   // a selected row whose page entry is outside the cache is reported and skipped
        const bool sel = lane < d.rows && d.mask != 0u;
        const bool bad = sel && (d.page < 0 || d.page >= a.num_pages);
        if (bad) report(a.status, SD_ERR_INDEX_OOB);
        row_idx = (sel && !bad) ? (uint32_t)d.page * (uint32_t)(kPageSize * a.Hkv) + d.sub : kNoRow;
    }
    if (lane < kTileRows) ws.meta_mask[stage][lane] = (lane < d.rows && row_idx != kNoRow) ? d.mask : 0u;
    if (lane == 0) {
        ws.info[stage][0] = d.rows;
        ws.info[stage][1] = d.flags;
        ws.info[stage][2] = d.owner;
        ws.info[stage][3] = d.seg_j;
        ws.info[stage][4] = d.nseg;
    }
    if (d.rows > 0) {
        const uint32_t kdst = smem_addr(ws.kv[stage][0]);
        const uint32_t vdst = smem_addr(ws.kv[stage][1]);
        const char* kb = reinterpret_cast<const char*>(a.K);
        const char* vb = reinterpret_cast<const char*>(a.V);
        const int ch = lane & 15;
#pragma unroll
        for (int i = 0; i < kTileRows / 2; ++i) {
            const int r = (lane >> 4) + 2 * i;
            const uint32_t ri = __shfl_sync(0xffffffffu, row_idx, r);
            const bool ok = r < d.rows && ri != kNoRow;
            const size_t off = ok ? (((size_t)ri << 8) + (ch << 4)) : 0;
            const uint32_t doff = (uint32_t)(r * kRowPitch + (ch << 4));
            cp_async_16(kdst + doff, kb + off, ok);
            cp_async_16(vdst + doff, vb + off, ok);
        }
    }
    cp_async_commit();
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

// Consumer-side state of one warp: NT groups of 8 columns (query heads).
template <int NT>
struct Softmax {
    float m[NT][2];          // running max (log2 units) of columns nt*8 + 2c + e
    float l[NT][2];          // per-thread partial sums of the same columns
    float acc[NT][8][4];     // O^T fragments: dims 16*mt + g (+8) x columns nt*8 + 2c (+1)
    uint32_t qb[NT][8][2];   // Q^T fragments (B operand) of the current owner
};

template <int NT>
__device__ __forceinline__ void reset_state(Softmax<NT>& st) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        st.m[nt][0] = st.m[nt][1] = -INFINITY;
        st.l[nt][0] = st.l[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) st.acc[nt][mt][0] = st.acc[nt][mt][1] = st.acc[nt][mt][2] = st.acc[nt][mt][3] = 0.f;
    }
}

template <int NT>
__device__ __forceinline__ void compute_tile(const DecodeArgs& a, const DecodeSmem& ws, int stage, Softmax<NT>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint32_t kbase = smem_addr(ws.kv[stage][0]);
    const uint32_t vbase = smem_addr(ws.kv[stage][1]);
    const int mi = lane >> 3, r8 = lane & 7;

    // S (16 rows x 8 columns per nt) = K_tile . Q^T
    float s[NT][4], s2[NT][4];   // two accumulators (even / odd k-blocks) halve the MMA dependency chain
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
    {
        const uint32_t rowaddr = kbase + (uint32_t)((((mi & 1) << 3) + r8) * kRowPitch + ((mi >> 1) << 4));
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(rowaddr + 32 * j, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (j & 1) mma_bf16_16816(s2[nt], a0, a1, a2, a3, st.qb[nt][j][0], st.qb[nt][j][1]);
                else mma_bf16_16816(s[nt], a0, a1, a2, a3, st.qb[nt][j][0], st.qb[nt][j][1]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
    }
    // mask columns that do not attend to a row (rows g and g+8 of the tile), online softmax per column
    const uint32_t mr0 = ws.meta_mask[stage][g], mr1 = ws.meta_mask[stage][g + 8];
    float p[NT][2][2];   // [nt][e][row g / g+8]
    float alpha[NT][2];
    bool rescale = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int hh = nt * 8 + 2 * c + e;
            const float z0 = ((mr0 >> hh) & 1u) ? s[nt][e] * a.scale_log2 : -INFINITY;
            const float z1 = ((mr1 >> hh) & 1u) ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
            float tm = fmaxf(z0, z1);
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
            const float mo = st.m[nt][e];
            const float mn = fmaxf(mo, tm);
            const float base = (mn == -INFINITY) ? 0.f : mn;
            p[nt][e][0] = fast_exp2(z0 - base);
            p[nt][e][1] = fast_exp2(z1 - base);
            const float al = (mo == mn || mo == -INFINITY) ? 1.f : fast_exp2(mo - mn);
            alpha[nt][e] = al;
            rescale |= al != 1.f;
            st.l[nt][e] = st.l[nt][e] * al + p[nt][e][0] + p[nt][e][1];
            st.m[nt][e] = mn;
        }
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                st.acc[nt][mt][0] *= alpha[nt][0];
                st.acc[nt][mt][1] *= alpha[nt][1];
                st.acc[nt][mt][2] *= alpha[nt][0];
                st.acc[nt][mt][3] *= alpha[nt][1];
            }
    }
    // P as the B operand (16 rows x 8 columns): bf16 high part and residual, transposed by movmatrix
    uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const uint32_t hi = pack_bf16x2(p[nt][0][rr], p[nt][1][rr]);
            const uint32_t lo = pack_bf16x2(p[nt][0][rr] - bf16_lo(hi), p[nt][1][rr] - bf16_hi(hi));
            bh[nt][rr] = movmatrix_trans(hi);
            bl[nt][rr] = movmatrix_trans(lo);
        }
    }
    // O^T += V_tile^T . P
    {
        const uint32_t rowaddr = vbase + (uint32_t)((((mi >> 1) << 3) + r8) * kRowPitch + ((mi & 1) << 4));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(rowaddr + 32 * mt, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(st.acc[nt][mt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
                mma_bf16_16816(st.acc[nt][mt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
            }
        }
    }
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// ---------------------------------------------------------------------------------------------
// sparse decode: rows_kernel
// ---------------------------------------------------------------------------------------------
// One group of a.tpr threads (whole warps) per row, a.rpc rows per CTA.  Each thread takes kRowBatch
// consecutive entries per pass (the whole row in one pass when k_max <= kRowBatch * tpr), so
// consecutive lanes hold consecutive runs and an entry's predecessor is in the same thread or the
// lane before.  Checks the row (ascending positions below N_b, then negative padding only), finds
// its length (the index of the first negative entry), zeroes the output of empty rows and the
// row's arrival counter, and writes per-CTA length sums.  Positions are mapped to cache rows by the
// decode kernel itself, as it streams.
// U passes over a row have their loads in flight together (rows longer than two passes take U = 4,
// with one CTA per SM for the registers).
template <int U>
__global__ void __launch_bounds__(1024, U == 1 ? 2 : 1) rows_kernel(DecodeArgs a) {
    __shared__ int s_neg[32];   // per warp: first negative entry it saw
    __shared__ int s_len[32];   // per row of this CTA
    // The decode kernel is released only after this wait: when its grid starts, all earlier work in
    // the stream (the indexer writing idx, anything writing q, K, V or the page table) is complete, so
    // it may read idx before its own wait, which it needs only for the row lengths and counters.
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tpr = a.tpr, wpr = tpr >> 5;
    const int rl = tid / tpr, t = tid - rl * tpr;
    const int R = a.B * a.Hq;
    const int r = blockIdx.x * a.rpc + rl;
    const int k_max = a.k_max;
    int first_neg = k_max;
    int drawn = 0;   // weighted mode: entries carrying kSampledFlag
    if (r < R) {   // uniform over the row's warps
        const int b = r / a.Hq;
        const int n = checked_len(a.lens, b, a.n_cap, a.status);
        const int32_t* row = a.idx + (long)r * k_max;
        for (int base = 0; base < k_max; base += U * tpr * kRowBatch) {   // uniform over the row's threads
            int v[U][kRowBatch], pv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {   // pass u: entries base + u tpr kRowBatch + ...
                const int j0 = base + (u * tpr + t) * kRowBatch;
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) v[u][i] = j0 + i < k_max ? __ldg(row + j0 + i) : -1;
                // the entry before this warp's first one (inside the row)
                pv[u] = (lane == 0 && j0 > 0 && j0 < k_max) ? __ldg(row + j0 - 1) : -1;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j0 = base + (u * tpr + t) * kRowBatch;
                if (a.weighted) {   // positions without the flag; count the drawn entries
#pragma unroll
                    for (int i = 0; i < kRowBatch; ++i)
                        if (v[u][i] >= 0) {
                            drawn += (v[u][i] & kSampledFlag) ? 1 : 0;
                            v[u][i] &= kPosMask;
                        }
                    if (pv[u] >= 0) pv[u] &= kPosMask;
                }
                int p = __shfl_up_sync(0xffffffffu, v[u][kRowBatch - 1], 1);
                if (lane == 0) p = pv[u];
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) {
                    const int j = j0 + i;
                    if (j < k_max) {
                        if (v[u][i] < 0) {
                            first_neg = min(first_neg, j);
                        } else if (v[u][i] >= n) {
                            report(a.status, SD_ERR_INDEX_OOB);
                        } else if (j > 0 && (p < 0 || p >= v[u][i])) {
                            report(a.status, SD_ERR_ORDER);
                        }
                    }
                    p = v[u][i];
                }
            }
        }
    }
    first_neg = __reduce_min_sync(0xffffffffu, first_neg);
    drawn = __reduce_add_sync(0xffffffffu, drawn);
    __shared__ int s_drawn[32];
    if (lane == 0) {
        s_neg[warp] = first_neg;
        s_drawn[warp] = drawn;
    }
    __syncthreads();
    if (t == 0) {
        int m = k_max, dr = 0;
        for (int w = 0; w < wpr; ++w) {
            m = min(m, s_neg[rl * wpr + w]);
            dr += s_drawn[rl * wpr + w];
        }
        if (r < R) {
            a.rlen[r] = m;
            a.arrive[r] = 0;
            if (a.weighted) {   // each drawn entry stands for (N_b - plain entries) / drawn rows
                const int n = checked_len(a.lens, r / a.Hq, a.n_cap, nullptr);
                a.rlw[r] = dr > 0 && n > m - dr ? log2f((float)(n - (m - dr)) / (float)dr) : 0.f;
            }
        } else {
            m = 0;
        }
        s_len[rl] = m;
    }
    __syncthreads();
    if (r < R && s_len[rl] == 0)
        for (int d = t; d < kHeadDim; d += tpr) a.out[(long)r * kHeadDim + d] = 0.f;
    if (tid == 0) {
        int sum = 0;
        for (int i = 0; i < a.rpc; ++i) sum += s_len[i];
        a.bsum[blockIdx.x] = sum;
    }
}

// ---------------------------------------------------------------------------------------------
// sparse decode: sparse_decode_kernel
// ---------------------------------------------------------------------------------------------
// Shared memory of one decode warp: kSparseStages tiles of 16 gathered rows.  A tile holds four
// 2 KB blocks -- K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127 -- each 16 rows of 128 B
// with the 128-byte swizzle of the TMA copy (16-byte chunk c of row r stored at chunk c ^ (r & 7)),
// so that ldmatrix reads eight rows of one chunk column without bank conflicts.
constexpr int kHalfBlock = kTileRows * 128;                 // 2 KB: 16 rows x 64 dims
constexpr int kGatherTile = 4 * kHalfBlock;                 // K and V, both halves
struct SparseSmem {   // placed at a 1024-byte aligned address (swizzle atoms)
    uint8_t kv[kSparseStages][kGatherTile];
    uint64_t full[kSparseStages];           // TMA completion of each stage
    int info[kSparseStages][4];             // rows | flags << 5 | valid-row mask << 16, row,
                                            // segment slot | segments << 16, drawn-row mask
    uint32_t q[kSparseStages][kHeadDim / 2];   // q of the row a tile opens (bf16 pairs)
};

size_t sparse_decode_smem() { return sizeof(SparseSmem) + 1008; }   // + alignment slack (the base is 16-byte aligned)

// The warp's walk over its entries.  Everything is warp-uniform; the per-row values are computed
// once when the walk enters a row.
struct RowWalker {
    int e, e_end;        // next entry (global order) and the end of this warp's share
    int epw;             // entries per warp
    int r;               // row b * Hq + h holding entry e
    int rstart, rend;    // global entry range of row r
    int next_len;        // length of row r + 1 (0 past the last row), loaded on entering row r
    int seg;             // segment slot of this warp in row r | the row's segment count << 16
    int pt_off;          // b * max_pages: row r's request in the page table
    int kvh;             // KV head of row r
    const int32_t* ix;   // idx of row r, indexed by global entry
    bool full;           // every row holds k_max entries (row lengths need no lookup)
    bool seg_new;        // the next tile opens a segment
    int seq;             // tiles handed out so far
    int o_lane, o_step;  // offset order: o(lane) and 32 k_max mod epw
};

// With full rows, the walk's slot i (entries [i k_max, (i + 1) k_max)) starts at offset
// o(i) = i k_max mod epw inside a warp's share, and every warp advances through its share at about
// the same pace: the entry at offset o is reached at about the same time o / rate in every warp.
// Rows are given to slots in the order of (o(i), i), so the G heads of a GQA group sit in slots of
// nearly equal offset and read the positions they share at nearly the same time: the second read
// comes from L2.  (In plain row order sibling heads drift apart by k_max mod epw per row.)  Row of
// slot i = the rank of (o(i), i) among all slots, counted by the warp (R / 32 steps per lane).
template <bool kOrder>
__device__ __forceinline__ int row_of_slot(const DecodeArgs& a, const RowWalker& w, int slot) {
    if constexpr (!kOrder) return slot;
    const int lane = threadIdx.x & 31;
    const int R = a.B * a.Hq;
    const int o = (int)((uint32_t)(slot * a.k_max) % (uint32_t)w.epw);   // slot k_max < 2^31
    int oi = w.o_lane;
    int rank = 0;
    for (int i = lane; i < R; i += 32) {
        rank += (oi < o || (oi == o && i < slot)) ? 1 : 0;
        oi += w.o_step;
        if (oi >= w.epw) oi -= w.epw;
    }
    return __reduce_add_sync(0xffffffffu, rank);
}

__device__ __forceinline__ void enter_row(const DecodeArgs& a, RowWalker& w, int r, int rstart, int len) {
    const int R = a.B * a.Hq;
    w.r = r;
    w.rstart = rstart;
    w.rend = rstart + len;
    const int first_warp = rstart / w.epw;
    w.seg = ((int)blockIdx.x - first_warp) | (((w.rend - 1) / w.epw - first_warp + 1) << 16);
    const int b = r / a.Hq;
    w.kvh = (r - b * a.Hq) / a.G;
    w.pt_off = b * a.max_pages;
    w.ix = a.idx + (long)r * a.k_max - rstart;
    w.next_len = r + 1 < R ? (w.full ? a.k_max : __ldg(a.rlen + r + 1)) : 0;
    w.seg_new = true;
}

// One tile of the walk: warp-uniform fields, plus per lane (lanes < rows) the selected position v
// and, one step later, its page-table entry.
struct RowTile {
    int hdr;            // rows | flags << 5 | stage << 8
    int r, seg;         // row and segment (as in RowWalker)
    int pt_off, kvh;
    int v;              // this lane's position (lanes < rows)
    int page;           // this lane's page-table entry (-1: not looked up)
    uint2 q2;           // a tile that opens a row: this lane's 8 bytes of the row's q
};

// The next tile of the walk; issues the loads of its positions (first used two steps later).
template <bool kOrder>
__device__ __forceinline__ RowTile next_row_tile(const DecodeArgs& a, RowWalker& w) {
    const int lane = threadIdx.x & 31;
    RowTile d;
    const int stage = w.seq++ & (kSparseStages - 1);
    d.r = w.r;
    d.seg = w.seg;
    d.pt_off = w.pt_off;
    d.kvh = w.kvh;
    d.v = -1;
    d.page = -1;
    d.q2 = make_uint2(0u, 0u);
    const int rows = min(kTileRows, min(w.rend, w.e_end) - w.e);
    if (rows <= 0) {   // the share is done (rows < 0 is not reached: lengths and sums come from one pass)
        w.e = w.e_end;
        d.hdr = (kFlagEnd << 5) | (stage << 8);
        return d;
    }
    int flags = w.seg_new ? kFlagFirst : 0;
    w.seg_new = false;
    if (lane < rows) d.v = __ldcg(w.ix + w.e + lane);   // L2: idx may be read before this grid's wait
    w.e += rows;
    if (w.e == w.rend || w.e == w.e_end) {
        flags |= kFlagLast;
        if (w.e < w.e_end) {   // the next non-empty row (one exists: entries remain)
            if (kOrder && w.full) {   // the next slot's row
                enter_row(a, w, row_of_slot<kOrder>(a, w, w.rend / a.k_max), w.rend, a.k_max);
            } else {
                const int R = a.B * a.Hq;
                int r = w.r + 1;
                int len = w.next_len;
                while (len == 0 && r + 1 < R) len = __ldg(a.rlen + (++r));
                enter_row(a, w, r, w.rend, len);
            }
        }
    }
    d.hdr = rows | (flags << 5) | (stage << 8);
    return d;
}

// Page-table lookup of the tile's positions (loaded two steps earlier), and the row's q when the
// tile opens the row.  A position at or past N_b is reported by rows_kernel; here only positions
// inside the page-table row (below max_pages * 16) are looked up.
__device__ __forceinline__ void lookup_pages(const DecodeArgs& a, RowTile& d) {
    const int lane = threadIdx.x & 31;
    const int pos = a.weighted ? (d.v & kPosMask) : d.v;
    if (d.v >= 0 && pos < a.n_cap) d.page = __ldcg(a.page_table + d.pt_off + (pos >> 4));
    if ((d.hdr >> 5) & kFlagFirst) d.q2 = __ldcg(reinterpret_cast<const uint2*>(a.q + (long)d.r * kHeadDim) + lane);
}

// 4-row gather of 128-byte half rows (2-D tensor [cache rows][128 dims], box {64, 1}) into shared
// memory, completing on `bar`.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void* tmap, int x, int r0, int r1, int r2, int r3,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3, %4, %5, %6}], [%7];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
        : "memory");
}

// Maps the tile's positions to cache rows, records the tile in its stage and issues its gathers:
// four four-row copies per 64-dim half of K and of V, issued by lane 0 (the copy takes its tensor
// map and coordinates from one thread).  Rows past the tile's end or without a valid page repeat
// the tile's first mapped row (an L2 hit) and are masked out: every row of the stage holds finite
// data, since a masked row's zero weight still multiplies its V row.
__device__ __forceinline__ void issue_row_tile(const DecodeArgs& a, SparseSmem& ws, uint32_t kv0, const RowTile& d,
                                               const CUtensorMap* kmap, const CUtensorMap* vmap) {
    const int lane = threadIdx.x & 31;
    const int st = (d.hdr >> 8) & (kSparseStages - 1);
    const int rows = d.hdr & 31;
    bool ok = false;
    uint32_t ri = 0;
    if (d.v >= 0) {   // lanes < rows
        if (d.page >= 0 && d.page < a.num_pages) {
            ok = true;
            ri = ((uint32_t)d.page * kPageSize + (uint32_t)(d.v & (kPageSize - 1))) * (uint32_t)a.Hkv + (uint32_t)d.kvh;
            // (the flag bit of a drawn entry lies above the slot bits used here)
        } else {
            report(a.status, SD_ERR_INDEX_OOB);   // a page entry outside the cache, or a position at or past N_b
        }
    }
    const uint32_t okm = __ballot_sync(0xffffffffu, ok);
    const uint32_t drawn = a.weighted ? __ballot_sync(0xffffffffu, ok && (d.v & kSampledFlag)) : 0u;
    if (lane == 0)
        *reinterpret_cast<int4*>(ws.info[st]) =
            make_int4((d.hdr & 0xff) | (int)((okm & 0xffffu) << 16), d.r, d.seg, (int)(drawn & 0xffffu));
    if ((d.hdr >> 5) & kFlagFirst) reinterpret_cast<uint2*>(ws.q[st])[lane] = d.q2;
    if (rows == 0) return;
    const uint32_t sub = okm ? __shfl_sync(0xffffffffu, ri, __ffs(okm) - 1) : 0u;   // every lane takes part
    if (!ok) ri = sub;
    const uint32_t bar = smem_addr(&ws.full[st]);
    if (lane == 0) mbar_arrive_expect_tx(&ws.full[st], (uint32_t)kGatherTile);
    const uint32_t dst = kv0 + (uint32_t)(st * kGatherTile);
#pragma unroll
    for (int gq = 0; gq < kTileRows / 4; ++gq) {
        const int q0 = __shfl_sync(0xffffffffu, (int)ri, 4 * gq + 0);
        const int q1 = __shfl_sync(0xffffffffu, (int)ri, 4 * gq + 1);
        const int q2 = __shfl_sync(0xffffffffu, (int)ri, 4 * gq + 2);
        const int q3 = __shfl_sync(0xffffffffu, (int)ri, 4 * gq + 3);
        if (lane == 0) {
            const uint32_t o = (uint32_t)(gq * 4 * 128);
            tma_gather4(dst + o, kmap, 0, q0, q1, q2, q3, bar);
            tma_gather4(dst + kHalfBlock + o, kmap, 64, q0, q1, q2, q3, bar);
            tma_gather4(dst + 2 * kHalfBlock + o, vmap, 0, q0, q1, q2, q3, bar);
            tma_gather4(dst + 3 * kHalfBlock + o, vmap, 64, q0, q1, q2, q3, bar);
        }
    }
}

// Consumer state of one query head: the online softmax over its selected rows.  In the score MMA q
// is column 0 of the B operand; in the P.V MMA column 0 carries the bf16 high part of the weights
// and column 1 their bf16 residual, so the head's output is the sum of accumulator columns 0 and 1
// (lanes with lane % 4 == 0 hold both).
struct HeadState {
    float lw;           // weighted mode: log2 of the weight of the row's drawn entries
    float m;            // running max of column 0 (log2 units; lanes % 4 == 0)
    float l;            // partial sum of rows g, g + 8 (lanes % 4 == 0)
    float acc[8][4];    // O^T fragments: dims 16 mt + g (+ 8) x columns 2 (lane % 4) (+ 1)
    uint32_t qb[8][2];  // q as column 0 of the B operand
};

__device__ __forceinline__ void reset_head(HeadState& st) {
    st.m = -INFINITY;   // (lw belongs to the row and is set when its first tile is consumed)
    st.l = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) st.acc[mt][0] = st.acc[mt][1] = st.acc[mt][2] = st.acc[mt][3] = 0.f;
}

// q of the row from the stage (staged there when the tile was issued).
__device__ __forceinline__ void load_q_head(const uint32_t* qr, HeadState& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        st.qb[j][0] = g == 0 ? qr[8 * j + c] : 0u;
        st.qb[j][1] = g == 0 ? qr[8 * j + c + 4] : 0u;
    }
}

// One tile: S = K_tile . q (8 MMAs), masked online softmax over the tile's valid rows, O^T += V_tile^T .
// [p_hi, p_lo] (8 MMAs).  `koff` / `voff` are this lane's ldmatrix offsets (row and chunk, swizzled).
__device__ __forceinline__ void compute_row_tile(const DecodeArgs& a, uint32_t tile, uint32_t valid, uint32_t drawn,
                                                 const uint32_t (&koff)[4], const uint32_t (&voff)[4],
                                                 HeadState& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(tile + (uint32_t)((j >> 2) * kHalfBlock) + koff[j & 3], a0, a1, a2, a3);
        if (j & 1) mma_bf16_16816(s2, a0, a1, a2, a3, st.qb[j][0], st.qb[j][1]);
        else mma_bf16_16816(s, a0, a1, a2, a3, st.qb[j][0], st.qb[j][1]);
    }
    // column 0: rows g (s[0]) and g + 8 (s[2]) in lanes with c == 0
    // (a drawn entry's logit is raised by log2 of its weight: its exp is multiplied by the weight)
    const float z0 = ((valid >> g) & 1u) ? (s[0] + s2[0]) * a.scale_log2 + (((drawn >> g) & 1u) ? st.lw : 0.f)
                                         : -INFINITY;
    const float z1 = ((valid >> (g + 8)) & 1u)
                         ? (s[2] + s2[2]) * a.scale_log2 + (((drawn >> (g + 8)) & 1u) ? st.lw : 0.f)
                         : -INFINITY;
    float tm = fmaxf(z0, z1);
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
    const float mo = st.m;
    const float mn = fmaxf(mo, tm);
    const float base = (mn == -INFINITY) ? 0.f : mn;
    const float p0 = fast_exp2(z0 - base), p1 = fast_exp2(z1 - base);
    const float al = (mo == mn || mo == -INFINITY) ? 1.f : fast_exp2(mo - mn);
    st.l = st.l * al + p0 + p1;
    st.m = mn;
    if (__any_sync(0xffffffffu, al != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            st.acc[mt][0] *= al;
            st.acc[mt][1] *= al;
            st.acc[mt][2] *= al;
            st.acc[mt][3] *= al;
        }
    }
    // B operand: lane (g', c') holds rows 2c', 2c'+1 (b0) and 2c'+8, 2c'+9 (b1) of column g';
    // column 0 = bf16(p), column 1 = bf16(p - bf16(p)), the other columns zero.  Row i < 8 of the
    // tile is p0 of lane 4 i, row i + 8 its p1.
    const float pa0 = __shfl_sync(0xffffffffu, p0, 8 * c), pa1 = __shfl_sync(0xffffffffu, p0, 8 * c + 4);
    const float pb0 = __shfl_sync(0xffffffffu, p1, 8 * c), pb1 = __shfl_sync(0xffffffffu, p1, 8 * c + 4);
    const uint32_t h0 = pack_bf16x2(pa0, pa1), h1 = pack_bf16x2(pb0, pb1);
    uint32_t b0 = 0u, b1 = 0u;
    if (g == 0) {
        b0 = h0;
        b1 = h1;
    } else if (g == 1) {
        b0 = pack_bf16x2(pa0 - bf16_lo(h0), pa1 - bf16_hi(h0));
        b1 = pack_bf16x2(pb0 - bf16_lo(h1), pb1 - bf16_hi(h1));
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(tile + (uint32_t)(2 * kHalfBlock + (mt >> 2) * kHalfBlock) + voff[mt & 3], a0, a1, a2, a3);
        mma_bf16_16816(st.acc[mt], a0, a1, a2, a3, b0, b1);
    }
}

// One warp: log-sum-exp merge of the nseg partials of row r (lane l owns dimensions 4l .. 4l+3),
// kMergeBatch partial outputs per lane in flight together.
constexpr int kMergeBatch = 8;
__device__ __forceinline__ void merge_row(const DecodeArgs& a, int r, int nseg) {
    const int lane = threadIdx.x & 31;
    const float2* ml = a.ml + (long)r * a.jmax;
    float M = -INFINITY;
    for (int j0 = 0; j0 < nseg; j0 += 32) {
        float mj = (j0 + lane < nseg) ? __ldcg(ml + j0 + lane).x : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mj = fmaxf(mj, __shfl_xor_sync(0xffffffffu, mj, o));
        M = fmaxf(M, mj);
    }
    float L = 0.f;
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* src = reinterpret_cast<const float4*>(a.acc + (long)r * a.jmax * kHeadDim) + lane;
    for (int j0 = 0; j0 < nseg; j0 += kMergeBatch) {
        float4 x[kMergeBatch];
        float2 v[kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {   // clamped (in-range) loads, all in flight together
            const int j = min(j0 + i, nseg - 1);
            x[i] = __ldcg(src + (long)j * (kHeadDim / 4));
            v[i] = __ldcg(ml + j);
        }
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            const float wj = (j0 + i >= nseg || v[i].x == -INFINITY) ? 0.f : exp2f(v[i].x - M);
            L += wj * v[i].y;
            o4.x += wj * x[i].x;
            o4.y += wj * x[i].y;
            o4.z += wj * x[i].z;
            o4.w += wj * x[i].w;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    reinterpret_cast<float4*>(a.out + (long)r * kHeadDim)[lane] =
        make_float4(o4.x * inv, o4.y * inv, o4.z * inv, o4.w * inv);
}

// End of this warp's segment of row r: a row held by one warp is written out; otherwise the
// partial is stored, its arrival counted, and the last of the row's warps to arrive merges them.
__device__ __forceinline__ void finish_row_segment(const DecodeArgs& a, int r, int j, int nseg, const HeadState& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    float l = st.l;
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    if (nseg == 1) {   // the whole row is this warp's
        if (c == 0) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            float* dst = a.out + (long)r * kHeadDim;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                dst[16 * mt + g] = (st.acc[mt][0] + st.acc[mt][1]) * inv;
                dst[16 * mt + g + 8] = (st.acc[mt][2] + st.acc[mt][3]) * inv;
            }
        }
        return;
    }
    const long slot = (long)r * a.jmax + j;
    if (lane == 0) a.ml[slot] = make_float2(st.m, l);
    if (c == 0) {
        float* dst = a.acc + slot * kHeadDim;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            dst[16 * mt + g] = st.acc[mt][0] + st.acc[mt][1];
            dst[16 * mt + g + 8] = st.acc[mt][2] + st.acc[mt][3];
        }
    }
    __threadfence();   // this partial is visible before the arrival is counted
    __syncwarp();
    int old = 0;
    if (lane == 0) old = atomicAdd(a.arrive + r, 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != nseg - 1) return;
    __threadfence();   // every other partial of the row is visible
    merge_row(a, r, nseg);
}

template <bool kOrder>
__global__ void __launch_bounds__(32) sparse_decode_kernel(DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SparseSmem& ws = *reinterpret_cast<SparseSmem*>(
        smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u));   // 1024-byte aligned (swizzle atoms)
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kSparseStages; ++s) mbar_init(&ws.full[s], 1);
        mbar_fence_init();
    }
    __syncwarp();
    pdl_launch_dependents();

    const int R = a.B * a.Hq;
    RowWalker w;
    w.seq = 0;
    // this lane's ldmatrix offsets inside a 2 KB half block: K (A operand, rows 8 (lane>>3 & 1) +
    // (lane & 7), chunk 2 (j & 3) + (lane >> 4)) and V (A operand transposed, rows 8 (lane >> 4) +
    // (lane & 7), chunk 2 (mt & 3) + (lane >> 3 & 1)), each chunk swizzled by the row's low 3 bits
    uint32_t koff[4], voff[4];
    {
        const int rk = (((lane >> 3) & 1) << 3) + (lane & 7), rv = ((lane >> 4) << 3) + (lane & 7);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            koff[jj] = (uint32_t)(rk * 128 + (((2 * jj + (lane >> 4)) ^ (lane & 7)) << 4));
            voff[jj] = (uint32_t)(rv * 128 + (((2 * jj + ((lane >> 3) & 1)) ^ (lane & 7)) << 4));
        }
    }
    const uint32_t kv0 = smem_addr(ws.kv);
    RowTile dA, dB, dC;   // the pipeline's tile records (see the main loop)
    auto start_pipeline = [&]() {
        dA = next_row_tile<kOrder>(a, w);
        dB = next_row_tile<kOrder>(a, w);
        dC = next_row_tile<kOrder>(a, w);
        lookup_pages(a, dA);
        issue_row_tile(a, ws, kv0, dA, &kmap, &vmap);   // the walk's first tile
        dA = dB;
        dB = dC;
        dC = next_row_tile<kOrder>(a, w);
        lookup_pages(a, dA);
    };
    // Speculative start on the split that holds when every row has k_max entries (the indexer's
    // rows, the common case): the first tile is gathered while rows_kernel still runs.  After the
    // wait, the true entry count decides: equal to R * k_max, the split is the same and the walk
    // goes on; otherwise the speculative tile is drained and the walk restarts on the row lengths.
    const long e_full = (long)R * a.k_max;   // < 2^31 (checked on the host)
    w.full = true;
    w.epw = max(a.min_epw, (int)((e_full + a.total_warps - 1) / a.total_warps));
    if (kOrder) {
        w.o_lane = (int)((uint64_t)lane * (uint64_t)a.k_max % (uint64_t)w.epw);
        w.o_step = (int)(32ull * (uint64_t)a.k_max % (uint64_t)w.epw);
    }
    const bool spec = (long)blockIdx.x * w.epw < e_full;
    if (spec) {
        w.e = (int)blockIdx.x * w.epw;
        w.e_end = (int)min(e_full, (long)w.e + w.epw);
        const int slot = w.e / a.k_max;
        enter_row(a, w, row_of_slot<kOrder>(a, w, slot), slot * a.k_max, a.k_max);
        start_pipeline();
    }
    pdl_wait();   // rows_kernel: row lengths, checks, zeroed arrival counters
    // E = all entries: the length sums of the rows_kernel CTAs, each lane summing kPrologue
    // consecutive ones per round
    int E = 0;
    for (int base = 0; base < a.nb; base += 32 * kPrologue) {
        const int k0 = base + kPrologue * lane;
#pragma unroll
        for (int i = 0; i < kPrologue; ++i) E += k0 + i < a.nb ? __ldg(a.bsum + k0 + i) : 0;
    }
    E = __reduce_add_sync(0xffffffffu, E);
    int t = 0;   // the tile the main loop consumes first
    // A speculative tile that is not used is left to complete while the walk restarts at tile 1;
    // stage 0 is waited for before its next use or before the warp exits.
    bool spec_pending = false;
    auto drain_spec = [&]() -> bool {
        if (!spec_pending) return true;
        spec_pending = false;
        const bool done = __all_sync(0xffffffffu, mbar_wait(&ws.full[0], 0u));
        if (!done && lane == 0) report(a.status, SD_ERR_TIMEOUT);
        return done;
    };
    if (!(spec && E == e_full)) {
        if (spec) {
            spec_pending = true;
            t = 1;
        }
        if (E == 0) {
            drain_spec();
            return;
        }
        w.full = false;
        w.epw = max(a.min_epw, (int)(((long)E + a.total_warps - 1) / a.total_warps));
        const long e0 = (long)blockIdx.x * w.epw;
        if (e0 >= E) {
            drain_spec();
            return;
        }
        w.e = (int)e0;
        w.e_end = (int)min((long)E, e0 + w.epw);
        // the rows_kernel CTA whose rows hold entry w.e: one scan of the lanes' sums per round (the
        // sums are in L1 now), then the lane that holds it walks its kPrologue sums
        int blk = -1, blk0 = 0, blen = 0;
        {
            int acc = 0;
            for (int base = 0; base < a.nb && blk < 0; base += 32 * kPrologue) {
                const int k0 = base + kPrologue * lane;
                int v[kPrologue], sum = 0;
#pragma unroll
                for (int i = 0; i < kPrologue; ++i) {
                    v[i] = k0 + i < a.nb ? __ldg(a.bsum + k0 + i) : 0;
                    sum += v[i];
                }
                const int incl = warp_inclusive_scan(sum);
                const uint32_t hit = __ballot_sync(0xffffffffu, acc + incl > w.e);
                if (hit != 0u) {
                    const int l = __ffs(hit) - 1;
                    int c = acc + incl - sum, kb = -1, kb0 = 0, kl = 0;   // lane l: its sums in order
#pragma unroll
                    for (int i = 0; i < kPrologue; ++i) {
                        if (kb < 0 && c + v[i] > w.e) {
                            kb = k0 + i;
                            kb0 = c;
                            kl = v[i];
                        }
                        c += v[i];
                    }
                    blk = __shfl_sync(0xffffffffu, kb, l);
                    blk0 = __shfl_sync(0xffffffffu, kb0, l);
                    blen = __shfl_sync(0xffffffffu, kl, l);
                }
                acc += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (blk < 0) {   // not reached: w.e < E
            drain_spec();
            return;
        }
        if (a.rpc == 1) {      // one row per CTA of the row pass
            enter_row(a, w, blk, blk0, blen);
        } else {
            const int r0 = blk * a.rpc;
            const int v = (lane < a.rpc && r0 + lane < R) ? __ldg(a.rlen + r0 + lane) : 0;
            const int incl = warp_inclusive_scan(v);
            const uint32_t hit = __ballot_sync(0xffffffffu, blk0 + incl > w.e);
            if (hit == 0u) {   // not reached: the CTA's rows hold entry w.e
                drain_spec();
                return;
            }
            const int l = __ffs(hit) - 1;
            enter_row(a, w, r0 + l, blk0 + __shfl_sync(0xffffffffu, incl - v, l), __shfl_sync(0xffffffffu, v, l));
        }
        w.seq = t;
        start_pipeline();
    }
    // Software pipeline over tiles, so that no load but the gather itself is waited for: while tile
    // t is consumed, tile t + 1 is gathered (its pages were looked up a step earlier), the pages of
    // tile t + 2 are looked up (its positions were loaded two steps earlier) and the positions of
    // tile t + 4 are loaded.  (Each page lookup follows the rotation of the records, so that no
    // record is copied while a load into it is in flight: such a register copy would wait for the
    // load.)
    static_assert(kSparseStages == 2, "the pipeline gathers one tile ahead");
    HeadState st;
    reset_head(st);
    st.lw = 0.f;
    bool ok = true;
    for (;; ++t) {
        const int stage = t & (kSparseStages - 1);
        if (spec_pending && ((dA.hdr >> 8) & (kSparseStages - 1)) == 0 && !drain_spec()) {
            ok = false;
            break;
        }
        issue_row_tile(a, ws, kv0, dA, &kmap, &vmap);   // into the stage tile t - 1 used
        dA = dB;
        dB = dC;
        dC = next_row_tile<kOrder>(a, w);
        lookup_pages(a, dA);
        __syncwarp();
        const int4 info = *reinterpret_cast<const int4*>(ws.info[stage]);
        const int flags = (info.x >> 5) & 7;
        if (flags & kFlagEnd) break;
        if (flags & kFlagFirst) {
            load_q_head(ws.q[stage], st);
            st.lw = a.weighted ? __ldcg(a.rlw + info.y) : 0.f;
        }
        ok = mbar_wait(&ws.full[stage], (uint32_t)((t / kSparseStages) & 1));
        ok = __all_sync(0xffffffffu, ok);   // warp-uniform before the collective ops below
        if (!ok) break;
        compute_row_tile(a, kv0 + (uint32_t)(stage * kGatherTile), (uint32_t)info.x >> 16, (uint32_t)info.w, koff,
                         voff, st);
        if (flags & kFlagLast) {
            finish_row_segment(a, info.y, info.z & 0xffff, info.z >> 16, st);
            reset_head(st);
        }
        __syncwarp();   // every lane has read the stage before it is refilled
    }
    drain_spec();
    if (!ok) {
        // A copy never completed: record it, wait (bounded) for this warp's copies still in
        // flight, and return; the rows this warp held are left unwritten.
        if (lane == 0) report(a.status, SD_ERR_TIMEOUT);
        for (int u = t; u < t + kSparseStages; ++u) {
            const int hdr = ws.info[u % kSparseStages][0];
            if ((hdr & 31) > 0) mbar_wait(&ws.full[u % kSparseStages], (uint32_t)((u / kSparseStages) & 1));
        }
    }
}

// ---------------------------------------------------------------------------------------------
// dense decode: ranges_kernel, dense_decode_kernel, merge_kernel
// ---------------------------------------------------------------------------------------------
// Dense decode: the row count of each range (every position below N_b is a row).
__global__ void __launch_bounds__(256) ranges_kernel(DecodeArgs a) {
    pdl_enter();
    const int ri = blockIdx.x * blockDim.x + threadIdx.x;
    if (ri >= a.nrt) return;
    const int grp = ri / a.nrp, rloc = ri - grp * a.nrp;
    const int n = checked_len(a.lens, grp / a.Hkv, a.n_cap, a.status);
    const int lo = rloc * kRange;
    a.counts[ri] = lo < n ? min(kRange, n - lo) : 0;
}

// ---------------------------------------------------------------------------------------------
// sparse decode over GQA groups: union_masks_kernel
// ---------------------------------------------------------------------------------------------
// First index j of an idx row (ascending positions, then negative padding) whose position is at
// least `target` (len if none): a 32-way search by one warp, every probe of a round in flight
// together.  Negative entries count as past every position.
__device__ __forceinline__ int first_at_least(const int32_t* row, int len, int target) {
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = len;   // the answer lies in [lo, hi]
    while (hi - lo > 32) {
        const int step = (hi - lo + 31) / 32;
        const int x = min(lo + (lane + 1) * step - 1, hi - 1);
        const int v = __ldg(row + x);
        const uint32_t ge = __ballot_sync(0xffffffffu, v < 0 || v >= target);
        if (ge == 0u) {
            lo = min(lo + 32 * step, hi);   // past the last probe (which is hi - 1)
        } else {
            const int f = __ffs(ge) - 1;
            const int xf = min(lo + (f + 1) * step - 1, hi - 1);
            lo = f == 0 ? lo : min(lo + f * step, hi);
            hi = xf;
        }
    }
    const int x = lo + lane;
    const int v = x < hi ? __ldg(row + x) : 0;
    const uint32_t ge = __ballot_sync(0xffffffffu, x < hi && (v < 0 || v >= target));
    return ge ? lo + __ffs(ge) - 1 : hi;
}

// The group walk's check of idx: every rule a row must follow is one on adjacent entries (positions
// ascending, below N_b, no position after the first negative entry), so the rows are cut into chunks of
// kValidateEntries consecutive entries, one thread each, over the whole grid (no per-row reduction:
// the group walk needs no row lengths).  A chunk whose start is 16-byte aligned is loaded as vectors.
constexpr int kValidateEntries = 16;
__global__ void __launch_bounds__(256) validate_kernel(DecodeArgs a) {
    pdl_enter();
    const long per_row = (a.k_max + kValidateEntries - 1) / kValidateEntries;
    const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long r = t / per_row;
    if (r >= (long)a.B * a.Hq) return;
    const int j0 = (int)(t - r * per_row) * kValidateEntries;
    const int32_t* row = a.idx + r * a.k_max;
    const int n = checked_len(a.lens, (int)(r / a.Hq), a.n_cap, a.status);
    int v[kValidateEntries];
    const int cnt = min(kValidateEntries, a.k_max - j0);
    if (cnt == kValidateEntries && (reinterpret_cast<uintptr_t>(row + j0) & 15u) == 0) {
#pragma unroll
        for (int i = 0; i < kValidateEntries / 4; ++i) {
            const int4 q = __ldg(reinterpret_cast<const int4*>(row + j0) + i);
            v[4 * i] = q.x;
            v[4 * i + 1] = q.y;
            v[4 * i + 2] = q.z;
            v[4 * i + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < kValidateEntries; ++i) v[i] = i < cnt ? __ldg(row + j0 + i) : -1;
    }
    int p = j0 > 0 ? __ldg(row + j0 - 1) : -1;
    bool oob = false, order = false;
#pragma unroll
    for (int i = 0; i < kValidateEntries; ++i) {
        if (i < cnt && v[i] >= 0) {
            oob |= v[i] >= n;
            order |= (j0 + i > 0) && (p < 0 || p >= v[i]);
        }
        p = v[i];
    }
    if (oob) report(a.status, SD_ERR_INDEX_OOB);
    else if (order) report(a.status, SD_ERR_ORDER);
}

// One CTA per (group, kRange-position range): the heads of the group that selected each position,
// as bits of a per-position mask (MT: 8 bits for G <= 8, 16 for G <= 16) in the workspace, and the
// range's position count (the unit the group walk is split in).  Each warp finds a head's entries
// in the range by a 32-way search of its idx row and sets their bits in shared memory.
template <typename MT>
__global__ void __launch_bounds__(256) union_masks_kernel(DecodeArgs a) {
    constexpr int kPer = 4 / (int)sizeof(MT);            // masks per 32-bit word
    __shared__ uint32_t m[kRange / kPer];
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ri = blockIdx.x;
    const int grp = ri / a.nrp, rloc = ri - grp * a.nrp;
    const int b = grp / a.Hkv, kvh = grp - b * a.Hkv;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int r0 = rloc * kRange, r1 = min(n, r0 + kRange);
    if (tid == 0) a.counts[ri] = r1 > r0 ? r1 - r0 : 0;
    if (r0 >= r1) return;
    for (int i = tid; i < kRange / kPer; i += blockDim.x) m[i] = 0u;
    __syncthreads();
    for (int g = warp; g < a.G; g += (int)(blockDim.x >> 5)) {
        const int32_t* row = a.idx + ((long)b * a.Hq + (long)kvh * a.G + g) * a.k_max;
        const int lo = first_at_least(row, a.k_max, r0);
        const int hi = first_at_least(row, a.k_max, r1);
        if (hi - lo == r1 - r0) {
            // every position of the range (strictly ascending entries in [r0, r1)): the head's bit in
            // every mask, one word per lane
            uint32_t rep = 0u;
#pragma unroll
            for (int i = 0; i < kPer; ++i) rep |= (1u << g) << (8 * (int)sizeof(MT) * i);
            const int words = (r1 - r0 + kPer - 1) / kPer;
            for (int i = lane; i < words; i += 32) {
                const int pl = (i + 1) * kPer - (r1 - r0);   // positions of the last word past r1
                atomicOr(&m[i], pl > 0 ? rep & (0xffffffffu >> (8 * (int)sizeof(MT) * pl)) : rep);
            }
            continue;
        }
        for (int j = lo + lane; j < hi; j += 32) {
            const int p = __ldg(row + j) - r0;
            if (p >= 0 && p < r1 - r0)   // (an unsorted row is reported by rows_kernel)
                atomicOr(&m[p / kPer], (1u << g) << (8 * (int)sizeof(MT) * (p % kPer)));
        }
    }
    __syncthreads();
    // positions r0 .. r1 - 1 of the group's masks (rounded up to 16 bytes: still inside the group's
    // row, whose length max_pages * 16 is a multiple of 16)
    uint4* dst = reinterpret_cast<uint4*>(a.umask + ((long)grp * a.n_cap + r0) * (long)sizeof(MT));
    const int nvec = ((r1 - r0) * (int)sizeof(MT) + 15) / 16;
    for (int i = tid; i < nvec; i += blockDim.x) dst[i] = reinterpret_cast<const uint4*>(m)[i];
}

// The warp's walk over its rows (all fields warp-uniform).
struct GroupWalker {
    int e, e_end;     // next global row and the end of this warp's share
    int ri, off;      // range holding row e, and e's offset in it
    int cnt;          // rows in range ri
    int grp;          // group (b * Hkv + kvh) of the current segment
    int seg_j;        // segment slot of the current segment
    bool seg_new;     // the next tile opens a segment
    int epw;          // rows per warp
    // group walk over selected positions: this lane's head mask in the 32-position window (aligned
    // within range ri) at offset win, and in the window after it, loaded one window ahead
    int win, nwin;    // window offsets in range ri (-1: none)
    uint32_t wmk, nmk;
};

// The next non-empty range after ri (one exists while rows remain; at the last range *cnt = 0).
__device__ __forceinline__ int next_range(const DecodeArgs& a, int ri, int* cnt) {
    int c = 0;
    while (ri + 1 < a.nrt) {
        c = __ldg(a.counts + (++ri));
        if (c != 0) break;
    }
    *cnt = c;
    return ri;
}

// The next tile of a group walk.  Dense: the next 16 positions, every head.  Union (kUnion): the
// walk still advances over positions, but a tile takes only the positions some head of the group
// selected (mask != 0, 32 positions examined per round), each with its heads' mask.
template <int NT, bool kUnion>
__device__ __forceinline__ TileDesc prefetch_group_tile(const DecodeArgs& a, GroupWalker& w) {
    const int lane = threadIdx.x & 31;
    TileDesc d = empty_tile();
    if (w.e >= w.e_end) {
        d.flags = kFlagEnd;
        return d;
    }
    const int grp = w.grp;
    const int b = grp / a.Hkv, kvh = grp - b * a.Hkv;
    d.owner = grp;
    d.seg_j = w.seg_j;
    if (w.seg_new) d.flags |= kFlagFirst;
    w.seg_new = false;
    const uint32_t full_mask = (1u << a.G) - 1u;
    int filled = 0;
    while (filled < kTileRows && w.e < w.e_end) {
        if (w.off == w.cnt) {   // next non-empty range; stop at a group boundary
            int c;
            const int ri = next_range(a, w.ri, &c);
            if (ri / a.nrp != grp) break;
            w.ri = ri;
            w.off = 0;
            w.cnt = c;
            w.win = w.nwin = -1;
        }
        using MT = typename std::conditional<NT == 1, uint8_t, uint16_t>::type;
        const MT* gm = kUnion ? reinterpret_cast<const MT*>(a.umask) + (long)grp * a.n_cap +
                                    (long)(w.ri - grp * a.nrp) * kRange   // the masks of range ri
                              : nullptr;
        if (kUnion && !a.union_tiles) {
            const int wo = w.off & ~31;
            if (w.win != wo) {   // enter the window: from the prefetch, else loaded now
                w.wmk = (w.nwin == wo) ? w.nmk : (wo + lane < w.cnt ? (uint32_t)__ldg(gm + wo + lane) : 0u);
                w.win = wo;
                w.nwin = wo + 32 < w.cnt ? wo + 32 : -1;
                w.nmk = (w.nwin >= 0 && w.nwin + lane < w.cnt) ? (uint32_t)__ldg(gm + w.nwin + lane) : 0u;
            }
            // positions w.off .. limit - 1 of this window are examined
            const int limit = min(min(wo + 32, w.cnt), w.off + (w.e_end - w.e));
            if (limit <= w.off) {   // not reached (counts are consistent); ends the walk
                w.e = w.e_end;
                break;
            }
            const int at = wo + lane;
            uint32_t take = __ballot_sync(0xffffffffu, at >= w.off && at < limit && w.wmk != 0u);
            int consumed = limit - w.off;
            const int need = kTileRows - filled;
            // one run of selected positions (a window the group selected in full): the i-th selected
            // position is the run's start + i, no bit search needed
            const int low = __ffs(take) - 1;
            const bool run = take != 0u && ((take + (1u << low)) & take) == 0u;
            if (__popc(take) > need) {   // the tile fills up: stop after the need-th selected position
                const int last = run ? low + need - 1 : (int)__fns(take, 0, need);
                take &= last == 31 ? 0xffffffffu : ((2u << last) - 1u);
                consumed = wo + last + 1 - w.off;
            }
            const int cnt = __popc(take);
            const bool mine = lane >= filled && lane < filled + cnt;
            const int src = mine ? (run ? low + lane - filled : (int)__fns(take, 0, lane - filled + 1)) : 0;
            const uint32_t msrc = __shfl_sync(0xffffffffu, w.wmk, src);
            if (mine) {
                const int p = (w.ri - grp * a.nrp) * kRange + wo + src;
                d.page = __ldg(a.page_table + (long)b * a.max_pages + p / kPageSize);
                d.sub = (uint32_t)(p & (kPageSize - 1)) * (uint32_t)a.Hkv + kvh;
                d.mask = msrc;
            }
            filled += cnt;
            w.off += consumed;
            w.e += consumed;
            continue;
        }
        const int take = min(min(kTileRows - filled, w.cnt - w.off), w.e_end - w.e);
        if (take <= 0) {   // not reached (counts are consistent); ends the walk
            w.e = w.e_end;
            break;
        }
        if (lane >= filled && lane < filled + take) {
            const int off = w.off + lane - filled;
            const int p = (w.ri - grp * a.nrp) * kRange + off;
            if (kUnion) {
                // group walk in whole tiles (the union covers nearly every position): a position no head
                // selected (mask 0) is not gathered -- zero-filled and masked for every head
                d.page = __ldg(a.page_table + (long)b * a.max_pages + p / kPageSize);
                d.sub = (uint32_t)(p & (kPageSize - 1)) * (uint32_t)a.Hkv + kvh;
                d.mask = (uint32_t)__ldg(gm + off);
            } else {
                const int page = __ldg(a.page_table + (long)b * a.max_pages + p / kPageSize);
                if (page < 0 || page >= a.num_pages) {
                    report(a.status, SD_ERR_INDEX_OOB);
                    d.row_idx = kNoRow;
                } else {
                    d.row_idx =
                        ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + kvh;
                }
                d.mask = full_mask;
            }
        }
        filled += take;
        w.off += take;
        w.e += take;
    }
    d.rows = filled;
    // does the segment end here?
    bool last = w.e >= w.e_end;
    if (!last && w.off == w.cnt) {
        int c;
        const int ri = next_range(a, w.ri, &c);
        if (ri / a.nrp != grp) {
            last = true;
            w.ri = ri;   // the next segment starts in range ri
            w.off = 0;
            w.cnt = c;
            w.win = w.nwin = -1;
            w.grp = ri / a.nrp;
            w.seg_j = (int)(blockIdx.x - w.e / w.epw);   // w.e is the first row of the new group
            w.seg_new = true;
        }
    }
    if (last) d.flags |= kFlagLast;
    return d;
}

template <int NT>
__device__ __forceinline__ void load_q_group(const DecodeArgs& a, int b, int kvh, Softmax<NT>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + g;
        const bool ok = hh < a.G;
        const uint32_t* qr =
            reinterpret_cast<const uint32_t*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + (ok ? hh : 0)) * kHeadDim);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            st.qb[nt][j][0] = ok ? __ldg(qr + 8 * j + c) : 0u;
            st.qb[nt][j][1] = ok ? __ldg(qr + 8 * j + c + 4) : 0u;
        }
    }
}

template <int NT>
__device__ __forceinline__ void flush_group(const DecodeArgs& a, int b, int kvh, int seg_j, Softmax<NT>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = st.l[nt][e];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            const int hh = nt * 8 + 2 * c + e;
            if (hh < a.G) {
                const long slot = ((long)b * a.Hq + (long)kvh * a.G + hh) * a.jmax + seg_j;
                if (g == 0) a.ml[slot] = make_float2(st.m[nt][e], l);
                float* dst = a.acc + slot * kHeadDim;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    dst[16 * mt + g] = st.acc[nt][mt][e];
                    dst[16 * mt + g + 8] = st.acc[nt][mt][2 + e];
                }
            }
        }
    }
}

// Sum of the range counts [lo, hi), kPrologue loads per lane in flight (warp-uniform result).
__device__ __forceinline__ int sum_counts(const DecodeArgs& a, int lo, int hi) {
    const int lane = threadIdx.x & 31;
    int s = 0;
    for (int base = lo; base < hi; base += 32 * kPrologue) {
        int v[kPrologue];
#pragma unroll
        for (int i = 0; i < kPrologue; ++i) {
            const int k = base + 32 * i + lane;
            v[i] = k < hi ? __ldg(a.counts + k) : 0;
        }
#pragma unroll
        for (int i = 0; i < kPrologue; ++i) s += v[i];
    }
    return __reduce_add_sync(0xffffffffu, s);
}

template <int NT, bool kUnion>
__global__ void __launch_bounds__(32) dense_decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    DecodeSmem& ws = *reinterpret_cast<DecodeSmem*>(smem);
    pdl_enter();

    const int lane = threadIdx.x & 31;
    const int E = sum_counts(a, 0, a.nrt);
    if (E == 0) return;
    GroupWalker w;
    w.epw = max(1, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    const long e0 = (long)blockIdx.x * w.epw;
    if (e0 >= E) return;
    w.e = (int)e0;
    w.e_end = (int)min((long)E, e0 + w.epw);
    // the range holding row w.e (prefix over the counts, kPrologue loads per lane in flight)
    int ri = -1, ri0 = 0;
    {
        int acc = 0;
        for (int base = 0; base < a.nrt && ri < 0; base += 32 * kPrologue) {
            int v[kPrologue];
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int k = base + 32 * i + lane;
                v[i] = k < a.nrt ? __ldg(a.counts + k) : 0;
            }
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int incl = warp_inclusive_scan(v[i]);
                const uint32_t hit = __ballot_sync(0xffffffffu, acc + incl > w.e);
                if (ri < 0 && hit != 0u) {
                    const int l = __ffs(hit) - 1;
                    ri = base + 32 * i + l;
                    ri0 = acc + __shfl_sync(0xffffffffu, incl - v[i], l);
                }
                acc += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
    }
    if (ri < 0) return;   // not reached: w.e < E
    w.ri = ri;
    w.off = w.e - ri0;
    w.cnt = __ldg(a.counts + ri);
    w.grp = ri / a.nrp;
    w.win = w.nwin = -1;
    w.wmk = w.nmk = 0u;
    const int e0grp = ri0 - sum_counts(a, w.grp * a.nrp, ri);   // first row of the group
    w.seg_j = (int)(blockIdx.x - e0grp / w.epw);
    w.seg_new = true;

    Softmax<NT> st;
    reset_state(st);
    TileDesc next = prefetch_group_tile<NT, kUnion>(a, w);
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue_tile<kUnion>(a, ws, s, next);
        next = prefetch_group_tile<NT, kUnion>(a, w);
    }
    for (int t = 0;; ++t) {
        const int stage = t % kStages;
        // the stage of tile t-1 is free: issue tile t+kStages-1 before waiting for tile t
        issue_tile<kUnion>(a, ws, (t + kStages - 1) % kStages, next);
        next = prefetch_group_tile<NT, kUnion>(a, w);
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int rows = ws.info[stage][0], flags = ws.info[stage][1];
        if (flags & kFlagEnd) break;
        const int grp = ws.info[stage][2], tj = ws.info[stage][3];
        const int tb = grp / a.Hkv, tkvh = grp - tb * a.Hkv;
        if (flags & kFlagFirst) load_q_group(a, tb, tkvh, st);
        if (rows > 0) compute_tile(a, ws, stage, st);
        if (flags & kFlagLast) {
            flush_group(a, tb, tkvh, tj, st);
            reset_state(st);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------------------------
// dense decode: merge_kernel
// ---------------------------------------------------------------------------------------------
constexpr int kMergeWarps = 4;
constexpr int kMergeLoads = 16;   // partials per lane whose loads are in flight together

// One CTA of kMergeWarps warps per (b, h): log-sum-exp merge of the partials of the segments of its
// group.  Every thread takes segments t, t + 128, ... for the maxima and weights; warp w then sums the
// outputs of segments w, w + kMergeWarps, ... (lane l owns dimensions 4l .. 4l+3), and the warps' sums
// are added in shared memory.
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(DecodeArgs a) {
    __shared__ float s_red[kMergeWarps];
    __shared__ float4 s_o[kMergeWarps][32];
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
    const int grp = b * a.Hkv + h / a.G;
    // all rows, the rows of the groups before this one and this group's rows, in one pass over the counts
    int E = 0, e0 = 0, eg = 0;
    {
        const int g0 = grp * a.nrp, g1 = g0 + a.nrp;
        for (int base = 0; base < a.nrt; base += 32 * kPrologue) {
            int v[kPrologue];
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int k = base + 32 * i + lane;
                v[i] = k < a.nrt ? __ldg(a.counts + k) : 0;
            }
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int k = base + 32 * i + lane;
                E += v[i];
                e0 += k < g0 ? v[i] : 0;
                eg += (k >= g0 && k < g1) ? v[i] : 0;
            }
        }
        E = __reduce_add_sync(0xffffffffu, E);
        e0 = __reduce_add_sync(0xffffffffu, e0);
        eg = __reduce_add_sync(0xffffffffu, eg);
    }
    const int e1 = e0 + eg;
    const int epw = max(1, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    const int nseg = (e1 > e0) ? ((e1 - 1) / epw - e0 / epw + 1) : 0;
    const float2* ml = a.ml + bh * a.jmax;
    // M = max over the segments' maxima
    float mx = -INFINITY;
    for (int j = tid; j < nseg; j += blockDim.x) mx = fmaxf(mx, ml[j].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    float M = s_red[0];
#pragma unroll
    for (int w = 1; w < kMergeWarps; ++w) M = fmaxf(M, s_red[w]);
    __syncthreads();
    // warp `warp` sums segments warp, warp + kMergeWarps, ...
    float L = 0.f;
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* src = reinterpret_cast<const float4*>(a.acc + bh * a.jmax * kHeadDim) + lane;
    for (int j0 = warp; j0 < nseg; j0 += kMergeWarps * kMergeLoads) {
        float4 x[kMergeLoads];
        float2 v[kMergeLoads];
#pragma unroll
        for (int i = 0; i < kMergeLoads; ++i) {   // unconditional (clamped) loads, all in flight together
            const int j = min(j0 + i * kMergeWarps, nseg - 1);
            x[i] = __ldg(src + (long)j * (kHeadDim / 4));
            v[i] = __ldg(ml + j);
        }
#pragma unroll
        for (int i = 0; i < kMergeLoads; ++i) {
            const bool live = j0 + i * kMergeWarps < nseg;
            const float wj = (!live || v[i].x == -INFINITY) ? 0.f : exp2f(v[i].x - M);
            L += wj * v[i].y;
            o4.x += wj * x[i].x;
            o4.y += wj * x[i].y;
            o4.z += wj * x[i].z;
            o4.w += wj * x[i].w;
        }
    }
    s_o[warp][lane] = o4;
    if (lane == 0) s_red[warp] = L;
    __syncthreads();
    if (warp == 0) {
        float Lt = 0.f;
        float4 ot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) {
            Lt += s_red[w];
            ot.x += s_o[w][lane].x;
            ot.y += s_o[w][lane].y;
            ot.z += s_o[w][lane].z;
            ot.w += s_o[w][lane].w;
        }
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        reinterpret_cast<float4*>(a.out + bh * kHeadDim)[lane] = make_float4(ot.x * inv, ot.y * inv, ot.z * inv, ot.w * inv);
    }
}

// ---------------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------------
template <typename K>
static cudaError_t occupancy_of(K kernel, int* ctas) {
    const size_t smem = decode_smem();
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, kernel, 32, smem);
}

cudaError_t decode_occupancy(bool dense, int G, int* ctas_per_sm) {
    if (!dense) {
        const size_t smem = sparse_decode_smem();
        cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(sparse_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int ordered = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ordered, sparse_decode_kernel<true>, 32, smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, sparse_decode_kernel<false>, 32, smem);
        if (e == cudaSuccess && ordered < *ctas_per_sm) *ctas_per_sm = ordered;
        return e;
    }
    // (the group walk over selected positions runs with the same shared memory and occupancy)
    int union_ctas = 0;
    cudaError_t e = G <= 8 ? occupancy_of(dense_decode_kernel<1, true>, &union_ctas)
                           : occupancy_of(dense_decode_kernel<2, true>, &union_ctas);
    if (e != cudaSuccess) return e;
    e = G <= 8 ? occupancy_of(dense_decode_kernel<1, false>, ctas_per_sm)
               : occupancy_of(dense_decode_kernel<2, false>, ctas_per_sm);
    if (e == cudaSuccess && union_ctas < *ctas_per_sm) *ctas_per_sm = union_ctas;
    return e;
}

namespace {

// The K and V caches as 2-D tensors [num_pages * 16 * Hkv cache rows][128 dims] for the row
// gathers: box {64 dims, 1 row}, 128-byte swizzle.  Encoded on the host through the driver entry
// point, and kept for the last (device, K, V, rows).
struct RowMapCache {
    std::mutex mu;
    PFN_cuTensorMapEncodeTiled encode = nullptr;
    int dev = -1;
    const void* K = nullptr;
    const void* V = nullptr;
    long rows = 0;
    CUtensorMap kmap, vmap;
};
RowMapCache g_rowmap;

CUresult encode_rows(PFN_cuTensorMapEncodeTiled encode, CUtensorMap* m, const void* base, long rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

cudaError_t row_tensor_maps(const DecodeArgs& a, CUtensorMap* kmap, CUtensorMap* vmap) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const long rows = (long)a.num_pages * kPageSize * a.Hkv;
    std::lock_guard<std::mutex> lock(g_rowmap.mu);
    if (g_rowmap.encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
        g_rowmap.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
    }
    if (g_rowmap.dev != dev || g_rowmap.K != a.K || g_rowmap.V != a.V || g_rowmap.rows != rows) {
        if (encode_rows(g_rowmap.encode, &g_rowmap.kmap, a.K, rows) != CUDA_SUCCESS ||
            encode_rows(g_rowmap.encode, &g_rowmap.vmap, a.V, rows) != CUDA_SUCCESS) {
            g_rowmap.dev = -1;
            return cudaErrorInvalidValue;
        }
        g_rowmap.dev = dev;
        g_rowmap.K = a.K;
        g_rowmap.V = a.V;
        g_rowmap.rows = rows;
    }
    *kmap = g_rowmap.kmap;
    *vmap = g_rowmap.vmap;
    return cudaSuccess;
}

}  // namespace

// The row pass: rows longer than two passes of the CTA's threads keep four passes of loads in flight.
cudaError_t launch_rows(const DecodeArgs& a, cudaStream_t stream) {
    const bool deep = (long)a.k_max > 2L * a.tpr * kRowBatch;
    return deep ? launch_pdl(rows_kernel<4>, dim3(a.nb), dim3(a.tpr * a.rpc), 0, stream, a)
                : launch_pdl(rows_kernel<1>, dim3(a.nb), dim3(a.tpr * a.rpc), 0, stream, a);
}

cudaError_t launch_sparse(const DecodeArgs& a, cudaStream_t stream) {
    CUtensorMap kmap, vmap;
    cudaError_t e = row_tensor_maps(a, &kmap, &vmap);
    if (e != cudaSuccess) return e;
    e = launch_rows(a, stream);
    if (e != cudaSuccess) return e;
    e = a.order_rows
            ? launch_pdl(sparse_decode_kernel<true>, dim3(a.total_warps), dim3(32), sparse_decode_smem(), stream, a, kmap, vmap)
            : launch_pdl(sparse_decode_kernel<false>, dim3(a.total_warps), dim3(32), sparse_decode_smem(), stream, a, kmap,
                         vmap);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Sparse decode over GQA groups (rows many heads of a group share): the checks of idx, the groups'
// selection masks, the group walk over the selected positions, the merge of the segments.
cudaError_t launch_sparse_union(const DecodeArgs& a, cudaStream_t stream) {
    const long chunks = (long)a.B * a.Hq * ((a.k_max + kValidateEntries - 1) / kValidateEntries);
    cudaError_t e = launch_pdl(validate_kernel, dim3((unsigned)((chunks + 255) / 256)), dim3(256), 0, stream, a);
    if (e != cudaSuccess) return e;
    e = a.G <= 8 ? launch_pdl(union_masks_kernel<uint8_t>, dim3((unsigned)a.nrt), dim3(256), 0, stream, a)
                 : launch_pdl(union_masks_kernel<uint16_t>, dim3((unsigned)a.nrt), dim3(256), 0, stream, a);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.total_warps), block(32);
    e = a.G <= 8 ? launch_pdl(dense_decode_kernel<1, true>, grid, block, decode_smem(), stream, a)
                 : launch_pdl(dense_decode_kernel<2, true>, grid, block, decode_smem(), stream, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(merge_kernel, dim3((unsigned)((long)a.B * a.Hq)), dim3(kMergeWarps * 32), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dense(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(ranges_kernel, dim3((unsigned)((a.nrt + 255) / 256)), dim3(256), 0, stream, a);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.total_warps), block(32);
    e = a.G <= 8 ? launch_pdl(dense_decode_kernel<1, false>, grid, block, decode_smem(), stream, a)
                 : launch_pdl(dense_decode_kernel<2, false>, grid, block, decode_smem(), stream, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(merge_kernel, dim3((unsigned)((long)a.B * a.Hq)), dim3(kMergeWarps * 32), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
