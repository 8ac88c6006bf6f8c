// sparse_decode.cu -- exact attention over the selected rows of a paged GQA KV cache ("Sparse" mode
// of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?"; SDPA of the xllm
// survey sec. 1.1 restricted to the selected set), and the dense comparator over every row
// ("Dense" mode of the same figure).
//
// Sparse decode, two kernels per call:
//   rows_kernel           one group of threads per (request, query head) row of idx: checks the row
//                         (ascending positions below N_b, then negative padding only), finds its length
//                         (the index of the first negative entry), maps every position to its cache row
//                         through the page table, zeroes the output of empty rows and the row's arrival
//                         counter, and writes per-CTA length sums.
//   sparse_decode_kernel  one warp per CTA, a persistent grid of one wave.  The selected entries of all
//                         rows, in (request, head, position) order, are cut evenly across the warps; a
//                         warp finds its first row from the length sums and streams its entries in
//                         tiles of 16 rows: 16-byte cp.async gathers of the 256-byte K and V rows into
//                         272-byte padded shared-memory rows, three tiles in flight.  The heads of a GQA
//                         group are consecutive rows, so their warps run side by side and a row several
//                         of them selected is mostly served from L2 after its first read.  On the tensor
//                         cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), with q in column 0 of the
//                         B operand:
//                             S   = K_tile (16 rows x 128) . q                  8 MMAs
//                             o  += V_tile^T (128 x 16 rows) . p                16 MMAs (p as bf16 hi + lo)
//                         and an fp32 online softmax in between.  A warp's part of one row is a
//                         "segment": a row held by one warp is written out directly; otherwise each
//                         warp stores its (max, sum, output) partial and the last of the row's warps to
//                         arrive (a counter per row) merges the partials by log-sum-exp.
//
// Dense decode (the comparator), three kernels: ranges_kernel counts the positions of each
// kRange-position range of every (request, KV head) group; dense_decode_kernel walks all rows of every
// group with the same tile pipeline, one 16-row tile serving all G heads of the group (S = K_tile . Q^T
// with the G heads as columns), its first range found from the counts; merge_kernel (four warps per
// (b, h)) combines the segment partials.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kStages = 3;                  // tiles in flight per decode warp
constexpr int kTileRows = 16;
constexpr int kRowPitch = kRowBytes + 16;   // padded shared-memory row: ldmatrix phases hit 8 distinct bank groups
constexpr int kTileBytes = kTileRows * kRowPitch;
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;
constexpr uint32_t kNoRow = 0xffffffffu;    // rowidx entry of a position that maps to no cache row
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

// A tile fetched one iteration ahead: row descriptors live in lanes 0..15.
struct TileDesc {
    int rows, flags;
    int owner;          // dense: group b * Hkv + kvh; sparse: row b * Hq + h
    int seg_j, nseg;    // segment slot of this warp in the owner, and the owner's segment count (sparse)
    uint32_t row_idx;   // this lane's cache row (lanes < rows); kNoRow: none (the row is skipped)
    uint32_t mask;      // heads (columns) that attend to it
};

__device__ __forceinline__ TileDesc empty_tile() {
    TileDesc d;
    d.rows = 0;
    d.flags = 0;
    d.owner = d.seg_j = d.nseg = 0;
    d.row_idx = 0;
    d.mask = 0;
    return d;
}

// Writes the tile's metadata to `stage` and issues its row gathers: 16-byte cp.async chunks, lane l
// copying chunk l % 16 of rows l / 16, l / 16 + 2, ...; missing rows are zero-filled.  One
// cp.async group per tile.  This is the first use of the row indices loaded by the prefetch one
// iteration earlier, so that load stays in flight while the warp computes the previous tile.
__device__ __forceinline__ void issue_tile(const DecodeArgs& a, DecodeSmem& ws, int stage, const TileDesc& d) {
    const int lane = threadIdx.x & 31;
    if (lane < kTileRows) ws.meta_mask[stage][lane] = (lane < d.rows && d.row_idx != kNoRow) ? d.mask : 0u;
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
            const uint32_t ri = __shfl_sync(0xffffffffu, d.row_idx, r);
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
// lane before.  rowidx rows are a.rstride (a multiple of kRowBatch) entries apart.
__global__ void __launch_bounds__(1024, 2) rows_kernel(DecodeArgs a) {
    __shared__ int s_neg[32];   // per warp: first negative entry it saw
    __shared__ int s_len[32];   // per row of this CTA
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tpr = a.tpr, wpr = tpr >> 5;
    const int rl = tid / tpr, t = tid - rl * tpr;
    const int R = a.B * a.Hq;
    const int r = blockIdx.x * a.rpc + rl;
    const int k_max = a.k_max;
    int first_neg = k_max;
    if (r < R) {   // uniform over the row's warps
        const int b = r / a.Hq, kvh = (r - b * a.Hq) / a.G;
        const int n = checked_len(a.lens, b, a.n_cap, a.status);
        const int32_t* row = a.idx + (long)r * k_max;
        uint32_t* dst = a.rowidx + (long)r * a.rstride;
        const int32_t* ptrow = a.page_table + (long)b * a.max_pages;
        for (int base = 0; base < k_max; base += tpr * kRowBatch) {   // uniform over the row's threads
            const int j0 = base + t * kRowBatch;
            int v[kRowBatch];
#pragma unroll
            for (int i = 0; i < kRowBatch; ++i) v[i] = j0 + i < k_max ? __ldg(row + j0 + i) : -1;
            const int pv = (lane == 0 && j0 > 0) ? __ldg(row + j0 - 1) : -1;
            int p = __shfl_up_sync(0xffffffffu, v[kRowBatch - 1], 1);
            if (lane == 0) p = pv;
            int pg[kRowBatch];
#pragma unroll
            for (int i = 0; i < kRowBatch; ++i) {
                const int j = j0 + i;
                pg[i] = -2;   // no cache row looked up
                if (j < k_max) {
                    if (v[i] < 0) {
                        first_neg = min(first_neg, j);
                    } else if (v[i] >= n) {
                        report(a.status, SD_ERR_INDEX_OOB);
                    } else {
                        if (j > 0 && (p < 0 || p >= v[i])) report(a.status, SD_ERR_ORDER);
                        pg[i] = __ldg(ptrow + (v[i] >> 4));
                    }
                }
                p = v[i];
            }
            uint32_t ri[kRowBatch];
#pragma unroll
            for (int i = 0; i < kRowBatch; ++i) {
                ri[i] = kNoRow;
                if (pg[i] >= 0 && pg[i] < a.num_pages)
                    ri[i] = ((uint32_t)pg[i] * kPageSize + (uint32_t)(v[i] & (kPageSize - 1))) * (uint32_t)a.Hkv + kvh;
                else if (pg[i] != -2)
                    report(a.status, SD_ERR_INDEX_OOB);
            }
            static_assert(kRowBatch == 4, "one 16-byte store per pass");
            if (j0 < k_max) *reinterpret_cast<uint4*>(dst + j0) = make_uint4(ri[0], ri[1], ri[2], ri[3]);
        }
    }
    first_neg = __reduce_min_sync(0xffffffffu, first_neg);
    if (lane == 0) s_neg[warp] = first_neg;
    __syncthreads();
    if (t == 0) {
        int m = k_max;
        for (int w = 0; w < wpr; ++w) m = min(m, s_neg[rl * wpr + w]);
        if (r < R) {
            a.rlen[r] = m;
            a.arrive[r] = 0;
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
// The warp's walk over its entries (all fields warp-uniform).
struct RowWalker {
    int e, e_end;        // next entry (global order) and the end of this warp's share
    int epw;             // entries per warp
    int r;               // row holding entry e
    int rstart, rend;    // global entry range of row r
    bool seg_new;        // the next tile opens a segment
};

__device__ __forceinline__ TileDesc prefetch_row_tile(const DecodeArgs& a, RowWalker& w) {
    const int lane = threadIdx.x & 31;
    TileDesc d = empty_tile();
    if (w.e >= w.e_end) {
        d.flags = kFlagEnd;
        return d;
    }
    d.owner = w.r;
    const int first_warp = w.rstart / w.epw;
    d.seg_j = (int)blockIdx.x - first_warp;
    d.nseg = (w.rend - 1) / w.epw - first_warp + 1;
    if (w.seg_new) d.flags |= kFlagFirst;
    w.seg_new = false;
    const int rows = min(kTileRows, min(w.rend, w.e_end) - w.e);
    if (rows <= 0) {   // not reached (row lengths and their sums come from one pass); ends the walk
        w.e = w.e_end;
        d.flags = kFlagEnd;
        return d;
    }
    if (lane < rows) {   // not examined until the tile is issued (one iteration later)
        d.row_idx = __ldg(a.rowidx + (long)w.r * a.rstride + (w.e - w.rstart) + lane);
        d.mask = 1u;
    }
    d.rows = rows;
    w.e += rows;
    if (w.e == w.rend || w.e == w.e_end) {
        d.flags |= kFlagLast;
        if (w.e < w.e_end) {   // the next non-empty row (one exists: entries remain)
            const int R = a.B * a.Hq;
            int r = w.r + 1;
            int len = __ldg(a.rlen + r);
            while (len == 0 && r + 1 < R) len = __ldg(a.rlen + (++r));
            w.r = r;
            w.rstart = w.rend;
            w.rend = w.rstart + len;
            w.seg_new = true;
        }
    }
    return d;
}

// Column 0 of the B operand is q[b][h]; the other columns are zero.
__device__ __forceinline__ void load_q_row(const DecodeArgs& a, int r, Softmax<1>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint32_t* qr = reinterpret_cast<const uint32_t*>(a.q + (long)r * kHeadDim);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        st.qb[0][j][0] = g == 0 ? __ldg(qr + 8 * j + c) : 0u;
        st.qb[0][j][1] = g == 0 ? __ldg(qr + 8 * j + c + 4) : 0u;
    }
}

// One warp: log-sum-exp merge of the nseg partials of row r (lane l owns dimensions 4l .. 4l+3).
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
    for (int j0 = 0; j0 < nseg; j0 += 32) {
        const float2 v = (j0 + lane < nseg) ? __ldcg(ml + j0 + lane) : make_float2(-INFINITY, 0.f);
        const float wj = (v.x == -INFINITY) ? 0.f : exp2f(v.x - M);
        float lw = wj * v.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
        L += lw;
        const int cnt = min(32, nseg - j0);
        const float4* src = reinterpret_cast<const float4*>(a.acc + ((long)r * a.jmax + j0) * kHeadDim) + lane;
        for (int jj = 0; jj < cnt; ++jj) {
            const float ww = __shfl_sync(0xffffffffu, wj, jj);
            const float4 x = __ldcg(src + (long)jj * (kHeadDim / 4));
            o4.x += ww * x.x;
            o4.y += ww * x.y;
            o4.z += ww * x.z;
            o4.w += ww * x.w;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    reinterpret_cast<float4*>(a.out + (long)r * kHeadDim)[lane] =
        make_float4(o4.x * inv, o4.y * inv, o4.z * inv, o4.w * inv);
}

// End of this warp's segment of row r (column 0 of the state).
__device__ __forceinline__ void finish_row_segment(const DecodeArgs& a, int r, int j, int nseg, Softmax<1>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    float l = st.l[0][0];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    if (nseg == 1) {   // the whole row is this warp's
        if (c == 0) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            float* dst = a.out + (long)r * kHeadDim;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                dst[16 * mt + g] = st.acc[0][mt][0] * inv;
                dst[16 * mt + g + 8] = st.acc[0][mt][2] * inv;
            }
        }
        return;
    }
    const long slot = (long)r * a.jmax + j;
    if (lane == 0) a.ml[slot] = make_float2(st.m[0][0], l);
    if (c == 0) {
        float* dst = a.acc + slot * kHeadDim;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            dst[16 * mt + g] = st.acc[0][mt][0];
            dst[16 * mt + g + 8] = st.acc[0][mt][2];
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

__global__ void __launch_bounds__(32) sparse_decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    DecodeSmem& ws = *reinterpret_cast<DecodeSmem*>(smem);
    pdl_enter();

    const int lane = threadIdx.x & 31;
    const int R = a.B * a.Hq;
    // E = all entries: the length sums of the rows_kernel CTAs, kPrologue per lane in flight together
    int E = 0;
    for (int base = 0; base < a.nb; base += 32 * kPrologue) {
        int v[kPrologue];
#pragma unroll
        for (int i = 0; i < kPrologue; ++i) {
            const int k = base + 32 * i + lane;
            v[i] = k < a.nb ? __ldg(a.bsum + k) : 0;
        }
#pragma unroll
        for (int i = 0; i < kPrologue; ++i) E += v[i];
    }
    E = __reduce_add_sync(0xffffffffu, E);
    if (E == 0) return;
    RowWalker w;
    w.epw = max(a.min_epw, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    const long e0 = (long)blockIdx.x * w.epw;
    if (e0 >= E) return;
    w.e = (int)e0;
    w.e_end = (int)min((long)E, e0 + w.epw);
    // the rows_kernel CTA whose rows hold entry w.e (prefix over the same sums, now in L1), then the row
    int blk = -1, blk0 = 0, blen = 0;
    {
        int acc = 0;
        for (int base = 0; base < a.nb && blk < 0; base += 32 * kPrologue) {
            int v[kPrologue];
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int k = base + 32 * i + lane;
                v[i] = k < a.nb ? __ldg(a.bsum + k) : 0;
            }
#pragma unroll
            for (int i = 0; i < kPrologue; ++i) {
                const int incl = warp_inclusive_scan(v[i]);
                const uint32_t hit = __ballot_sync(0xffffffffu, acc + incl > w.e);
                if (blk < 0 && hit != 0u) {
                    const int l = __ffs(hit) - 1;
                    blk = base + 32 * i + l;
                    blk0 = acc + __shfl_sync(0xffffffffu, incl - v[i], l);
                    blen = __shfl_sync(0xffffffffu, v[i], l);
                }
                acc += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
    }
    if (blk < 0) return;   // not reached: w.e < E
    if (a.rpc == 1) {      // one row per CTA of the row pass
        w.r = blk;
        w.rstart = blk0;
        w.rend = blk0 + blen;
    } else {
        const int r0 = blk * a.rpc;
        const int v = (lane < a.rpc && r0 + lane < R) ? __ldg(a.rlen + r0 + lane) : 0;
        const int incl = warp_inclusive_scan(v);
        const uint32_t hit = __ballot_sync(0xffffffffu, blk0 + incl > w.e);
        if (hit == 0u) return;   // not reached: the CTA's rows hold entry w.e
        const int l = __ffs(hit) - 1;
        w.r = r0 + l;
        w.rstart = blk0 + __shfl_sync(0xffffffffu, incl - v, l);
        w.rend = w.rstart + __shfl_sync(0xffffffffu, v, l);
    }
    w.seg_new = true;

    Softmax<1> st;
    reset_state(st);
    TileDesc next = prefetch_row_tile(a, w);
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue_tile(a, ws, s, next);
        next = prefetch_row_tile(a, w);
    }
    for (int t = 0;; ++t) {
        const int stage = t % kStages;
        // the stage of tile t-1 is free: issue tile t+kStages-1 before waiting for tile t
        issue_tile(a, ws, (t + kStages - 1) % kStages, next);
        next = prefetch_row_tile(a, w);
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int rows = ws.info[stage][0], flags = ws.info[stage][1];
        if (flags & kFlagEnd) break;
        const int r = ws.info[stage][2], j = ws.info[stage][3], nseg = ws.info[stage][4];
        if (flags & kFlagFirst) load_q_row(a, r, st);
        if (rows > 0) compute_tile(a, ws, stage, st);
        if (flags & kFlagLast) {
            finish_row_segment(a, r, j, nseg, st);
            reset_state(st);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
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

// The warp's walk over its rows (all fields warp-uniform).
struct GroupWalker {
    int e, e_end;     // next global row and the end of this warp's share
    int ri, off;      // range holding row e, and e's offset in it
    int cnt;          // rows in range ri
    int grp;          // group (b * Hkv + kvh) of the current segment
    int seg_j;        // segment slot of the current segment
    bool seg_new;     // the next tile opens a segment
    int epw;          // rows per warp
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
        }
        const int take = min(min(kTileRows - filled, w.cnt - w.off), w.e_end - w.e);
        if (take <= 0) {   // not reached (counts are consistent); ends the walk
            w.e = w.e_end;
            break;
        }
        if (lane >= filled && lane < filled + take) {
            const int off = w.off + lane - filled;
            const int p = (w.ri - grp * a.nrp) * kRange + off;
            const int page = __ldg(a.page_table + (long)b * a.max_pages + p / kPageSize);
            if (page < 0 || page >= a.num_pages) {
                report(a.status, SD_ERR_INDEX_OOB);
                d.row_idx = kNoRow;
            } else {
                d.row_idx = ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + kvh;
            }
            d.mask = full_mask;
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

template <int NT>
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
    const int e0grp = ri0 - sum_counts(a, w.grp * a.nrp, ri);   // first row of the group
    w.seg_j = (int)(blockIdx.x - e0grp / w.epw);
    w.seg_new = true;

    Softmax<NT> st;
    reset_state(st);
    TileDesc next = prefetch_group_tile(a, w);
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue_tile(a, ws, s, next);
        next = prefetch_group_tile(a, w);
    }
    for (int t = 0;; ++t) {
        const int stage = t % kStages;
        // the stage of tile t-1 is free: issue tile t+kStages-1 before waiting for tile t
        issue_tile(a, ws, (t + kStages - 1) % kStages, next);
        next = prefetch_group_tile(a, w);
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
    if (!dense) return occupancy_of(sparse_decode_kernel, ctas_per_sm);
    return G <= 8 ? occupancy_of(dense_decode_kernel<1>, ctas_per_sm) : occupancy_of(dense_decode_kernel<2>, ctas_per_sm);
}

cudaError_t launch_sparse(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(rows_kernel, dim3(a.nb), dim3(a.tpr * a.rpc), 0, stream, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(sparse_decode_kernel, dim3(a.total_warps), dim3(32), decode_smem(), stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dense(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(ranges_kernel, dim3((unsigned)((a.nrt + 255) / 256)), dim3(256), 0, stream, a);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.total_warps), block(32);
    e = a.G <= 8 ? launch_pdl(dense_decode_kernel<1>, grid, block, decode_smem(), stream, a)
                 : launch_pdl(dense_decode_kernel<2>, grid, block, decode_smem(), stream, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(merge_kernel, dim3((unsigned)((long)a.B * a.Hq)), dim3(kMergeWarps * 32), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
