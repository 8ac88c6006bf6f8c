// sparse_decode.cu -- exact attention over the selected rows of a paged GQA KV cache ("Sparse" mode
// of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?"; SDPA of the xllm
// survey sec. 1.1 restricted to the selected set), and the dense comparator over every row
// ("Dense" mode of the same figure).
//
// Three kernels per call:
//   union_kernel   one CTA per 8192-position range of each (request, KV head) group: finds each head's
//                  slice of its idx row for the range (warp-cooperative search), marks which of the
//                  group's G query heads selected each position, and writes the ascending union of
//                  the group's selections as {cache row index (page table applied), head mask}; the
//                  row counts are added atomically to per-group and global totals.  (Dense decode:
//                  every position is a row and no list is written.)
//   decode_kernel  one warp per CTA, a persistent grid of one wave.  The union rows of all groups,
//                  in (request, KV head, position) order, are cut evenly across the warps; each warp
//                  locates its start from the totals and streams its rows in tiles of 16: every row
//                  is fetched once for all heads of its group with 16-byte cp.async gathers (256-byte
//                  K and V rows into 272-byte padded shared-memory rows, three tiles in flight).  On
//                  the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//                      S   = K_tile (16 rows x 128) . Q^T (128 x 8 heads)          8 MMAs / 8 heads
//                      O^T += V_tile^T (128 x 16 rows) . P (16 rows x 8 heads)     16 MMAs / 8 heads
//                  Heads that did not select a row get -inf before an fp32 online softmax; P goes to
//                  the second product as a bf16 high part plus a bf16 residual (about 16 significant
//                  bits), transposed into operand layout with movmatrix.  The part of a warp's rows
//                  that falls in one group is a "segment"; its (max, sum, output) partial goes to
//                  the workspace.
//   merge_kernel   per (b, h): log-sum-exp merge of the segment partials.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kUnionThreads = 256;
constexpr int kStages = 3;                  // tiles in flight per decode warp
constexpr int kTileRows = 16;
constexpr int kRowPitch = kRowBytes + 16;   // padded shared-memory row: ldmatrix phases hit 8 distinct bank groups
constexpr int kTileBytes = kTileRows * kRowPitch;
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;

// ---------------------------------------------------------------------------------------------
// union_kernel
// ---------------------------------------------------------------------------------------------
size_t union_smem(const DecodeArgs& a) {
    (void)a;
    return sizeof(int) * 64 + sizeof(uint32_t) * (kRange / 2) + sizeof(uint32_t) * (kRange / 32) +
           sizeof(int) * (kRange / kPageSize);
}

// The slice [s, e) of an ascending, -1-padded row whose entries lie in [lo, hi): lanes 0..15 search
// for the first entry >= lo, lanes 16..31 for the first entry >= hi (negative entries count as +inf),
// 17-way per round.  Malformed rows still end the search in range.
__device__ __forceinline__ int2 warp_slice(const int32_t* row, int len, int lo, int hi) {
    const int lane = threadIdx.x & 31, half = lane >> 4, sub = lane & 15;
    const int target = half ? hi : lo;
    int l = 0, h = len;   // the answer lies in [l, h]
    while (__any_sync(0xffffffffu, l < h)) {
        const bool busy = l < h;
        const int span = h - l;
        const int p = l + (int)(((long)(sub + 1) * span) / 17);
        const int v = busy ? __ldg(row + p) : 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, busy && v >= 0 && v < target);
        const int cnt = __popc((bal >> (half * 16)) & 0xffffu);
        if (busy) {
            const int nl = cnt > 0 ? l + (int)(((long)cnt * span) / 17) + 1 : l;
            const int nh = cnt < 16 ? l + (int)(((long)(cnt + 1) * span) / 17) : h;
            l = nl;
            h = nh;
        }
    }
    const int s = __shfl_sync(0xffffffffu, l, 0);
    const int e = __shfl_sync(0xffffffffu, l, 16);
    return make_int2(s, max(s, e));
}

template <bool DENSE>
__global__ void __launch_bounds__(kUnionThreads, 4) union_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    int* scratch = reinterpret_cast<int*>(smem);                 // [64]
    uint32_t* mask = reinterpret_cast<uint32_t*>(scratch + 64);  // [kRange / 2]: two 16-bit head masks per word
    uint32_t* any = mask + kRange / 2;                           // [kRange / 32]: 1 bit per selected position
    int* pt = reinterpret_cast<int*>(any + kRange / 32);         // [kRange / 16]
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int ri = blockIdx.x;
    const int grp = ri / a.nr, r = ri - grp * a.nr;
    const int b = grp / a.Hkv, kvh = grp - b * a.Hkv;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    const int lo = r * kRange, hi = min(lo + kRange, n);
    int cnt = 0;
    if (lo < hi) {
        if constexpr (DENSE) {
            cnt = hi - lo;
        } else {
            uint4* m4 = reinterpret_cast<uint4*>(mask);   // mask and any are contiguous
            for (int i = tid; i < (kRange / 2 + kRange / 32) / 4; i += blockDim.x) m4[i] = make_uint4(0, 0, 0, 0);
            const int np = (hi - lo + kPageSize - 1) / kPageSize;
            const int32_t* ptrow = a.page_table + (long)b * a.max_pages + lo / kPageSize;
            for (int i = tid; i < np; i += blockDim.x) {
                int page = __ldg(ptrow + i);
                if (page < 0 || page >= a.num_pages) {
                    report(a.status, SD_ERR_INDEX_OOB);
                    page = -1;
                }
                pt[i] = page;
            }
            __syncthreads();
            for (int g = warp; g < a.G; g += nwarps) {
                const int32_t* row = a.idx + ((long)b * a.Hq + (long)kvh * a.G + g) * a.k_max;
                const int2 se = warp_slice(row, a.k_max, lo, hi);
                // chunks of 32 entries, four chunks' loads in flight; each entry is checked against
                // its predecessor in the row (strictly ascending, inside this range)
                for (int i0 = se.x; i0 < se.y; i0 += 128) {
                    int v[4], pv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + 32 * u + lane;
                        v[u] = (i < se.y) ? __ldg(row + i) : -1;
                        pv[u] = (lane == 0 && i < se.y && i > 0) ? __ldg(row + i - 1) : -1;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + 32 * u + lane;
                        int prev = __shfl_up_sync(0xffffffffu, v[u], 1);
                        if (lane == 0) prev = pv[u];
                        if (i < se.y) {
                            if (v[u] < lo || v[u] >= hi || (prev >= 0 && prev >= v[u])) {
                                report(a.status, SD_ERR_ORDER);
                            } else {
                                const int o = v[u] - lo;
                                atomicOr(&mask[o >> 1], (1u << g) << ((o & 1) * 16));
                                atomicOr(&any[o >> 5], 1u << (o & 31));
                            }
                        }
                    }
                }
                // the last range of a request: every entry after it must be padding
                if (hi == n && lane == 0 && se.y < a.k_max && __ldg(row + se.y) >= 0) report(a.status, SD_ERR_INDEX_OOB);
            }
            __syncthreads();
            // ordered compaction: thread t owns the 32 positions of bitmap word t
            static_assert(kRange / 32 == kUnionThreads, "one bitmap word per thread");
            uint32_t word = any[tid];
            const int o0 = tid * 32;
            int tot;
            int w = block_exclusive_scan(__popc(word), scratch, &tot);
            uint2* dst = a.entries + (long)ri * kRange;
            while (word) {
                const int o = o0 + __ffs(word) - 1;
                word &= word - 1u;
                const int page = pt[o >> 4];
                const uint32_t m = (mask[o >> 1] >> ((o & 1) * 16)) & 0xffffu;
                if (page >= 0) {
                    const int p = lo + o;
                    const uint32_t rowi =
                        ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + kvh;
                    dst[w++] = make_uint2(rowi, m);
                } else {
                    dst[w++] = make_uint2(0u, 0u);   // invalid page (reported): a row no head attends to
                }
            }
            cnt = tot;
        }
    }
    if (tid == 0) {
        a.counts[ri] = cnt;
        if (cnt > 0) {
            atomicAdd(&a.gtot[grp], cnt);
            atomicAdd(&a.hdr[0], cnt);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// decode_kernel
// ---------------------------------------------------------------------------------------------
struct __align__(128) DecodeSmem {
    uint8_t kv[kStages][2][kTileBytes];       // K tile, V tile: 16 rows x 272 B
    uint32_t meta_mask[kStages][kTileRows];   // head bitmask of each tile row (0: no row)
    int info[kStages][8];                     // rows, flags, b, kvh, segment slot
};

size_t decode_smem() { return sizeof(DecodeSmem); }

// The warp's walk over its union rows (all fields warp-uniform).
struct Walker {
    int e, e_end;     // next global row and the end of this warp's share
    int ri, off;      // range holding row e, and e's offset in it
    int cnt;          // rows in range ri
    int grp;          // group (b * Hkv + kvh) of the current segment
    int seg_j;        // segment slot of the current segment
    bool seg_new;     // the next tile opens a segment
    int epw;
};

// A tile fetched one iteration ahead: row descriptors live in lanes 0..15.
struct TileDesc {
    int rows, flags, b, kvh, seg_j;
    uint32_t row_idx;   // this lane's row (lanes < rows)
    uint32_t mask;
};

template <bool DENSE>
__device__ __forceinline__ TileDesc prefetch_tile(const DecodeArgs& a, Walker& w) {
    const int lane = threadIdx.x & 31;
    TileDesc d;
    d.rows = 0;
    d.flags = 0;
    d.b = d.kvh = d.seg_j = 0;
    d.row_idx = 0;
    d.mask = 0;
    if (w.e >= w.e_end) {
        d.flags = kFlagEnd;
        return d;
    }
    const int grp = w.grp;
    d.b = grp / a.Hkv;
    d.kvh = grp - d.b * a.Hkv;
    d.seg_j = w.seg_j;
    if (w.seg_new) d.flags |= kFlagFirst;
    w.seg_new = false;
    const uint32_t full_mask = (1u << a.G) - 1u;
    int filled = 0;
    while (filled < kTileRows && w.e < w.e_end) {
        if (w.off == w.cnt) {   // next non-empty range; stop at a group boundary
            int ri = w.ri + 1;
            int c = __ldg(a.counts + ri);
            while (c == 0) c = __ldg(a.counts + (++ri));
            if (ri / a.nr != grp) break;
            w.ri = ri;
            w.off = 0;
            w.cnt = c;
        }
        const int take = min(min(kTileRows - filled, w.cnt - w.off), w.e_end - w.e);
        if (lane >= filled && lane < filled + take) {
            const int off = w.off + lane - filled;
            if constexpr (DENSE) {
                const int p = (w.ri - grp * a.nr) * kRange + off;
                int page = __ldg(a.page_table + (long)d.b * a.max_pages + p / kPageSize);
                uint32_t m = full_mask;
                if (page < 0 || page >= a.num_pages) {
                    report(a.status, SD_ERR_INDEX_OOB);
                    page = 0;
                    m = 0;
                }
                d.row_idx = ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + d.kvh;
                d.mask = m;
            } else {
                const uint2 ent = a.entries[(long)w.ri * kRange + off];
                d.row_idx = ent.x;
                d.mask = ent.y;
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
        int ri = w.ri + 1;
        int c = __ldg(a.counts + ri);
        while (c == 0) c = __ldg(a.counts + (++ri));
        if (ri / a.nr != grp) {
            last = true;
            w.ri = ri;   // the next segment starts in range ri
            w.off = 0;
            w.cnt = c;
            w.grp = ri / a.nr;
            w.seg_j = (int)(blockIdx.x - w.e / w.epw);   // w.e is the first row of the new group
            w.seg_new = true;
        }
    }
    if (last) d.flags |= kFlagLast;
    return d;
}

// Writes the tile's metadata to `stage` and issues its row gathers: 16-byte cp.async chunks, lane l
// copying chunk l % 16 of rows l / 16, l / 16 + 2, ...; missing rows are zero-filled.  One
// cp.async group per tile.
__device__ __forceinline__ void issue_tile(const DecodeArgs& a, DecodeSmem& ws, int stage, const TileDesc& d) {
    const int lane = threadIdx.x & 31;
    if (lane < kTileRows) ws.meta_mask[stage][lane] = lane < d.rows ? d.mask : 0u;
    if (lane == 0) {
        ws.info[stage][0] = d.rows;
        ws.info[stage][1] = d.flags;
        ws.info[stage][2] = d.b;
        ws.info[stage][3] = d.kvh;
        ws.info[stage][4] = d.seg_j;
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
            const bool ok = r < d.rows;
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

// Consumer-side state of one warp: NT groups of 8 query heads.
template <int NT>
struct Softmax {
    float m[NT][2];          // running max (log2 units) of heads nt*8 + 2c + e
    float l[NT][2];          // per-thread partial sums of the same heads
    float acc[NT][8][4];     // O^T fragments: dims 16*mt + g (+8) x heads nt*8 + 2c (+1)
    uint32_t qb[NT][8][2];   // Q^T fragments (B operand) of the current group
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
__device__ __forceinline__ void load_q(const DecodeArgs& a, int b, int kvh, Softmax<NT>& st) {
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
__device__ __forceinline__ void flush_state(const DecodeArgs& a, int b, int kvh, int seg_j, Softmax<NT>& st) {
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

template <int NT>
__device__ __forceinline__ void compute_tile(const DecodeArgs& a, const DecodeSmem& ws, int stage, Softmax<NT>& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint32_t kbase = smem_addr(ws.kv[stage][0]);
    const uint32_t vbase = smem_addr(ws.kv[stage][1]);
    const int mi = lane >> 3, r8 = lane & 7;

    // S (16 rows x 8 heads per nt) = K_tile . Q^T
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
    // mask heads that did not select a row (rows g and g+8 of the tile), online softmax per head
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
    // P as the B operand (16 rows x 8 heads): bf16 high part and residual, transposed by movmatrix
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

template <bool DENSE, int NT>
__global__ void __launch_bounds__(32) decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    DecodeSmem& ws = *reinterpret_cast<DecodeSmem*>(smem);
    pdl_enter();

    const int lane = threadIdx.x & 31;
    const int E = a.hdr[0];
    if (E == 0) return;
    Walker w;
    w.epw = max(1, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    w.e = (int)blockIdx.x * w.epw;
    if (w.e >= E) return;
    w.e_end = min(E, w.e + w.epw);
    // the group holding row w.e (prefix over the per-group totals), then its range
    int e0grp = 0;
    w.grp = -1;
    {
        const int ngroups = a.B * a.Hkv;
        int acc = 0;
        for (int base = 0; base < ngroups && w.grp < 0; base += 32) {
            const int v = (base + lane < ngroups) ? __ldg(a.gtot + base + lane) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int tot = __shfl_sync(0xffffffffu, incl, 31);
            if (w.e < acc + tot) {
                const int l = __ffs(__ballot_sync(0xffffffffu, acc + incl > w.e)) - 1;
                w.grp = base + l;
                e0grp = acc + __shfl_sync(0xffffffffu, incl - v, l);
            }
            acc += tot;
        }
        const int off_g = w.e - e0grp;
        int acc2 = 0;
        w.ri = -1;
        for (int base = 0; base < a.nr && w.ri < 0; base += 32) {
            const int v = (base + lane < a.nr) ? __ldg(a.counts + w.grp * a.nr + base + lane) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int tot = __shfl_sync(0xffffffffu, incl, 31);
            if (off_g < acc2 + tot) {
                const int l = __ffs(__ballot_sync(0xffffffffu, acc2 + incl > off_g)) - 1;
                w.ri = w.grp * a.nr + base + l;
                w.off = off_g - (acc2 + __shfl_sync(0xffffffffu, incl - v, l));
            }
            acc2 += tot;
        }
    }
    w.cnt = __ldg(a.counts + w.ri);
    w.seg_j = (int)(blockIdx.x - e0grp / w.epw);
    w.seg_new = true;

    Softmax<NT> st;
    reset_state(st);
    TileDesc next = prefetch_tile<DENSE>(a, w);
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue_tile(a, ws, s, next);
        next = prefetch_tile<DENSE>(a, w);
    }
    for (int t = 0;; ++t) {
        const int stage = t % kStages;
        // the stage of tile t-1 is free: issue tile t+kStages-1 before waiting for tile t
        issue_tile(a, ws, (t + kStages - 1) % kStages, next);
        next = prefetch_tile<DENSE>(a, w);
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int rows = ws.info[stage][0], flags = ws.info[stage][1];
        if (flags & kFlagEnd) break;
        const int tb = ws.info[stage][2], tkvh = ws.info[stage][3], tj = ws.info[stage][4];
        if (flags & kFlagFirst) load_q(a, tb, tkvh, st);
        if (rows > 0) compute_tile(a, ws, stage, st);
        if (flags & kFlagLast) {
            flush_state(a, tb, tkvh, tj, st);
            reset_state(st);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

// One CTA per (b, h), one thread per output dimension: log-sum-exp merge of the segment partials of
// its group, 32 segments at a time (all loads of a chunk are in flight together).
__global__ void __launch_bounds__(kHeadDim) merge_kernel(DecodeArgs a) {
    __shared__ float s_m[32];   // per-segment weights of the current chunk
    __shared__ float s_l[32];
    __shared__ float s_scale[1];
    pdl_enter();
    const int d = threadIdx.x;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq), kvh = h / a.G;
    __shared__ int s_e0;
    const int grp = b * a.Hkv + kvh;
    if (d < 32) {   // first union row of the group: prefix over the per-group totals
        int acc = 0;
        for (int base = 0; base < grp; base += 32) {
            int v = (base + d < grp) ? a.gtot[base + d] : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc += v;
        }
        if (d == 0) s_e0 = acc;
    }
    __syncthreads();
    const int E = a.hdr[0];
    const int epw = max(1, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    const int e0 = s_e0, e1 = e0 + a.gtot[grp];
    const int nseg = (e1 > e0) ? ((e1 - 1) / epw - e0 / epw + 1) : 0;
    const float2* ml = a.ml + bh * a.jmax;
    const float* accp = a.acc + bh * a.jmax * kHeadDim + d;
    float M = -INFINITY, L = 0.f, o = 0.f;
    for (int j0 = 0; j0 < nseg; j0 += 32) {
        const int cnt = min(32, nseg - j0);
        float x[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) x[jj] = (jj < cnt) ? accp[(long)(j0 + jj) * kHeadDim] : 0.f;
        if (d < 32) {   // warp 0: the chunk's max, then one weight per segment
            const float2 v = (d < cnt) ? ml[j0 + d] : make_float2(-INFINITY, 0.f);
            float cm = v.x;
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o2));
            const float nm = fmaxf(M, cm);
            s_m[d] = (v.x == -INFINITY) ? 0.f : exp2f(v.x - nm);   // weight of segment j0 + d
            s_l[d] = v.y;
            if (d == 0) s_scale[0] = nm;
        }
        __syncthreads();
        const float nm = s_scale[0];
        if (nm != -INFINITY) {
            const float sc = (M == -INFINITY) ? 0.f : exp2f(M - nm);
            o *= sc;
            L *= sc;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                o += s_m[jj] * x[jj];
                L += s_m[jj] * s_l[jj];
            }
            M = nm;
        }
        __syncthreads();
    }
    a.out[bh * kHeadDim + d] = L > 0.f ? o / L : 0.f;
}

// ---------------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------------
template <bool DENSE, int NT>
static cudaError_t occupancy_of(int* ctas) {
    const size_t smem = decode_smem();
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DENSE, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, decode_kernel<DENSE, NT>, 32, smem);
}

cudaError_t decode_occupancy(bool dense, int G, int* ctas_per_sm) {
    if (G <= 8) return dense ? occupancy_of<true, 1>(ctas_per_sm) : occupancy_of<false, 1>(ctas_per_sm);
    return dense ? occupancy_of<true, 2>(ctas_per_sm) : occupancy_of<false, 2>(ctas_per_sm);
}

cudaError_t launch_union(const DecodeArgs& a, bool dense, cudaStream_t stream) {
    const size_t smem = union_smem(a);
    cudaError_t e;
    if (dense) {
        e = cudaFuncSetAttribute(union_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(union_kernel<true>, dim3(a.nrt), dim3(kUnionThreads), smem, stream, a);
        if (e != cudaSuccess) return e;
    } else {
        e = cudaFuncSetAttribute(union_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(union_kernel<false>, dim3(a.nrt), dim3(kUnionThreads), smem, stream, a);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, bool dense, cudaStream_t stream) {
    const size_t smem = decode_smem();
    const dim3 grid(a.total_warps), block(32);
    cudaError_t e;
    if (a.G <= 8) e = dense ? launch_pdl(decode_kernel<true, 1>, grid, block, smem, stream, a)
                            : launch_pdl(decode_kernel<false, 1>, grid, block, smem, stream, a);
    else e = dense ? launch_pdl(decode_kernel<true, 2>, grid, block, smem, stream, a)
                   : launch_pdl(decode_kernel<false, 2>, grid, block, smem, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(merge_kernel, dim3((unsigned)((long)a.B * a.Hq)), dim3(kHeadDim), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Zeroes the per-group and global union-row totals that union_kernel accumulates.
__global__ void __launch_bounds__(256) prep_kernel(DecodeArgs a) {
    pdl_enter();
    for (int i = threadIdx.x; i < 4 + a.B * a.Hkv; i += blockDim.x) a.hdr[i] = 0;
}

cudaError_t launch_prep(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t e = launch_pdl(prep_kernel, dim3(1), dim3(256), 0, stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sd
