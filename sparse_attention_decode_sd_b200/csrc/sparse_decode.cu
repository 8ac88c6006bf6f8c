// sparse_decode.cu -- exact attention over the selected rows of a paged GQA KV cache ("Sparse" mode
// of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?"; SDPA of the xllm
// survey sec. 1.1 restricted to the selected set), and the dense comparator over every row
// ("Dense" mode of the same figure).
//
// Three kernels per call:
//   union_kernel   one CTA per 8192-position range of each (request, KV head) group: marks which of
//                  the group's G query heads selected each position, and writes the ascending union
//                  of the group's selections as {cache row index (page table applied), head mask}.
//                  The last CTA to finish prefix-sums the per-range counts and cuts the flattened
//                  union-row sequence evenly across the decode warps.  (Dense decode: every
//                  position is a row and no list is written.)
//   decode_kernel  one warp per CTA, a persistent grid of one wave.  Each warp streams its share of
//                  union rows in tiles of 16: every row is fetched once for all heads of its group
//                  with 16-byte cp.async gathers (256-byte K and V rows into 272-byte padded
//                  shared-memory rows, three tiles in flight).  On the
//                  tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
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
__device__ __forceinline__ int len_checked(const DecodeArgs& a, int b) {
    return checked_len(a.lens, b, a.n_cap, a.status);
}

size_t union_smem(const DecodeArgs& a) {
    const size_t build = sizeof(uint32_t) * (kRange / 2) + sizeof(int) * (kRange / kPageSize);
    const size_t tail = sizeof(int) * ((size_t)a.nrt + 1);
    return sizeof(int) * 64 + (build > tail ? build : tail);
}

// One thread per idx entry (grid: entry chunks x rows): entry i of row (b, h) opens every range r'
// in (range(prev), range(v)] -- bounds[b,h][r'] = i -- and the row's last valid entry closes the
// remaining ranges.  Every slot of a well-formed row is written exactly once, so nothing needs
// clearing.  Also checks the row: entries must lie in [0, N_b) and be strictly ascending, with
// padding only at the end.
__global__ void __launch_bounds__(256) bounds_kernel(DecodeArgs a) {
    const int lane = threadIdx.x & 31;
    const long bh = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = (int)(bh / a.Hq);
    const int n = len_checked(a, b);
    const int32_t* row = a.idx + bh * a.k_max;
    const int v = (i < a.k_max) ? row[i] : -1;
    int prev = __shfl_up_sync(0xffffffffu, v, 1);
    int next = __shfl_down_sync(0xffffffffu, v, 1);
    if (lane == 0) prev = (i > 0 && i - 1 < a.k_max) ? row[i - 1] : -1;
    if (lane == 31 || i + 1 >= a.k_max) next = (i + 1 < a.k_max) ? row[i + 1] : -1;
    if (i >= a.k_max) return;
    int* bounds = a.bounds + bh * (a.nr + 1);
    const bool valid = v >= 0 && v < n;
    if (v >= n) report(a.status, SD_ERR_INDEX_OOB);
    if (v >= 0 && i > 0 && (prev < 0 || prev >= v)) report(a.status, SD_ERR_ORDER);
    const bool prev_valid = i > 0 && prev >= 0 && prev < n;
    if (valid) {
        const int rv = v / kRange;
        const int rp = prev_valid ? min(prev / kRange, rv) : -1;
        for (int r = rp + 1; r <= rv; ++r) bounds[r] = i;
        const bool next_valid = next >= 0 && next < n;
        if (!next_valid)
            for (int r = rv + 1; r <= a.nr; ++r) bounds[r] = i + 1;
    } else if (i == 0) {   // a row that starts with padding has no selected rows
        for (int r = 0; r <= a.nr; ++r) bounds[r] = 0;
    }
}

template <bool DENSE>
__global__ void __launch_bounds__(kUnionThreads, 4) union_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    int* scratch = reinterpret_cast<int*>(smem);                 // [64]
    uint32_t* mask = reinterpret_cast<uint32_t*>(scratch + 64);  // [kRange / 2]: two 16-bit head masks per word
    int* pt = reinterpret_cast<int*>(mask + kRange / 2);         // [kRange / 16]
    __shared__ int s_last;
    __shared__ int s_lo[kMaxGroup], s_len[kMaxGroup], s_pre[kMaxGroup + 1];
    const int tid = threadIdx.x;
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
            uint4* m4 = reinterpret_cast<uint4*>(mask);
            for (int i = tid; i < kRange / 8; i += blockDim.x) m4[i] = make_uint4(0, 0, 0, 0);
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
            if (tid < a.G) {   // this range's slice [s, e) of each head's row (clamped: rows may be malformed)
                const int* bd = a.bounds + ((long)b * a.Hq + (long)kvh * a.G + tid) * (a.nr + 1);
                const int s = min(max(bd[r], 0), a.k_max);
                const int e = min(max(bd[r + 1], s), a.k_max);
                s_lo[tid] = s;
                s_len[tid] = e - s;
            }
            __syncthreads();
            if (tid == 0) {
                int acc = 0;
                for (int g = 0; g < a.G; ++g) {
                    s_pre[g] = acc;
                    acc += s_len[g];
                }
                s_pre[a.G] = acc;
            }
            __syncthreads();
            // every thread marks entries of the flattened slices, eight independent loads at a time
            const int tot_e = s_pre[a.G];
            const int32_t* rows0 = a.idx + ((long)b * a.Hq + (long)kvh * a.G) * a.k_max;
            constexpr int kBatch = 8;
            for (int x0 = 0; x0 < tot_e; x0 += kBatch * kUnionThreads) {
                int v[kBatch], gg[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int x = x0 + u * kUnionThreads + tid;
                    v[u] = -1;
                    gg[u] = 0;
                    if (x < tot_e) {
                        int g = 0;
                        while (x >= s_pre[g + 1]) ++g;
                        gg[u] = g;
                        v[u] = __ldg(rows0 + (long)g * a.k_max + s_lo[g] + (x - s_pre[g]));
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    if (v[u] >= lo && v[u] < hi) {
                        const int o = v[u] - lo;
                        atomicOr(&mask[o >> 1], (1u << gg[u]) << ((o & 1) * 16));
                    }
            }
            __syncthreads();
            // ordered compaction: thread t owns positions [32t, 32t + 32) of the range
            constexpr int kPer = kRange / kUnionThreads;
            const int o0 = tid * kPer;
            uint32_t words[kPer / 2];
            int c = 0;
#pragma unroll
            for (int k = 0; k < kPer / 2; ++k) {
                words[k] = mask[o0 / 2 + k];
                const int o = o0 + 2 * k;
                const bool v0 = o < hi - lo && (words[k] & 0xffffu) && pt[o >> 4] >= 0;
                const bool v1 = o + 1 < hi - lo && (words[k] >> 16) && pt[o >> 4] >= 0;
                c += v0 + v1;
            }
            int tot;
            int w = block_exclusive_scan(c, scratch, &tot);
            uint2* dst = a.entries + (long)ri * kRange;
#pragma unroll
            for (int k = 0; k < kPer / 2; ++k) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int o = o0 + 2 * k + h;
                    const uint32_t m = (words[k] >> (16 * h)) & 0xffffu;
                    if (o < hi - lo && m) {
                        const int page = pt[o >> 4];
                        if (page >= 0) {
                            const int p = lo + o;
                            const uint32_t rowi =
                                ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + kvh;
                            dst[w++] = make_uint2(rowi, m);
                        }
                    }
                }
            }
            cnt = tot;
        }
    }
    if (tid == 0) a.counts[ri] = cnt;

    // The last CTA to finish: prefix over all ranges and the decode warps' starting points.
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.hdr[2], 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    int* offs = scratch + 64;   // [nrt + 1]
    const volatile int* vcounts = a.counts;
    int carry = 0;
    for (int base = 0; base < a.nrt; base += blockDim.x) {
        const int i = base + tid;
        const int v = (i < a.nrt) ? vcounts[i] : 0;
        int tot;
        const int ex = block_exclusive_scan(v, scratch, &tot);
        if (i < a.nrt) {
            offs[i] = carry + ex;
            a.offsets[i] = carry + ex;
        }
        carry += tot;
    }
    const int E = carry;
    const int epw = max(1, (int)(((long)E + a.total_warps - 1) / a.total_warps));
    if (tid == 0) {
        offs[a.nrt] = E;
        a.offsets[a.nrt] = E;
        a.hdr[0] = E;
        a.hdr[1] = epw;
    }
    __syncthreads();
    for (int w = tid; w < a.total_warps; w += blockDim.x) {
        const long e0 = (long)w * epw;
        int2 start = make_int2(-1, 0);
        if (e0 < E) {   // largest range with offs <= e0 (it is non-empty)
            int l = 0, h = a.nrt;
            while (h - l > 1) {
                const int mid = (l + h) >> 1;
                if (offs[mid] <= e0) l = mid; else h = mid;
            }
            start = make_int2(l, (int)(e0 - offs[l]));
        }
        a.warp_start[w] = start;
    }
    if (tid == 0) a.hdr[2] = 0;   // ticket ready for the next call
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
            w.seg_j = (int)(blockIdx.x - __ldg(a.offsets + w.grp * a.nr) / w.epw);
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
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
        const uint32_t rowaddr = kbase + (uint32_t)((((mi & 1) << 3) + r8) * kRowPitch + ((mi >> 1) << 4));
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(rowaddr + 32 * j, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a0, a1, a2, a3, st.qb[nt][j][0], st.qb[nt][j][1]);
        }
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

    const int2 start = a.warp_start[blockIdx.x];
    if (start.x < 0) return;
    const int E = a.hdr[0];
    Walker w;
    w.epw = a.hdr[1];
    w.e = (int)blockIdx.x * w.epw;
    w.e_end = min(E, w.e + w.epw);
    w.ri = start.x;
    w.off = start.y;
    w.cnt = __ldg(a.counts + w.ri);
    w.grp = w.ri / a.nr;
    w.seg_j = (int)(blockIdx.x - __ldg(a.offsets + w.grp * a.nr) / w.epw);
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
        cp_async_wait<kStages - 2>();
        __syncwarp();
        const int rows = ws.info[stage][0], flags = ws.info[stage][1];
        if (flags & kFlagEnd) break;
        const int tb = ws.info[stage][2], tkvh = ws.info[stage][3], tj = ws.info[stage][4];
        issue_tile(a, ws, (t + kStages - 1) % kStages, next);
        next = prefetch_tile<DENSE>(a, w);
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
    const int d = threadIdx.x;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq), kvh = h / a.G;
    const int grp = b * a.Hkv + kvh;
    const int e0 = a.offsets[grp * a.nr], e1 = a.offsets[(grp + 1) * a.nr];
    const int epw = a.hdr[1];
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

cudaError_t launch_bounds(const DecodeArgs& a, cudaStream_t stream) {
    const dim3 grid((unsigned)((a.k_max + 255) / 256), (unsigned)((long)a.B * a.Hq));
    bounds_kernel<<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_union(const DecodeArgs& a, bool dense, cudaStream_t stream) {
    const size_t smem = union_smem(a);
    cudaError_t e;
    if (dense) {
        e = cudaFuncSetAttribute(union_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        union_kernel<true><<<a.nrt, kUnionThreads, smem, stream>>>(a);
    } else {
        e = cudaFuncSetAttribute(union_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        union_kernel<false><<<a.nrt, kUnionThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, bool dense, cudaStream_t stream) {
    const size_t smem = decode_smem();
    const int ctas = a.total_warps;
    if (a.G <= 8) {
        if (dense) decode_kernel<true, 1><<<ctas, 32, smem, stream>>>(a);
        else decode_kernel<false, 1><<<ctas, 32, smem, stream>>>(a);
    } else {
        if (dense) decode_kernel<true, 2><<<ctas, 32, smem, stream>>>(a);
        else decode_kernel<false, 2><<<ctas, 32, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream) {
    merge_kernel<<<(unsigned)((long)a.B * a.Hq), kHeadDim, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace sd
