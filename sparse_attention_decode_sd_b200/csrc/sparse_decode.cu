// sparse_decode.cu -- exact attention over the selected rows of a paged GQA KV cache ("Sparse" mode
// of Fig. 1(a) of "Inference-time context sparsity: illusion or opportunity?"; SDPA of the xllm
// survey sec. 1.1 restricted to the selected set), and the dense comparator over every row
// ("Dense" mode of the same figure).
//
// Design (B200, HBM-bound gather):
//   * Work is split into 128-position granules of each (request, KV head) group.  The granules of
//     all groups form one sequence that is cut evenly across a persistent grid of warps (one wave),
//     so long, short and ragged contexts all balance.  The piece of a warp's range that falls in
//     one group is a "segment"; a warp keeps one online-softmax state per segment and writes one
//     partial (running max, sum, un-normalised output) per segment.  merge_kernel combines them
//     with a log-sum-exp merge.
//   * Each warp is an independent pipeline (no block barriers).  For every 1024-position chunk of
//     its segment it marks, in a shared-memory bitmap, which of the G query heads selected each
//     position (the union of the group's index lists), then streams the union rows in tiles of 16:
//     16-byte cp.async gathers of whole 256-byte K and V rows, addressed through the page table,
//     three tiles deep.  Every union row is read from HBM once for all heads of the group.
//   * Per tile: S^T = Q_group (16 heads) x K_tile^T and O += P x V_tile on the tensor cores
//     (mma.sync m16n8k16, bf16 inputs, fp32 accumulation; P is split into a bf16 high part and a
//     bf16 residual, so P is carried to ~16 significant bits), with heads that did not select a row
//     masked to -inf before an fp32 online softmax.
#include "common.cuh"
#include "kernels.h"

namespace sd {

constexpr int kGran = 128;     // granule of the balanced split (positions)
constexpr int kChunk = 1024;   // positions marked per bitmap rebuild
constexpr int kStages = 3;     // tiles in flight per warp
constexpr int kTileRows = 16;
constexpr int kPend = 64;      // ring of union rows found but not yet issued
constexpr int kTileBytes = kTileRows * kRowBytes;

constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;

struct __align__(128) WarpSmem {
    uint8_t kv[kStages][2][kTileBytes];       // K tile, V tile (16 rows x 256 B, 16-byte chunks XOR-swizzled)
    uint32_t meta_row[kStages][kTileRows];    // cache row index of each tile row
    uint32_t meta_mask[kStages][kTileRows];   // head bitmask of each tile row
    int info[kStages][8];                     // rows, flags, b, kvh, segment slot
    uint32_t mask[kChunk / 2];                // head bitmask per position of the chunk (16 bits each)
    int pt[kChunk / kPageSize];               // page-table entries of the chunk (-1: invalid)
    uint32_t pend_row[kPend];
    uint32_t pend_mask[kPend];
    int cursor[kMaxGroup];                    // per head: next unread idx entry
};

size_t decode_smem() { return sizeof(WarpSmem) * kDecodeWarpsPerCta; }

__device__ __forceinline__ int granules_of(int n) { return (n + kGran - 1) / kGran; }

// Sum over requests of Hkv * granules (the length of the flattened granule sequence); lengths are
// validated (an invalid one is reported and counts as 0).  Warp-cooperative.
__device__ __forceinline__ long total_granules(const DecodeArgs& a) {
    const int lane = threadIdx.x & 31;
    long tot = 0;
    for (int base = 0; base < a.B; base += 32) {
        const int r = base + lane;
        int v = 0;
        if (r < a.B) {
            const int n = a.lens[r];
            v = (n < 0 || (long)n > a.n_cap) ? 0 : a.Hkv * granules_of(n);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        tot += v;
    }
    return tot;
}

// Request containing global granule gs: returns b and the first global granule of b.
__device__ __forceinline__ void locate_granule(const DecodeArgs& a, long gs, int* b_out, long* rp_out) {
    const int lane = threadIdx.x & 31;
    long acc = 0;
    for (int base = 0; base < a.B; base += 32) {
        const int r = base + lane;
        int v = 0;
        if (r < a.B) {
            const int n = a.lens[r];
            v = (n < 0 || (long)n > a.n_cap) ? 0 : a.Hkv * granules_of(n);
        }
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        if (gs < acc + tot) {
            const uint32_t hit = __ballot_sync(0xffffffffu, acc + incl > gs);
            const int l = __ffs(hit) - 1;
            *b_out = base + l;
            *rp_out = acc + __shfl_sync(0xffffffffu, incl - v, l);
            return;
        }
        acc += tot;
    }
    *b_out = a.B;
    *rp_out = acc;
}

__device__ __forceinline__ int checked_len_silent(const DecodeArgs& a, int b) {
    const int n = a.lens[b];
    return (n < 0 || (long)n > a.n_cap) ? 0 : n;
}

// Producer-side state of one warp (all fields warp-uniform).
struct Walker {
    long gnext, gend, gpw;
    int warp_id;
    int b, gran, n;       // current request, its granules per group, its length
    long rp;              // first global granule of request b
    int kvh, seg_j, seg_lo, seg_hi;
    bool seg_open, seg_tiles, seg_done;
    int c0, c1, scan;
    int pend_head, pend_cnt;
};

// First index of an ascending, -1-padded list whose entry is >= target (padding counts as +inf).
// LPH lanes cooperate per head (heads 0..G-1 in parallel); the result is written to ws.cursor.
template <int LPH>
__device__ __forceinline__ void search_cursors(const DecodeArgs& a, int b, int kvh, int target, WarpSmem& ws) {
    const int lane = threadIdx.x & 31;
    const int hg = lane / LPH, sub = lane % LPH;
    const bool active = hg < a.G;
    const int32_t* list = a.idx + ((long)b * a.Hq + (long)kvh * a.G + (active ? hg : 0)) * a.k_max;
    int lo = 0, hi = a.k_max;   // the answer lies in [lo, hi]
    while (__any_sync(0xffffffffu, active && lo < hi)) {
        const bool busy = active && lo < hi;
        const int len = hi - lo;
        bool less = false;
        if (busy) {
            const int p = lo + (int)(((long)(sub + 1) * len) / (LPH + 1));
            const int v = __ldg(list + p);
            less = v >= 0 && v < target;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, busy && less);
        const int cnt = __popc((bal >> (hg * LPH)) & ((1u << LPH) - 1u));
        if (busy) {
            const int nlo = cnt > 0 ? lo + (int)(((long)cnt * len) / (LPH + 1)) + 1 : lo;
            const int nhi = cnt < LPH ? lo + (int)(((long)(cnt + 1) * len) / (LPH + 1)) : hi;
            lo = nlo;
            hi = nhi;
        }
    }
    if (active && sub == 0) ws.cursor[hg] = lo;
    __syncwarp();
}

template <bool DENSE>
__device__ __forceinline__ void open_segment(const DecodeArgs& a, Walker& w, WarpSmem& ws) {
    // advance to the request holding w.gnext
    while (w.gnext >= w.rp + (long)a.Hkv * w.gran) {
        w.rp += (long)a.Hkv * w.gran;
        ++w.b;
        w.n = checked_len_silent(a, w.b);
        w.gran = granules_of(w.n);
    }
    const long off = w.gnext - w.rp;
    w.kvh = (int)(off / w.gran);
    const int gi = (int)(off - (long)w.kvh * w.gran);
    const long g0 = w.rp + (long)w.kvh * w.gran;          // first global granule of the group
    const long seg_end = min(g0 + w.gran, w.gend);
    w.seg_lo = gi * kGran;
    w.seg_hi = (int)min((long)w.n, (long)(gi + (seg_end - w.gnext)) * kGran);
    w.seg_j = (int)(w.warp_id - g0 / w.gpw);
    w.gnext = seg_end;
    w.seg_open = true;
    w.seg_tiles = false;
    w.seg_done = false;
    w.c0 = w.c1 = w.scan = w.seg_lo;
    if (!DENSE) {
        if (a.G <= 8) search_cursors<4>(a, w.b, w.kvh, w.seg_lo, ws);
        else search_cursors<2>(a, w.b, w.kvh, w.seg_lo, ws);
    }
}

template <bool DENSE>
__device__ __forceinline__ void open_chunk(const DecodeArgs& a, Walker& w, WarpSmem& ws) {
    const int lane = threadIdx.x & 31;
    w.c0 = w.c1;
    w.c1 = min(w.c0 + kChunk, w.seg_hi);
    w.scan = w.c0;
    // page-table entries of the chunk (c0 is a multiple of the granule, hence of the page size)
    const int np = (w.c1 - w.c0 + kPageSize - 1) / kPageSize;
    const int32_t* ptrow = a.page_table + (long)w.b * a.max_pages + w.c0 / kPageSize;
    int pv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = lane + 32 * i;
        pv[i] = (e < np) ? __ldg(ptrow + e) : 0;
    }
    int lv[kMaxGroup];
    if (!DENSE) {
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            lv[g] = -1;
            if (g < a.G) {
                const int i = ws.cursor[g] + lane;
                if (i < a.k_max) lv[g] = __ldg(a.idx + ((long)w.b * a.Hq + (long)w.kvh * a.G + g) * a.k_max + i);
            }
        }
        uint4* m4 = reinterpret_cast<uint4*>(ws.mask);
#pragma unroll
        for (int i = 0; i < kChunk / 2 / 4 / 32; ++i) m4[lane + 32 * i] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = lane + 32 * i;
        if (e < np) {
            int page = pv[i];
            if (page < 0 || page >= a.num_pages) {
                report(a.status, SD_ERR_INDEX_OOB);
                page = -1;
            }
            ws.pt[e] = page;
        }
    }
    __syncwarp();
    if (!DENSE) {
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g >= a.G) break;
            int cur = ws.cursor[g];
            int v = lv[g];
            while (true) {
                const bool valid = v >= 0;
                const bool inr = valid && v >= w.c0 && v < w.c1;
                if (valid && v < w.c0) report(a.status, SD_ERR_ORDER);
                if (inr) {
                    const int o = v - w.c0;
                    atomicOr(&ws.mask[o >> 1], (1u << g) << ((o & 1) * 16));
                }
                const int nin = __popc(__ballot_sync(0xffffffffu, inr));
                cur += nin;
                if (nin < 32) break;
                const int i = cur + lane;
                v = (i < a.k_max) ? __ldg(a.idx + ((long)w.b * a.Hq + (long)w.kvh * a.G + g) * a.k_max + i) : -1;
            }
            // at the end of the request every remaining non-padding entry is >= N_b
            if (w.c1 == w.n && w.c1 == w.seg_hi) {
                const int i = cur + lane;
                const int rest = (i < a.k_max) ? __ldg(a.idx + ((long)w.b * a.Hq + (long)w.kvh * a.G + g) * a.k_max + i) : -1;
                if (__any_sync(0xffffffffu, rest >= 0)) report(a.status, SD_ERR_INDEX_OOB);
            }
            if (lane == 0) ws.cursor[g] = cur;
        }
        __syncwarp();
    }
}

// Finds union rows until 16 are pending or the segment is exhausted.
template <bool DENSE>
__device__ __forceinline__ void fill_pending(const DecodeArgs& a, Walker& w, WarpSmem& ws) {
    const int lane = threadIdx.x & 31;
    const uint32_t full_mask = (a.G >= 32) ? 0xffffffffu : ((1u << a.G) - 1u);
    while (w.pend_cnt < kTileRows && !w.seg_done) {
        if (w.scan >= w.c1) {
            if (w.c1 >= w.seg_hi) {
                w.seg_done = true;
                break;
            }
            open_chunk<DENSE>(a, w, ws);
        }
        const int p = w.scan + lane;
        uint32_t m = 0;
        int page = -1;
        if (p < w.c1) {
            const int o = p - w.c0;
            m = DENSE ? full_mask : ((ws.mask[o >> 1] >> ((o & 1) * 16)) & 0xffffu);
            page = ws.pt[o >> 4];
            if (page < 0) m = 0;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, m != 0);
        if (m != 0) {
            const int slot = (w.pend_head + w.pend_cnt + __popc(bal & ((1u << lane) - 1u))) & (kPend - 1);
            ws.pend_row[slot] = ((uint32_t)page * kPageSize + (uint32_t)(p & (kPageSize - 1))) * (uint32_t)a.Hkv + w.kvh;
            ws.pend_mask[slot] = m;
        }
        w.pend_cnt += __popc(bal);
        w.scan += 32;
    }
    __syncwarp();
}

// Assembles the next tile into `stage` and issues its K/V gathers (one cp.async group).
template <bool DENSE>
__device__ __forceinline__ void produce_tile(const DecodeArgs& a, Walker& w, WarpSmem& ws, int stage) {
    const int lane = threadIdx.x & 31;
    int rows = 0, flags = 0;
    if (!w.seg_open && w.gnext >= w.gend) {
        flags = kFlagEnd;
    } else {
        if (!w.seg_open) open_segment<DENSE>(a, w, ws);
        fill_pending<DENSE>(a, w, ws);
        rows = min(kTileRows, w.pend_cnt);
        flags = w.seg_tiles ? 0 : kFlagFirst;
        if (w.seg_done && w.pend_cnt == rows) flags |= kFlagLast;
        if (lane < kTileRows) {
            const int slot = (w.pend_head + lane) & (kPend - 1);
            ws.meta_row[stage][lane] = lane < rows ? ws.pend_row[slot] : 0u;
            ws.meta_mask[stage][lane] = lane < rows ? ws.pend_mask[slot] : 0u;
        }
        w.pend_head = (w.pend_head + rows) & (kPend - 1);
        w.pend_cnt -= rows;
        w.seg_tiles = true;
        if (flags & kFlagLast) w.seg_open = false;
    }
    if (lane == 0) {
        ws.info[stage][0] = rows;
        ws.info[stage][1] = flags;
        ws.info[stage][2] = w.b;
        ws.info[stage][3] = w.kvh;
        ws.info[stage][4] = w.seg_j;
    }
    __syncwarp();
    if (rows > 0) {
        const uint32_t kdst = smem_addr(ws.kv[stage][0]);
        const uint32_t vdst = smem_addr(ws.kv[stage][1]);
        const int ch = lane & 15;
#pragma unroll
        for (int i = 0; i < kTileRows / 2; ++i) {
            const int r = (lane >> 4) + 2 * i;
            const bool ok = r < rows;
            const size_t src = (size_t)(ok ? ws.meta_row[stage][r] : 0u) * kHeadDim + ch * 8;
            const uint32_t doff = (uint32_t)(r * kRowBytes + ((ch ^ (r & 7)) << 4));
            cp_async_16(kdst + doff, a.K + src, ok);
            cp_async_16(vdst + doff, a.V + src, ok);
        }
    }
    cp_async_commit();
}

// Consumer-side state of one warp.
struct Softmax {
    float m[2];          // running max (log2 units) of heads g and g+8
    float l[2];          // per-thread partial sums
    float acc[16][4];    // O fragment: heads g, g+8 x dims 8*nt + 2c, +1
    uint32_t qa[8][4];   // Q fragments (A operand) of the current group
};

__device__ __forceinline__ void reset_state(Softmax& st) {
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) st.acc[nt][0] = st.acc[nt][1] = st.acc[nt][2] = st.acc[nt][3] = 0.f;
}

__device__ __forceinline__ void load_q(const DecodeArgs& a, int b, int kvh, Softmax& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + g) * kHeadDim);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((long)b * a.Hq + (long)kvh * a.G + g + 8) * kHeadDim);
    const bool ok0 = g < a.G, ok1 = g + 8 < a.G;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        st.qa[j][0] = ok0 ? __ldg(q0 + 8 * j + c) : 0u;
        st.qa[j][1] = ok1 ? __ldg(q1 + 8 * j + c) : 0u;
        st.qa[j][2] = ok0 ? __ldg(q0 + 8 * j + c + 4) : 0u;
        st.qa[j][3] = ok1 ? __ldg(q1 + 8 * j + c + 4) : 0u;
    }
}

__device__ __forceinline__ void flush_state(const DecodeArgs& a, int b, int kvh, int seg_j, Softmax& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = st.l[e];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int hh = g + 8 * e;
        if (hh < a.G) {
            const long slot = ((long)b * a.Hq + (long)kvh * a.G + hh) * a.jmax + seg_j;
            if (c == 0) a.ml[slot] = make_float2(st.m[e], l);
            float2* dst = reinterpret_cast<float2*>(a.acc + slot * kHeadDim);
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) dst[4 * nt + c] = make_float2(st.acc[nt][2 * e], st.acc[nt][2 * e + 1]);
        }
    }
}

__device__ __forceinline__ void compute_tile(const DecodeArgs& a, const WarpSmem& ws, int stage, Softmax& st) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const uint32_t kbase = smem_addr(ws.kv[stage][0]);
    const uint32_t vbase = smem_addr(ws.kv[stage][1]);
    const int mi = lane >> 3, r8 = lane & 7;

    // S^T (16 heads x 16 rows) = Q x K^T
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
        const int r = ((mi >> 1) << 3) + r8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ch = 2 * j + (mi & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(kbase + r * kRowBytes + ((ch ^ (r & 7)) << 4), b0, b1, b2, b3);
            mma_bf16_16816(s0, st.qa[j][0], st.qa[j][1], st.qa[j][2], st.qa[j][3], b0, b1);
            mma_bf16_16816(s1, st.qa[j][0], st.qa[j][1], st.qa[j][2], st.qa[j][3], b2, b3);
        }
    }
    // mask heads that did not select a row; scale to log2 units
    const uint32_t mk0 = ws.meta_mask[stage][2 * c], mk1 = ws.meta_mask[stage][2 * c + 1];
    const uint32_t mk2 = ws.meta_mask[stage][2 * c + 8], mk3 = ws.meta_mask[stage][2 * c + 9];
    float z[2][4];   // [head g / g+8][rows 2c, 2c+1, 2c+8, 2c+9]
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int hh = g + 8 * e;
        z[e][0] = ((mk0 >> hh) & 1u) ? s0[2 * e] * a.scale_log2 : -INFINITY;
        z[e][1] = ((mk1 >> hh) & 1u) ? s0[2 * e + 1] * a.scale_log2 : -INFINITY;
        z[e][2] = ((mk2 >> hh) & 1u) ? s1[2 * e] * a.scale_log2 : -INFINITY;
        z[e][3] = ((mk3 >> hh) & 1u) ? s1[2 * e + 1] * a.scale_log2 : -INFINITY;
    }
    float p[2][4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float tm = fmaxf(fmaxf(z[e][0], z[e][1]), fmaxf(z[e][2], z[e][3]));
        tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
        tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
        const float mn = fmaxf(st.m[e], tm);
        const bool none = mn == -INFINITY;
        const float alpha = none ? 1.f : exp2f(st.m[e] - mn);
        const float base = none ? 0.f : mn;
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            p[e][r] = exp2f(z[e][r] - base);
            sum += p[e][r];
        }
        st.m[e] = mn;
        st.l[e] = st.l[e] * alpha + sum;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            st.acc[nt][2 * e] *= alpha;
            st.acc[nt][2 * e + 1] *= alpha;
        }
    }
    // P (A operand: 16 heads x 16 rows) as bf16 high part + bf16 residual
    uint32_t ph[4], pl[4];
    {
        const float v[4][2] = {{p[0][0], p[0][1]}, {p[1][0], p[1][1]}, {p[0][2], p[0][3]}, {p[1][2], p[1][3]}};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ph[i] = pack_bf16x2(v[i][0], v[i][1]);
            pl[i] = pack_bf16x2(v[i][0] - bf16_lo(ph[i]), v[i][1] - bf16_hi(ph[i]));
        }
    }
    // O += P x V
    {
        const int r = ((mi & 1) << 3) + r8;
#pragma unroll
        for (int ntp = 0; ntp < 8; ++ntp) {
            const int ch = 2 * ntp + (mi >> 1);
            uint32_t v0, v1, v2, v3;
            ldmatrix_x4_trans(vbase + r * kRowBytes + ((ch ^ (r & 7)) << 4), v0, v1, v2, v3);
            mma_bf16_16816(st.acc[2 * ntp], ph[0], ph[1], ph[2], ph[3], v0, v1);
            mma_bf16_16816(st.acc[2 * ntp], pl[0], pl[1], pl[2], pl[3], v0, v1);
            mma_bf16_16816(st.acc[2 * ntp + 1], ph[0], ph[1], ph[2], ph[3], v2, v3);
            mma_bf16_16816(st.acc[2 * ntp + 1], pl[0], pl[1], pl[2], pl[3], v2, v3);
        }
    }
}

template <bool DENSE>
__global__ void __launch_bounds__(kDecodeWarpsPerCta * 32, 2) decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem)[warp];

    const long Tg = total_granules(a);
    if (Tg == 0) return;
    Walker w;
    w.warp_id = blockIdx.x * kDecodeWarpsPerCta + warp;
    w.gpw = (Tg + a.total_warps - 1) / a.total_warps;
    w.gnext = (long)w.warp_id * w.gpw;
    w.gend = min(Tg, w.gnext + w.gpw);
    if (w.gnext >= w.gend) return;
    locate_granule(a, w.gnext, &w.b, &w.rp);
    w.n = checked_len_silent(a, w.b);
    w.gran = granules_of(w.n);
    w.seg_open = false;
    w.pend_head = w.pend_cnt = 0;
    w.kvh = w.seg_j = 0;

    Softmax st;
    reset_state(st);
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) produce_tile<DENSE>(a, w, ws, s);
    for (int t = 0;; ++t) {
        cp_async_wait<kStages - 2>();
        __syncwarp();
        const int stage = t % kStages;
        const int rows = ws.info[stage][0], flags = ws.info[stage][1];
        if (flags & kFlagEnd) break;
        const int tb = ws.info[stage][2], tkvh = ws.info[stage][3], tj = ws.info[stage][4];
        produce_tile<DENSE>(a, w, ws, (t + kStages - 1) % kStages);
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

// One warp per (b, h): log-sum-exp merge of the segment partials of its group.
__global__ void __launch_bounds__(128) merge_kernel(DecodeArgs a) {
    const int lane = threadIdx.x & 31;
    const long bh = (long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (bh >= (long)a.B * a.Hq) return;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq), kvh = h / a.G;
    const int n = checked_len(a.lens, b, a.n_cap, a.status);
    float4* out = reinterpret_cast<float4*>(a.out + bh * kHeadDim);
    if (n == 0) {
        out[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    const long Tg = total_granules(a);
    long rp = 0;   // first global granule of request b: sum over earlier requests
    for (int base = 0; base < b; base += 32) {
        const int r = base + lane;
        int v = (r < b) ? a.Hkv * granules_of(checked_len_silent(a, r)) : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        rp += v;
    }
    const int gran = granules_of(n);
    const long gfirst = rp + (long)kvh * gran;
    const long gpw = (Tg + a.total_warps - 1) / a.total_warps;
    const int nseg = (int)((gfirst + gran - 1) / gpw - gfirst / gpw + 1);
    const float2* ml = a.ml + bh * a.jmax;
    const float* accp = a.acc + bh * a.jmax * kHeadDim;
    float M = -INFINITY;
    for (int j = lane; j < nseg; j += 32) M = fmaxf(M, ml[j].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
        for (int j = 0; j < nseg; ++j) {
            const float2 v = ml[j];
            if (v.x == -INFINITY) continue;
            const float wgt = exp2f(v.x - M);
            L += wgt * v.y;
            const float4 x = reinterpret_cast<const float4*>(accp + (long)j * kHeadDim)[lane];
            o4.x += wgt * x.x;
            o4.y += wgt * x.y;
            o4.z += wgt * x.z;
            o4.w += wgt * x.w;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    out[lane] = make_float4(o4.x * inv, o4.y * inv, o4.z * inv, o4.w * inv);
}

cudaError_t decode_occupancy(int* ctas_per_sm) {
    const size_t smem = decode_smem();
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_kernel<false>, kDecodeWarpsPerCta * 32,
                                                         smem);
}

cudaError_t launch_decode(const DecodeArgs& a, bool dense, int ctas, cudaStream_t stream) {
    const size_t smem = decode_smem();
    if (dense) decode_kernel<true><<<ctas, kDecodeWarpsPerCta * 32, smem, stream>>>(a);
    else decode_kernel<false><<<ctas, kDecodeWarpsPerCta * 32, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream) {
    const long rows = (long)a.B * a.Hq;
    merge_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace sd
