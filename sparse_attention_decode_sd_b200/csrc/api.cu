// api.cu -- the C ABI of libsparsedecode (declared in include/sparsedecode.h): host-side argument
// validation, workspace layout, launch configuration and status codes.  No allocation, no state
// beyond a per-device cache of the SM count and decode occupancy.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace sd;

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kSmemBudget = 227 * 1024;   // opt-in shared memory per CTA on sm_100
constexpr int kSelectCapMax = 24 * 1024;      // select: candidate entries kept in shared memory
constexpr size_t kScoreStageBytes = 65536;    // score pass: bytes per pipeline stage (whole pages)

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int decode_ctas_per_sm[2][2] = {{0, 0}, {0, 0}};   // [dense][G > 8]
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

sd_status device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SD_ERR_CUDA;
        for (int dense = 0; dense < 2; ++dense)
            for (int wide = 0; wide < 2; ++wide) {
                int ctas = 0;
                if (decode_occupancy(dense != 0, wide ? 16 : 8, &ctas) != cudaSuccess || ctas < 1) return SD_ERR_CUDA;
                d.decode_ctas_per_sm[dense][wide] = ctas;
            }
        d.sms = sms;
        d.ready = true;
    }
    *out = d;
    return SD_OK;
}

struct Dims {
    int B, Hq, Hkv, G, max_pages, k_max, num_pages;
    long n_cap;   // max_pages * page size
    int nrp;      // dense decode: counted ranges per (b, kv head) group
    int nrt;      // B * Hkv * nrp
    int jmax;     // dense decode: segment slots per (b, h)
};

sd_status check_shape(const sd_shape* s, Dims* d) {
    if (s == nullptr) return SD_ERR_INVALID_ARG;
    if (s->batch < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1 || s->max_pages_per_req < 1 || s->k_max < 1 ||
        s->num_pages < 1)
        return SD_ERR_INVALID_ARG;
    if (s->num_q_heads % s->num_kv_heads != 0) return SD_ERR_INVALID_ARG;
    if (s->head_dim != kHeadDim || s->page_size != kPageSize) return SD_ERR_UNSUPPORTED;
    const int G = s->num_q_heads / s->num_kv_heads;
    if (G > kMaxGroup || s->num_kv_heads > 16 || s->batch > kMaxBatch) return SD_ERR_UNSUPPORTED;
    const long n_cap = (long)s->max_pages_per_req * kPageSize;
    if (n_cap > (1L << 30)) return SD_ERR_UNSUPPORTED;
    // cache rows are indexed in 32 bits, and as signed TMA coordinates by the sparse decode
    if ((long)s->num_pages * kPageSize * s->num_kv_heads >= (1L << 31)) return SD_ERR_UNSUPPORTED;
    const long nr = (n_cap + kRange - 1) / kRange;
    const long nrt = (long)s->batch * s->num_kv_heads * nr;
    if (nrt * kRange >= (1L << 31)) return SD_ERR_UNSUPPORTED;   // rows are counted in int32
    d->B = s->batch;
    d->Hq = s->num_q_heads;
    d->Hkv = s->num_kv_heads;
    d->G = G;
    d->max_pages = s->max_pages_per_req;
    d->k_max = s->k_max;
    d->num_pages = s->num_pages;
    d->n_cap = n_cap;
    d->nrp = (int)nr;
    d->nrt = (int)nrt;
    d->jmax = (int)((n_cap < kMaxDecodeWarps ? n_cap : kMaxDecodeWarps) + 1);
    return SD_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// indexer workspace, in order: candidate streams (B*Hq*n_cap fp32), per-(head, page) records
// {stream offset, candidate mask} [B][Hq][mstride] uint2, thresholds [B][Hq] fp32, input pointers [3]
long topk_mstride(const Dims& d) { return ((long)d.max_pages + 7) & ~7L; }
struct TopkLayout {
    size_t cand, prec, tau, inputs, total;
};
TopkLayout topk_layout(const Dims& d) {
    TopkLayout L;
    const size_t rows = (size_t)d.B * d.Hq;
    L.cand = 0;
    L.prec = align256(rows * d.n_cap * sizeof(float));
    L.tau = L.prec + align256(rows * topk_mstride(d) * sizeof(uint2));
    L.inputs = L.tau + align256(rows * sizeof(float));
    L.total = L.inputs + align256(3 * sizeof(void*));
    return L;
}
size_t topk_workspace(const Dims& d) { return topk_layout(d).total; }

// dense decode workspace, in order: acc [B][Hq][jmax][128] fp32, ml [B][Hq][jmax] float2, counts [nrt]
struct DenseLayout {
    size_t acc, ml, counts, total;
};
DenseLayout dense_layout(const Dims& d) {
    DenseLayout L;
    const size_t slots = (size_t)d.B * d.Hq * d.jmax;
    L.acc = 0;
    L.ml = L.acc + align256(slots * kHeadDim * sizeof(float));
    L.counts = L.ml + align256(slots * sizeof(float2));
    L.total = L.counts + align256((size_t)d.nrt * sizeof(int));
    return L;
}

// sparse decode: rows_kernel shape (threads per row: enough warps for kRowBatch entries each, up to
// 1024; CTAs of at least 256 threads when rows are short) and its workspace, in order:
// acc [B][Hq][kRowSegs][128] fp32, ml [B][Hq][kRowSegs] float2, rlen [B*Hq], arrive [B*Hq], bsum [nb],
// rlw [B*Hq] fp32
struct SparseLayout {
    int tpr, rpc, nb;
    size_t acc, ml, rlen, arrive, bsum, rlw, total;
};
SparseLayout sparse_layout(const Dims& d) {
    SparseLayout L;
    const long rows = (long)d.B * d.Hq;
    const long need = ((long)d.k_max + kRowBatch - 1) / kRowBatch;   // threads for one pass over a row
    long tpr = (need + 31) / 32 * 32;
    if (tpr > 1024) tpr = 1024;
    L.tpr = (int)tpr;
    L.rpc = tpr >= 256 ? 1 : (int)(256 / tpr);
    L.nb = (int)((rows + L.rpc - 1) / L.rpc);
    const size_t slots = (size_t)rows * kRowSegs;
    L.acc = 0;
    L.ml = L.acc + align256(slots * kHeadDim * sizeof(float));
    L.rlen = L.ml + align256(slots * sizeof(float2));
    L.arrive = L.rlen + align256((size_t)rows * sizeof(int));
    L.bsum = L.arrive + align256((size_t)rows * sizeof(int));
    L.rlw = L.bsum + align256((size_t)L.nb * sizeof(int));
    L.total = L.rlw + align256((size_t)rows * sizeof(float));
    return L;
}
// entries of all rows are counted in int32
bool sparse_fits(const Dims& d) { return (long)d.B * d.Hq * d.k_max < (1L << 31); }

// The sparse decode walks GQA groups (one gathered row serves every head of the group that selected
// it) instead of heads when the shape says the heads' selections overlap heavily: with a fraction
// f = k_max / capacity selected per head, independent selections of the G heads would have the
// group read G f N rows per head walk against (1 - (1 - f)^G) N rows of their union.
// Expected duplication of a GQA group's selections: entries per distinct position when each head
// selects a fraction f = k_max / capacity of the positions independently, G f / (1 - (1 - f)^G).
double expected_duplication(const Dims& d) {
    const double f = d.n_cap > 0 ? (double)d.k_max / (double)d.n_cap : 1.0;
    const double fc = f < 1.0 ? f : 1.0;
    const double uni = 1.0 - pow(1.0 - fc, (double)d.G);
    return uni > 0.0 ? d.G * fc / uni : 1.0;
}
constexpr double kUnionDuplication = 1.4;   // from here on, one gathered tile serves a group's heads
constexpr double kOrderDuplication = 1.1;   // from here on, the per-head walk aligns a group's heads
bool use_group_walk(const Dims& d) { return expected_duplication(d) >= kUnionDuplication; }
// Expected fraction of a group's positions that some head selects: 1 - (1 - f)^G.
double expected_coverage(const Dims& d) {
    const double f = d.n_cap > 0 ? (double)d.k_max / (double)d.n_cap : 1.0;
    return 1.0 - pow(1.0 - (f < 1.0 ? f : 1.0), (double)d.G);
}
constexpr double kUnionTilesCoverage = 0.9;   // from here on, the group walk takes whole tiles

// sparse decode over GQA groups: the row pass's part of the sparse layout, then the dense layout,
// then the groups' selection masks [B*Hkv][n_cap] (1 byte per position for G <= 8, else 2)
struct UnionLayout {
    SparseLayout rows;
    DenseLayout grp;
    size_t base_grp, umask, total;
};
UnionLayout union_layout(const Dims& d) {
    UnionLayout L;
    L.rows = sparse_layout(d);
    L.grp = dense_layout(d);
    L.base_grp = L.rows.total;
    L.umask = L.base_grp + L.grp.total;
    L.total = L.umask + align256((size_t)d.B * d.Hkv * d.n_cap * (d.G <= 8 ? 1 : 2));
    return L;
}

size_t decode_workspace(const Dims& d, bool dense) {
    if (dense) return dense_layout(d).total;
    return use_group_walk(d) ? union_layout(d).total : sparse_layout(d).total;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

long d_k_max_of(const sd_shape* s) { return s ? (long)s->k_max : 0; }

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

sd_status launch_status(cudaError_t e) {
    if (e == cudaSuccess) return SD_OK;
    g_last_cuda_error = e;
    return SD_ERR_CUDA;
}

sd_status decode_common(const sd_shape* shape, const void* q, const void* K, const void* V, const int32_t* page_table,
                        const int32_t* lens, const int32_t* idx, float* out, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream, bool dense, bool weighted = false) {
    Dims d;
    sd_status st = check_shape(shape, &d);
    if (st != SD_OK) return st;
    if (!q || !K || !V || !page_table || !lens || !out || !workspace || !dev_status || (!dense && !idx))
        return SD_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
        !aligned(page_table, 4) || !aligned(lens, 4) || (!dense && !aligned(idx, 4)) || !aligned(dev_status, 4))
        return SD_ERR_INVALID_ARG;
    if (!dense && !sparse_fits(d)) return SD_ERR_UNSUPPORTED;
    if (workspace_bytes < decode_workspace(d, dense)) return SD_ERR_WORKSPACE;
    DeviceInfo di;
    st = device_info(&di);
    if (st != SD_OK) return st;
    DecodeArgs a = {};
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.K = static_cast<const __nv_bfloat16*>(K);
    a.V = static_cast<const __nv_bfloat16*>(V);
    a.page_table = page_table;
    a.lens = lens;
    a.idx = dense ? nullptr : idx;
    a.out = out;
    a.status = dev_status;
    a.B = d.B;
    a.Hq = d.Hq;
    a.Hkv = d.Hkv;
    a.G = d.G;
    a.max_pages = d.max_pages;
    a.num_pages = d.num_pages;
    a.k_max = dense ? 0 : d.k_max;
    a.n_cap = d.n_cap;
    a.nrp = d.nrp;
    a.nrt = d.nrt;
    int warps = di.sms * di.decode_ctas_per_sm[dense ? 1 : 0][d.G > 8 ? 1 : 0];
    const int cap = dense ? kMaxDecodeWarps : kMaxSparseWarps;
    if (warps > cap) warps = cap;
    a.total_warps = warps;   // one warp per CTA
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)kHeadDim));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dense) {
        const DenseLayout L = dense_layout(d);
        a.acc = reinterpret_cast<float*>(ws + L.acc);
        a.ml = reinterpret_cast<float2*>(ws + L.ml);
        a.counts = reinterpret_cast<int*>(ws + L.counts);
        a.jmax = d.jmax;
        return launch_status(launch_dense(a, s));
    }
    if (use_group_walk(d) && !weighted) {   // (drawn rows are weighted by the per-head walk, whose
                                             // workspace lies at the start of this layout)
        const UnionLayout U = union_layout(d);
        a.rlen = reinterpret_cast<int*>(ws + U.rows.rlen);
        a.arrive = reinterpret_cast<int*>(ws + U.rows.arrive);
        a.bsum = reinterpret_cast<int*>(ws + U.rows.bsum);
        a.rlw = reinterpret_cast<float*>(ws + U.rows.rlw);
        a.tpr = U.rows.tpr;
        a.rpc = U.rows.rpc;
        a.nb = U.rows.nb;
        a.weighted = weighted ? 1 : 0;
        a.acc = reinterpret_cast<float*>(ws + U.base_grp + U.grp.acc);
        a.ml = reinterpret_cast<float2*>(ws + U.base_grp + U.grp.ml);
        a.counts = reinterpret_cast<int*>(ws + U.base_grp + U.grp.counts);
        a.umask = ws + U.umask;
        a.jmax = d.jmax;
        a.union_tiles = expected_coverage(d) >= kUnionTilesCoverage ? 1 : 0;
        int gw = di.sms * di.decode_ctas_per_sm[1][d.G > 8 ? 1 : 0];
        a.total_warps = gw > kMaxDecodeWarps ? kMaxDecodeWarps : gw;
        return launch_status(launch_sparse_union(a, s));
    }
    const SparseLayout L = sparse_layout(d);
    a.acc = reinterpret_cast<float*>(ws + L.acc);
    a.ml = reinterpret_cast<float2*>(ws + L.ml);
    a.rlen = reinterpret_cast<int*>(ws + L.rlen);
    a.arrive = reinterpret_cast<int*>(ws + L.arrive);
    a.bsum = reinterpret_cast<int*>(ws + L.bsum);
    a.rlw = reinterpret_cast<float*>(ws + L.rlw);
    a.weighted = weighted ? 1 : 0;
    a.tpr = L.tpr;
    a.rpc = L.rpc;
    a.nb = L.nb;
    a.jmax = kRowSegs;
    a.order_rows = (d.G > 1 && (long)d.B * d.Hq <= kOrderMaxRows && expected_duplication(d) >= kOrderDuplication) ? 1 : 0;
    a.min_epw = (d.k_max + kRowSegs - 2) / (kRowSegs - 1);   // ceil(k_max / (kRowSegs - 1))
    return launch_status(launch_sparse(a, s));
}

}  // namespace

extern "C" {

sd_status sd_workspace_size(const sd_shape* shape, int32_t op, size_t* bytes) {
    if (bytes == nullptr) return SD_ERR_INVALID_ARG;
    Dims d;
    sd_status st = check_shape(shape, &d);
    if (st != SD_OK) return st;
    switch (op) {
        case SD_OP_TOPK: *bytes = topk_workspace(d); return SD_OK;
        case SD_OP_SPARSE:
            if (!sparse_fits(d)) return SD_ERR_UNSUPPORTED;
            *bytes = decode_workspace(d, false);
            return SD_OK;
        case SD_OP_DENSE: *bytes = decode_workspace(d, true); return SD_OK;
        case SD_OP_QUEST: *bytes = align256((size_t)d.B * d.Hq * d.max_pages * sizeof(float)); return SD_OK;
        default: return SD_ERR_INVALID_ARG;
    }
}

namespace {

sd_status topk_args(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                    const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace, size_t workspace_bytes,
                    int32_t* dev_status, bool need_scores_inputs, bool need_idx, TopkArgs* a, DeviceInfo* di) {
    Dims d;
    sd_status st = check_shape(shape, &d);
    if (st != SD_OK) return st;
    if (!lens || !k || !workspace || !dev_status) return SD_ERR_INVALID_ARG;
    if (need_scores_inputs && (!q || !K || !page_table)) return SD_ERR_INVALID_ARG;
    if (need_idx && !idx) return SD_ERR_INVALID_ARG;
    if ((need_scores_inputs && (!aligned(q, 16) || !aligned(K, 16) || !aligned(page_table, 4))) ||
        (need_idx && !aligned(idx, 4)) || !aligned(workspace, 256) || !aligned(lens, 4) || !aligned(k, 4) ||
        !aligned(dev_status, 4))
        return SD_ERR_INVALID_ARG;
    if (workspace_bytes < topk_workspace(d)) return SD_ERR_WORKSPACE;
    st = device_info(di);
    if (st != SD_OK) return st;
    a->q = static_cast<const __nv_bfloat16*>(q);
    a->K = static_cast<const __nv_bfloat16*>(K);
    a->page_table = page_table;
    a->lens = lens;
    a->k = k;
    a->idx = idx;
    const TopkLayout L = topk_layout(d);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if ((long)d.B * d.Hq * d.n_cap >= (1L << 32)) return SD_ERR_UNSUPPORTED;   // stream offsets are 32-bit
    a->cand = reinterpret_cast<float*>(ws + L.cand);
    a->prec = reinterpret_cast<uint2*>(ws + L.prec);
    a->tau = reinterpret_cast<float*>(ws + L.tau);
    a->inputs = reinterpret_cast<const void**>(ws + L.inputs);
    a->mstride = (int)topk_mstride(d);
    // Rows with N_b <= 3 k_max + 4096 take every position as a candidate; longer rows keep the
    // scores at or above a sampled threshold.
    const long ccap = 3L * d.k_max + 4096;
    a->ccap = (int)(ccap < d.n_cap ? ccap : d.n_cap);
    a->status = dev_status;
    a->B = d.B;
    a->Hq = d.Hq;
    a->Hkv = d.Hkv;
    a->G = d.G;
    a->max_pages = d.max_pages;
    a->num_pages = d.num_pages;
    a->k_max = d.k_max;
    a->n_cap = d.n_cap;
    // score pass: pipeline stages of whole pages, about kScoreStageBytes each, as many as the shared
    // memory holds (2 to 6)
    const size_t page_bytes = (size_t)kPageSize * d.Hkv * kRowBytes;
    a->spp = (int)(page_bytes >= kScoreStageBytes ? 1 : kScoreStageBytes / page_bytes);
    const size_t fixed = sizeof(int) * (d.B + 1 + 40) + 1024;
    const size_t stage_bytes = page_bytes * a->spp;
    a->stages = (int)((kSmemBudget - fixed) / (stage_bytes + 2 * sizeof(uint64_t)));
    if (a->stages > 6) a->stages = 6;
    if (a->stages < 2) return SD_ERR_UNSUPPORTED;
    // select: candidate capacity from k_max, bounded by shared memory
    long cap = (long)d.k_max + d.k_max / 2 + 4096;
    if (cap > kSelectCapMax) cap = kSelectCapMax;
    a->cap = (int)cap;
    return SD_OK;
}

}  // namespace

sd_status sd_topk_scores(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                         const int32_t* lens, const int32_t* k, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream) {
    TopkArgs a;
    DeviceInfo di;
    sd_status st = topk_args(shape, q, K, page_table, lens, k, nullptr, workspace, workspace_bytes, dev_status, true,
                             false, &a, &di);
    if (st != SD_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_status(launch_threshold(a, s));
    if (st != SD_OK) return st;
    return launch_status(launch_score_pass(a, di.sms, s));
}

sd_status sd_topk_select(const sd_shape* shape, const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace,
                         size_t workspace_bytes, int32_t* dev_status, void* stream) {
    TopkArgs a;
    DeviceInfo di;
    sd_status st = topk_args(shape, nullptr, nullptr, nullptr, lens, k, idx, workspace, workspace_bytes, dev_status,
                             false, true, &a, &di);
    if (st != SD_OK) return st;
    return launch_status(launch_select(a, static_cast<cudaStream_t>(stream)));
}

sd_status sd_topk_index(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                        const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream) {
    TopkArgs a;
    DeviceInfo di;
    sd_status st = topk_args(shape, q, K, page_table, lens, k, idx, workspace, workspace_bytes, dev_status, true, true,
                             &a, &di);
    if (st != SD_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_status(launch_threshold(a, s));
    if (st != SD_OK) return st;
    st = launch_status(launch_score_pass(a, di.sms, s));
    if (st != SD_OK) return st;
    return launch_status(launch_select(a, s));
}

sd_status sd_sparse_decode(const sd_shape* shape, const void* q, const void* K, const void* V,
                           const int32_t* page_table, const int32_t* lens, const int32_t* idx, float* out,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return decode_common(shape, q, K, V, page_table, lens, idx, out, workspace, workspace_bytes, dev_status, stream,
                         false);
}

sd_status sd_sparse_decode_sampled(const sd_shape* shape, const void* q, const void* K, const void* V,
                                   const int32_t* page_table, const int32_t* lens, const int32_t* idx, float* out,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return decode_common(shape, q, K, V, page_table, lens, idx, out, workspace, workspace_bytes, dev_status, stream,
                         false, true);
}

sd_status sd_stochastic_index(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                              const int32_t* lens, const int32_t* k_det, const int32_t* k_samp, uint64_t seed,
                              uint32_t step, int32_t* idx, void* workspace, size_t workspace_bytes,
                              int32_t* dev_status, void* stream) {
    if (!k_samp || !aligned(k_samp, 4)) return SD_ERR_INVALID_ARG;
    TopkArgs a;
    DeviceInfo di;
    sd_status st = topk_args(shape, q, K, page_table, lens, k_det, idx, workspace, workspace_bytes, dev_status, true,
                             true, &a, &di);
    if (st != SD_OK) return st;
    SampleArgs sa = {};
    sa.lens = lens;
    sa.k_det = k_det;
    sa.k_samp = k_samp;
    sa.idx = idx;
    sa.status = dev_status;
    sa.seed = seed;
    sa.step = step;
    sa.B = a.B;
    sa.Hq = a.Hq;
    sa.k_max = a.k_max;
    sa.n_cap = a.n_cap;
    sa.words = (int)((a.n_cap + 31) / 32);
    // candidates: what shared memory holds next to two position bitmaps, the radix histogram and
    // the scan state; at least twice k_max (the threshold aims at about m + 6 sqrt(m) + 32 of them)
    sa.cap = 0;
    const size_t fixed = sample_smem(sa);
    if (fixed >= kSmemBudget) return SD_ERR_UNSUPPORTED;
    const long cap = (long)((kSmemBudget - fixed) / (sizeof(uint32_t) + 2 * sizeof(int)));
    if (cap < 2L * d_k_max_of(shape) + 1024) return SD_ERR_UNSUPPORTED;
    sa.cap = (int)(cap > (1 << 20) ? (1 << 20) : cap);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_status(launch_threshold(a, s));
    if (st != SD_OK) return st;
    st = launch_status(launch_score_pass(a, di.sms, s));
    if (st != SD_OK) return st;
    st = launch_status(launch_select(a, s));
    if (st != SD_OK) return st;
    return launch_status(launch_sample(sa, s));
}

sd_status sd_dense_decode(const sd_shape* shape, const void* q, const void* K, const void* V,
                          const int32_t* page_table, const int32_t* lens, float* out, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return decode_common(shape, q, K, V, page_table, lens, nullptr, out, workspace, workspace_bytes, dev_status,
                         stream, true);
}

namespace {
sd_status append_common(const sd_shape* shape, void* K, void* V, const int32_t* page_table, int32_t* lens,
                        const void* k_new, const void* v_new, int32_t* k_sel, int32_t ratio, void* boxes,
                        int32_t* dev_status, void* stream) {
    Dims d;
    sd_status st = check_shape(shape, &d);
    if (st != SD_OK) return st;
    if (!K || !V || !page_table || !lens || !k_new || !v_new || !dev_status || ratio < 1) return SD_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(page_table, 4) ||
        !aligned(lens, 4) || (k_sel && !aligned(k_sel, 4)) || !aligned(dev_status, 4))
        return SD_ERR_INVALID_ARG;
    AppendArgs a;
    a.K = static_cast<__nv_bfloat16*>(K);
    a.V = static_cast<__nv_bfloat16*>(V);
    a.page_table = page_table;
    a.lens = lens;
    a.k_new = static_cast<const __nv_bfloat16*>(k_new);
    a.v_new = static_cast<const __nv_bfloat16*>(v_new);
    a.k_sel = k_sel;
    a.boxes = static_cast<__nv_bfloat16*>(boxes);
    a.status = dev_status;
    a.B = d.B;
    a.Hkv = d.Hkv;
    a.max_pages = d.max_pages;
    a.num_pages = d.num_pages;
    a.ratio = ratio;
    return launch_status(launch_append(a, static_cast<cudaStream_t>(stream)));
}
}  // namespace

sd_status sd_append_kv(const sd_shape* shape, void* K, void* V, const int32_t* page_table, int32_t* lens,
                       const void* k_new, const void* v_new, int32_t* k_sel, int32_t ratio, int32_t* dev_status,
                       void* stream) {
    return append_common(shape, K, V, page_table, lens, k_new, v_new, k_sel, ratio, nullptr, dev_status, stream);
}

sd_status sd_quest_append_kv(const sd_shape* shape, void* K, void* V, const int32_t* page_table, int32_t* lens,
                             const void* k_new, const void* v_new, int32_t* k_sel, int32_t ratio, void* boxes,
                             int32_t* dev_status, void* stream) {
    if (boxes == nullptr || !aligned(boxes, 16)) return SD_ERR_INVALID_ARG;
    return append_common(shape, K, V, page_table, lens, k_new, v_new, k_sel, ratio, boxes, dev_status, stream);
}

namespace {

sd_status quest_args(const sd_shape* shape, QuestArgs* a, Dims* d) {
    sd_status st = check_shape(shape, d);
    if (st != SD_OK) return st;
    *a = QuestArgs{};
    a->B = d->B;
    a->Hq = d->Hq;
    a->Hkv = d->Hkv;
    a->G = d->G;
    a->max_pages = d->max_pages;
    a->num_pages = d->num_pages;
    a->k_max = d->k_max;
    a->n_cap = d->n_cap;
    return SD_OK;
}

}  // namespace

sd_status sd_quest_summarize(const sd_shape* shape, const void* K, const int32_t* page_table, const int32_t* lens,
                             void* boxes, int32_t last_page_only, int32_t* dev_status, void* stream) {
    QuestArgs a;
    Dims d;
    sd_status st = quest_args(shape, &a, &d);
    if (st != SD_OK) return st;
    if (!K || !page_table || !lens || !boxes || !dev_status) return SD_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(boxes, 16) || !aligned(page_table, 4) || !aligned(lens, 4) ||
        !aligned(dev_status, 4))
        return SD_ERR_INVALID_ARG;
    if (!last_page_only && (long)d.B * d.max_pages * d.Hkv >= (1L << 36)) return SD_ERR_UNSUPPORTED;
    a.K = static_cast<const __nv_bfloat16*>(K);
    a.boxes = static_cast<__nv_bfloat16*>(boxes);
    a.page_table = page_table;
    a.lens = lens;
    a.status = dev_status;
    a.last_only = last_page_only ? 1 : 0;
    return launch_status(launch_quest_summarize(a, static_cast<cudaStream_t>(stream)));
}

sd_status sd_quest_index(const sd_shape* shape, const void* q, const void* boxes, const int32_t* page_table,
                         const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream) {
    QuestArgs a;
    Dims d;
    sd_status st = quest_args(shape, &a, &d);
    if (st != SD_OK) return st;
    if (!q || !boxes || !page_table || !lens || !k || !idx || !workspace || !dev_status) return SD_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(boxes, 16) || !aligned(page_table, 4) || !aligned(lens, 4) || !aligned(k, 4) ||
        !aligned(idx, 4) || !aligned(workspace, 256) || !aligned(dev_status, 4))
        return SD_ERR_INVALID_ARG;
    if (d.max_pages > kQuestMaxPages) return SD_ERR_UNSUPPORTED;
    size_t need = 0;
    sd_workspace_size(shape, SD_OP_QUEST, &need);
    if (workspace_bytes < need) return SD_ERR_WORKSPACE;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.boxes = const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(boxes));
    a.page_table = page_table;
    a.lens = lens;
    a.k = k;
    a.idx = idx;
    a.rel = static_cast<float*>(workspace);
    a.status = dev_status;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_status(launch_quest_score(a, s));
    if (st != SD_OK) return st;
    return launch_status(launch_quest_select(a, s));
}

const char* sd_status_string(sd_status status) {
    switch (status) {
        case SD_OK: return "ok";
        case SD_ERR_INVALID_ARG: return "invalid argument";
        case SD_ERR_UNSUPPORTED: return "unsupported shape or size";
        case SD_ERR_CUDA: return "CUDA error";
        case SD_ERR_INDEX_OOB: return "index or page entry out of range";
        case SD_ERR_TIMEOUT: return "bounded wait in a kernel gave up";
        case SD_ERR_WORKSPACE: return "workspace too small";
        case SD_ERR_ORDER: return "index row not strictly ascending";
        default: return "unknown status";
    }
}

int32_t sd_last_cuda_error(const char** name) {
    if (name != nullptr) *name = cudaGetErrorName(g_last_cuda_error);
    return (int32_t)g_last_cuda_error;
}

int32_t sd_version(void) { return 100; }

}  // extern "C"
