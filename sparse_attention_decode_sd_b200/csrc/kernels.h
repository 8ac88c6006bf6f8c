// kernels.h -- internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sd {

constexpr int kSample = 2048;         // sampled positions per row for the candidate threshold
constexpr int kThresholdCluster = 8;  // CTAs (one cluster) that score one group's sample

struct TopkArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* K;
    const int32_t* page_table;
    const int32_t* lens;
    const int32_t* k;
    int32_t* idx;
    float* cand;        // workspace, B*Hq*n_cap floats: candidate scores, one sequential stream per
                        // score-pass warp; the candidates of one (page, head) are consecutive, in
                        // position order
    uint2* prec;        // workspace [B][Hq][mstride]: per (head, page) {where its candidates start in
                        // cand, 16-bit mask: bit i = position p*16 + i is a candidate}
    float* tau;         // workspace [B][Hq]: candidate threshold (scores >= tau are candidates;
                        // -inf: every position)
    const void** inputs;   // workspace [3]: q, K and page_table of the last score pass (the select
                           // step reads them from here when it has to recompute a row)
    int32_t* status;
    int B, Hq, Hkv, G, max_pages, num_pages, k_max;
    long n_cap;         // max_pages * page size: row stride of the score buffer
    int mstride;        // records per head row (max_pages rounded up to 8)
    int ccap;           // rows with N_b <= ccap take every position as a candidate
    int spp;            // pages per pipeline stage of the score pass
    int stages;         // pipeline depth of the score pass
    int cap;            // select: candidate entries that fit in shared memory
};

size_t score_pass_smem(const TopkArgs& a);
size_t threshold_smem(const TopkArgs& a);
cudaError_t launch_threshold(const TopkArgs& a, cudaStream_t stream);
size_t select_smem(const TopkArgs& a);
cudaError_t launch_score_pass(const TopkArgs& a, int grid, cudaStream_t stream);
cudaError_t launch_select(const TopkArgs& a, cudaStream_t stream);

constexpr int kRange = 16384;           // dense decode: positions per counted range
constexpr int kMaxDecodeWarps = 1280;   // dense decode: persistent warps (one per CTA) at most
constexpr int kMaxSparseWarps = 4096;   // sparse decode: persistent warps (one per CTA) at most
constexpr int kRowSegs = 64;            // sparse decode: segment slots per (b, h) row
constexpr int kOrderMaxRows = 2048;     // sparse decode: rows up to which the offset order is used
constexpr int kRowBatch = 4;            // sparse decode: consecutive idx entries per rows_kernel thread and pass
constexpr uint32_t kSampledFlag = 0x40000000u;   // idx entry: a row drawn by the stochastic selection
constexpr int kPosMask = 0x3fffffff;             // the position bits of an idx entry

struct DecodeArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    const int32_t* page_table;
    const int32_t* lens;
    const int32_t* idx;   // null for dense decode
    float* out;
    // workspace, sparse decode
    int* rlen;            // [B*Hq] entries before the first negative one
    int* arrive;          // [B*Hq] segments of the row finished so far (zeroed by rows_kernel)
    int* bsum;            // [nb] entries of the rows of each rows_kernel CTA
    float* rlw;           // [B*Hq] weighted mode: log2 of the weight of the row's drawn entries
    // workspace, dense decode and the sparse decode over GQA groups
    int* counts;          // [nrt] rows (positions) per range
    uint8_t* umask;       // sparse over groups: [B*Hkv][n_cap] heads of the group that selected each
                          // position (bit g: head kvh*G+g), 1 byte per position for G <= 8, else 2
    // workspace, both
    float2* ml;           // per (b, h, segment) running max (log2 units) and sum
    float* acc;           // per (b, h, segment) un-normalised output [128]
    int32_t* status;
    int B, Hq, Hkv, G, max_pages, num_pages, k_max;
    long n_cap;
    int nrp;              // dense: ranges per (b, kv head) group
    int nrt;              // dense: B * Hkv * nrp
    int tpr, rpc, nb;     // sparse: rows_kernel threads per row, rows per CTA, CTAs
    int min_epw;          // sparse: entries per warp at least (a row spans <= jmax warps)
    int jmax;             // segment slots per (b, h)
    int total_warps;      // persistent decode warps in the grid
    float scale_log2;     // log2(e) / sqrt(d)
    int weighted;         // sparse: idx entries with kSampledFlag are drawn rows of a stochastic
                          // selection, weighted by (N_b - plain entries) / drawn entries
    int order_rows;       // sparse: full rows are visited in offset order (heads of a group aligned)
    int union_tiles;      // group walk: whole 16-position tiles with head masks, instead of only the
                          // selected positions (the union covers nearly every position)
};

size_t decode_smem();
size_t sparse_decode_smem();
// CTAs (one warp each) of the decode kernel for (dense, G) that fit on one SM.
cudaError_t decode_occupancy(bool dense, int G, int* ctas_per_sm);
cudaError_t launch_sparse(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_sparse_union(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_dense(const DecodeArgs& a, cudaStream_t stream);

// Quest page-level indexer.
constexpr int kQuestMaxPages = 24 * 1024;   // pages per request the page select holds in shared memory

struct QuestArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* K;
    __nv_bfloat16* boxes;        // [num_pages][Hkv][2][128]: per-dimension minimum, then maximum
    const int32_t* page_table;
    const int32_t* lens;
    const int32_t* k;
    int32_t* idx;
    float* rel;                  // workspace [B][Hq][max_pages]: page relevance
    int32_t* status;
    int B, Hq, Hkv, G, max_pages, num_pages, k_max;
    long n_cap;
    int last_only;               // summarize: only each request's last page
};
cudaError_t launch_quest_summarize(const QuestArgs& a, cudaStream_t stream);
cudaError_t launch_quest_score(const QuestArgs& a, cudaStream_t stream);
cudaError_t launch_quest_select(const QuestArgs& a, cudaStream_t stream);
size_t quest_select_smem(const QuestArgs& a);

// Stochastic index selection: the draw from the rest of each row (stochastic.cu).
constexpr int kMaxSelectScratch = 64;   // ints of block-scan and selection state
struct SampleArgs {
    const int32_t* lens;
    const int32_t* k_det;
    const int32_t* k_samp;
    int32_t* idx;            // in: the exact top-k_det rows; out: those rows and the drawn ones
    int32_t* status;
    uint64_t seed;
    uint32_t step;
    int B, Hq, k_max;
    long n_cap;
    int words;               // 32-bit words of a bitmap over n_cap positions
    int cap;                 // candidate positions that fit in shared memory
};
size_t sample_smem(const SampleArgs& a);
cudaError_t launch_sample(const SampleArgs& a, cudaStream_t stream);

struct AppendArgs {
    __nv_bfloat16* K;
    __nv_bfloat16* V;
    const int32_t* page_table;
    int32_t* lens;
    const __nv_bfloat16* k_new;
    const __nv_bfloat16* v_new;
    int32_t* k_sel;
    __nv_bfloat16* boxes;   // Quest boxes [num_pages][Hkv][2][128] kept up to date for the written page, or null
    int32_t* status;
    int B, Hkv, max_pages, num_pages, ratio;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

}  // namespace sd
