/*
 * sparsedecode.h -- C ABI of libsparsedecode: exact top-k sparse decode attention over a paged,
 * grouped-query (GQA), bf16 KV cache, on NVIDIA B200 (sm_100a).
 *
 * The method (sources are the pages' titles and sections):
 *   - "Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit - Illusion oder
 *     Chance?", sec. 2, "Sparsitaetsmechanismen: Oracle Top-K": an exact top-k indexer picks, per
 *     decode query and query head, the k keys with the highest score q.K.
 *   - "Inference-time context sparsity: illusion or opportunity?", Fig. 1(a): dense decode reads
 *     O(N d) bytes per step, sparse decode routes through an indexer that keeps k rows and reads
 *     O(k d) bytes; sec. 1 ("sparsity is usable for systems gains"): the kernels handle sparsity
 *     that is irregular per token, per query and per head, under GQA, over a paged KV cache.
 *   - "Sparse Attention inference survey" (xllm), sec. 1.1: scaled dot-product attention,
 *     softmax(q K^T / sqrt(d)) V; here evaluated over the selected rows only, so the softmax is
 *     renormalised over the selected set.
 *
 * Conventions shared by every entry point
 *   Shapes      B requests, Hq query heads, Hkv KV heads, G = Hq / Hkv (1 <= G <= 16), head
 *               dimension d = 128, page size P = 16.  Query head h reads KV head h / G.
 *   q           bf16 [B][Hq][d], row-major, device memory, 16-byte aligned.
 *   K, V        bf16 [num_pages][P][Hkv][d] ("NHD" pages), device memory, 16-byte aligned.
 *               Logical position p of request b is row [page_table[b][p / P]][p % P].
 *   page_table  int32 [B][max_pages_per_req], device memory.  Entries at positions >= lens[b]
 *               are never read.
 *   lens        int32 [B], device memory: context length N_b, 0 <= N_b <= max_pages_per_req * P.
 *   idx         int32 [B][Hq][k_max], device memory: per (b, h) the selected positions in strictly
 *               ascending order, followed by padding (any negative value, -1 by convention).  A
 *               non-negative entry after padding is an ordering error (SD_ERR_ORDER).
 *   out         fp32 [B][Hq][d], device memory, 16-byte aligned.
 *   workspace   device scratch owned by the caller, at least sd_workspace_size() bytes,
 *               256-byte aligned.  Its contents need no initialisation and are not preserved.
 *   dev_status  int32, device memory, owned by the caller and zeroed by the caller.  Kernels
 *               never trap: a violated device-side precondition (bad length, bad k, an index or
 *               page entry out of range) makes the first failing kernel store its sd_status code
 *               there (first error wins; later calls keep it) and skip the offending access.
 *               Read it after synchronising the stream.  Outputs of a call that set it are
 *               unspecified.
 *   stream      a cudaStream_t passed as void*; NULL means the legacy default stream.  Every
 *               call is asynchronous on that stream, uses the current CUDA device, allocates
 *               nothing and keeps no state between calls.
 *   Return      host-side validation happens before any launch; a non-SD_OK return means nothing
 *               was launched (SD_ERR_CUDA: a launch failed; the CUDA error is not cleared).
 */
#ifndef SPARSEDECODE_H
#define SPARSEDECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SD_API __attribute__((visibility("default")))
#else
#define SD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sd_shape {
    int32_t batch;              /* B, >= 1 */
    int32_t num_q_heads;        /* Hq, >= 1, multiple of num_kv_heads */
    int32_t num_kv_heads;       /* Hkv, >= 1, Hq / Hkv <= 16 */
    int32_t head_dim;           /* d; only 128 is supported */
    int32_t page_size;          /* P; only 16 is supported */
    int32_t max_pages_per_req;  /* row length of page_table, >= 1 */
    int32_t k_max;              /* row length of idx, >= 1 */
    int32_t num_pages;          /* pages in each of K and V, >= 1 */
} sd_shape;

typedef int32_t sd_status;

enum {
    SD_OK = 0,
    SD_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, inconsistent shape, bad length or k */
    SD_ERR_UNSUPPORTED = 2,   /* head_dim != 128, page_size != 16, G > 16, sizes beyond limits */
    SD_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
    SD_ERR_INDEX_OOB = 4,     /* device: idx entry >= N_b, or page entry outside [0, num_pages) */
    SD_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel gave up */
    SD_ERR_WORKSPACE = 6,     /* workspace_bytes smaller than sd_workspace_size() */
    SD_ERR_ORDER = 7          /* device: an idx row is not strictly ascending */
};

enum { SD_OP_TOPK = 1, SD_OP_SPARSE = 2, SD_OP_DENSE = 3, SD_OP_QUEST = 4 };

/* Bytes of workspace that operation `op` (SD_OP_TOPK, SD_OP_SPARSE, SD_OP_DENSE, SD_OP_QUEST) needs
 * for `shape` (independent of the data and of the
 * device).  Returns SD_ERR_INVALID_ARG / SD_ERR_UNSUPPORTED for a shape the library rejects. */
SD_API sd_status sd_workspace_size(const sd_shape* shape, int32_t op, size_t* bytes);

/* Exact top-k indexer ("Oracle Top-K", gist.science summary sec. 2; the indexer of Fig. 1(a) of
 * "Inference-time context sparsity").
 *   For every request b and query head h: s_i = q[b,h] . K[b, h/G, i] for 0 <= i < N_b (fp32
 *   accumulation of exact bf16 products); keep the min(k[b], N_b) positions with the largest s,
 *   ties at the k-th score going to the lower position (-0.0 equals +0.0; NaN inputs are
 *   invalid); write them to idx[b][h] in ascending order, then -1 up to k_max.
 *   k       int32 [B], device memory, 1 <= k[b]; min(k[b], N_b) must not exceed k_max
 *           (else SD_ERR_INVALID_ARG in dev_status and that row is left all -1).
 *   Requests with k[b] >= N_b are returned as 0..N_b-1 without reading K. */
SD_API sd_status sd_topk_index(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                        const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream);

/* The two halves of sd_topk_index, for callers that schedule or time them separately.
 *   sd_topk_scores  scores every position of every request that needs a selection
 *                   (1 <= k[b] < N_b) and leaves in the workspace what the selection needs:
 *                   the whole fp32 row s[b][h][0..N_b) when N_b <= 3 k_max + 4096, otherwise
 *                   only the candidates (every score at or above a per-row threshold placed by a
 *                   sample of the row) with their positions.  The workspace layout is internal.
 *   sd_topk_select  reads those from the same workspace and writes idx exactly as sd_topk_index
 *                   does (in the rare case a row's candidates cannot decide the selection, it
 *                   recomputes that row from the q, K and page_table given to sd_topk_scores);
 *                   it must follow sd_topk_scores on the same workspace (stream order), with
 *                   q, K, page_table, lens and k unchanged in between. */
SD_API sd_status sd_topk_scores(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                         const int32_t* lens, const int32_t* k, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream);
SD_API sd_status sd_topk_select(const sd_shape* shape, const int32_t* lens, const int32_t* k, int32_t* idx,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/* sd_topk_index without a caller-provided workspace, for callers that cannot allocate device memory
 * (for example a plugin inside a host engine that passes it only inputs and outputs, or a service
 * whose device memory is fixed at start-up).  The pages have no counterpart of this entry point.
 *   Same inputs, outputs, checks and results as sd_topk_index.  The indexer's workspace lives in one
 *   file-scope device array of 48 MiB inside the library, held by every GPU that loads the library
 *   until the process exits; the call allocates nothing.
 *   Limit: sd_workspace_size(shape, SD_OP_TOPK) must not exceed 48 MiB (for example one request of
 *   64 query heads at 131072 positions and k_max 2621 fits), else SD_ERR_WORKSPACE and nothing is
 *   launched.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 *   device current and keeps it; make that first call before any stream capture.  The address
 *   belongs to the device's current context: after cudaDeviceReset the library's device code is
 *   loaded again and the kept address is no longer valid, so do not call this entry point after a
 *   cudaDeviceReset in the same process.
 *   Every call on a device uses the same array, which keeps the last call's scores: calls whose
 *   kernels overlap on the GPU (other streams, other host threads) race and must be serialised by
 *   the caller. */
SD_API sd_status sd_topk_index_static(const sd_shape* shape, const void* q, const void* K,
                                      const int32_t* page_table, const int32_t* lens, const int32_t* k,
                                      int32_t* idx, int32_t* dev_status, void* stream);

/* Sparse decode attention over the selected rows ("Sparse" mode of Fig. 1(a) of "Inference-time
 * context sparsity"; SDPA of the xllm survey sec. 1.1 restricted to the selected set).
 *   out[b,h] = sum_{i in S} w_i V[b, h/G, i],  w = softmax over S of (q[b,h] . K[b,h/G,i]) / sqrt(d),
 *   S = the entries of idx[b][h] before its first negative one.  An empty S gives out = 0.
 *   Two walks, chosen from the shape alone, give the same result up to rounding order:
 *   - per query head (the usual case): each head gathers its own rows; the heads of a GQA group are
 *     processed side by side, so a row that several of them selected is read from HBM about once and
 *     from L2 after that.  Two kernels; the second starts gathering before the first (the row
 *     checks) ends, so idx, q, K, V and the page table must be complete when the call is enqueued
 *     (stream order), as for every call of the library.
 *   - per GQA group, when the heads of a group are expected to share many rows (expected duplication
 *     G f / (1 - (1 - f)^G) >= 1.4, f = k_max / (max_pages_per_req * 16)): each row of the group's
 *     union is gathered once for every head that selected it.  Four kernels (row checks, the group's
 *     head masks, the walk, the merge).
 *   num_pages * 16 * Hkv must be below 2^31 (cache rows are TMA coordinates), else
 *   SD_ERR_UNSUPPORTED.
 *   Device checks: entries must be < N_b and map to a page-table entry in range (SD_ERR_INDEX_OOB),
 *   strictly ascending, with nothing but padding after the first negative entry (SD_ERR_ORDER).
 *   B * Hq * k_max must be below 2^31 (else SD_ERR_UNSUPPORTED, also from sd_workspace_size). */
SD_API sd_status sd_sparse_decode(const sd_shape* shape, const void* q, const void* K, const void* V,
                           const int32_t* page_table, const int32_t* lens, const int32_t* idx, float* out,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/* Stochastic index selection, the vAttention-style selection the pages evaluate ("Technische
 * Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2 "Stochastische Indexierung" and
 * sec. 3A "Stochastisch vs. Deterministisch"; the pages name the method, not its estimator, and the
 * reading implemented here is stated in full in the library's documentation):
 *   per (b, h): S_d = the exact top-k_det[b] rows (as sd_topk_index with k = k_det), plus
 *   m = min(k_samp[b], |R|) rows drawn uniformly without replacement from the rest
 *   R = [0, N_b) \ S_d.  Position p of R gets the key u(p) = top 32 bits of
 *   SM(SM(SM(seed + step) + b * Hq + h) + p), SM(x) being one SplitMix64 output from state x (a
 *   counter-based generator, so the draw is reproducible), and the m positions with the smallest
 *   (u, p) are drawn.
 *   idx[b][h] holds S_d and the drawn rows together in ascending position, each drawn row with
 *   SD_SAMPLED_FLAG (bit 30) set on its position, then -1; sd_sparse_decode_sampled weighs each drawn
 *   row by |R| / m.  k_det[b] >= 1 and k_samp[b] >= 0 (device array [B]); shape->k_max must hold
 *   k_det + k_samp rows of every request (else the row is left as S_d and dev_status records
 *   SD_ERR_INVALID_ARG).  Workspace: sd_workspace_size(shape, SD_OP_TOPK).  SD_ERR_UNSUPPORTED when
 *   the row bitmaps and candidates of max_pages_per_req * 16 positions do not fit one SM's shared
 *   memory (above about 600K positions per request). */
#define SD_SAMPLED_FLAG 0x40000000
SD_API sd_status sd_stochastic_index(const sd_shape* shape, const void* q, const void* K, const int32_t* page_table,
                                     const int32_t* lens, const int32_t* k_det, const int32_t* k_samp,
                                     uint64_t seed, uint32_t step, int32_t* idx, void* workspace,
                                     size_t workspace_bytes, int32_t* dev_status, void* stream);

/* sd_sparse_decode over the rows of a stochastic selection: an entry with SD_SAMPLED_FLAG is a drawn
 * row and its exp(z) counts w = (N_b - plain entries) / drawn entries times, in both the numerator and
 * the denominator of the softmax -- the inverse of its inclusion probability, so that the drawn rows
 * estimate the sums over all rows outside S_d without bias.  Without flagged entries the result is
 * that of sd_sparse_decode.  Positions are the entries' low 30 bits; the checks of sd_sparse_decode
 * apply to them.  Workspace: sd_workspace_size(shape, SD_OP_SPARSE). */
SD_API sd_status sd_sparse_decode_sampled(const sd_shape* shape, const void* q, const void* K, const void* V,
                                          const int32_t* page_table, const int32_t* lens, const int32_t* idx,
                                          float* out, void* workspace, size_t workspace_bytes,
                                          int32_t* dev_status, void* stream);

/* Dense decode attention over all N_b rows ("Dense" mode of Fig. 1(a)); the comparator of the
 * sparse kernel at the same shape.  shape->k_max is ignored. */
SD_API sd_status sd_dense_decode(const sd_shape* shape, const void* q, const void* K, const void* V,
                          const int32_t* page_table, const int32_t* lens, float* out, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream);

/* Append one decode step's K/V row per request (the growing cache of an agentic decode loop).
 *   For each b: p = lens[b]; the rows k_new[b][kvh][:] and v_new[b][kvh][:] (bf16 [B][Hkv][d],
 *   device memory) are written to K and V at position p through page_table; then lens[b] = p + 1
 *   and, if k_sel is not NULL, k_sel[b] = max(1, round_half_up((p + 1) / ratio)).
 *   p must satisfy p < max_pages_per_req * P and its page entry must be in range, else the row is
 *   not written, lens[b] is unchanged and dev_status records the error.  ratio >= 1. */
SD_API sd_status sd_append_kv(const sd_shape* shape, void* K, void* V, const int32_t* page_table, int32_t* lens,
                       const void* k_new, const void* v_new, int32_t* k_sel, int32_t ratio,
                       int32_t* dev_status, void* stream);

/* Quest, the page-level approximate indexer ("The Sparse Frontier" review, sec. 7.1 "Quest" and
 * Table 1; its memory model is Eq. 10 there): pages of P = 16 positions, each represented per KV head
 * by the per-dimension minimum and maximum of its keys ("boxes"); per decode query and query head the
 * most relevant pages are kept, always including the page of the current (last) position.
 *
 * sd_quest_summarize writes the boxes of every logical page of every request (last_page_only = 0), or
 * only of each request's last page (last_page_only != 0: after sd_append_kv added a row).
 *   boxes   bf16 [num_pages][Hkv][2][d], device memory, 16-byte aligned, owned by the caller and kept
 *           between calls: for physical page pg and KV head kvh, boxes[pg][kvh][0] is the minimum and
 *           boxes[pg][kvh][1] the maximum over the page's positions < N_b (exact bf16 values).
 *           Entries of pages no request holds are not written.
 *   A page-table entry out of range is reported (SD_ERR_INDEX_OOB) and that page is skipped. */
SD_API sd_status sd_quest_summarize(const sd_shape* shape, const void* K, const int32_t* page_table,
                                    const int32_t* lens, void* boxes, int32_t last_page_only,
                                    int32_t* dev_status, void* stream);

/* sd_append_kv that also keeps the Quest boxes current: the box of the page each row is written to
 * becomes the row itself when the row opens the page (p % 16 == 0), else the elementwise min / max of
 * the stored box and the row -- the same bf16 values sd_quest_summarize would write for the page's
 * rows, without a separate pass over K after each step.  Same arguments, checks and errors as
 * sd_append_kv, plus boxes (as for sd_quest_summarize; NULL or misaligned: SD_ERR_INVALID_ARG).  The
 * boxes of the other pages must be current already (sd_quest_summarize over the whole cache once). */
SD_API sd_status sd_quest_append_kv(const sd_shape* shape, void* K, void* V, const int32_t* page_table,
                                    int32_t* lens, const void* k_new, const void* v_new, int32_t* k_sel,
                                    int32_t ratio, void* boxes, int32_t* dev_status, void* stream);

/* sd_quest_index selects, per (b, h), ceil(k[b] / 16) pages: the current page (holding position
 * N_b - 1) plus the most relevant others, relevance of page j being the largest q.k any key inside its
 * box can reach, r_j = sum_d max(q_d * min_d, q_d * max_d) (fp32 accumulation of exact bf16 products);
 * ties go to the lower page.  idx[b][h] receives every position < N_b of the kept pages, ascending,
 * then -1 (the format sd_sparse_decode reads); when the budget covers every page, 0 .. N_b - 1.
 *   boxes      as written by sd_quest_summarize for the current lengths.
 *   k_max      must be at least 16 * ceil(k[b] / 16) for every b whose budget is below its page count,
 *              and at least N_b where it is not (else SD_ERR_INVALID_ARG in dev_status, row all -1).
 *   workspace  sd_workspace_size(shape, SD_OP_QUEST) bytes (the page relevance, fp32).
 *   Supported up to 24576 pages per request (SD_ERR_UNSUPPORTED beyond). */
SD_API sd_status sd_quest_index(const sd_shape* shape, const void* q, const void* boxes, const int32_t* page_table,
                                const int32_t* lens, const int32_t* k, int32_t* idx, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream);

/* Self-test of failure detection (no counterpart in the pages): launches one warp that waits, with
 * the bounded-wait helper every pipeline wait of the library uses, on a barrier that nothing completes.
 * The wait gives up after wait_ms (1 .. 10000) and stores SD_ERR_TIMEOUT in dev_status; the kernel
 * issues no copy, so it leaves nothing in flight and the context stays usable.  Asynchronous on stream;
 * read dev_status after synchronising. */
SD_API sd_status sd_selftest_wait_timeout(uint32_t wait_ms, int32_t* dev_status, void* stream);

/* Static English text for a status code ("unknown status" for other values). */
SD_API const char* sd_status_string(sd_status status);

/* The CUDA runtime error (a cudaError_t value, with its name in *name if name is not NULL) behind
 * the most recent SD_ERR_CUDA returned on the calling thread; 0 and "cudaSuccess" if there was none.
 * The name is static text. */
SD_API int32_t sd_last_cuda_error(const char** name);

/* Library version, major * 10000 + minor * 100 + patch. */
SD_API int32_t sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEDECODE_H */
