/*
 * oracle.c -- plain, slow, fp64 CPU restatement of exact top-k sparse decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file;
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg do.  It shares
 * no code, header, table or constant with the CUDA library and includes none of its files.
 *
 * What it computes (every step in double precision, no blocking, fusion or reordering):
 *
 *   score      s[b,h,i] = sum_j q[b,h,j] * K[b, h/G, i, j]              for 0 <= i < N_b
 *              -- the QK^T term of scaled dot-product attention
 *                 ("Sparse Attention inference survey" (xllm), sec. 1.1, the SDPA formula);
 *                 the 1/sqrt(d) factor is monotone and so does not change which rows win.
 *   select     S[b,h] = the k_b positions with the largest s, ties at the k-th score going to
 *              the lower position -- exact top-k
 *              ("Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit",
 *               sec. 2 "Sparsitaetsmechanismen: Oracle Top-K"; "Inference-time context
 *               sparsity: illusion or opportunity?", Fig. 1(a): the indexer keeps k rows).
 *   attend     out[b,h] = sum_{i in S} softmax_S(s_i / sqrt(d)) V[b, h/G, i]
 *              -- SDPA restricted to the selected rows, softmax renormalised over S only
 *              (same SDPA formula; Fig. 1(a) "Sparse" mode reads only the k selected rows).
 *   dense      attend with S = all N_b positions (Fig. 1(a) "Dense" mode).
 *   quest      the page-level approximate indexer Quest ("The Sparse Frontier" review (xllm),
 *              sec. 7.1 "Quest" and Table 1; memory model Eq. 10): pages of P positions, each
 *              represented per KV head by the per-dimension minimum and maximum of its keys;
 *              per (b, h) the "most relevant" pages are kept, always including the page that holds
 *              the current (last) position.  The pages do not spell out relevance; the reading
 *              here is the largest q.k that any key inside the page's box [min, max] can reach,
 *              r_j = sum_d max(q_d * min_d, q_d * max_d).  Budget: ceil(k_b / P) pages (the
 *              current page plus the best others, ties to the lower page); the selection is
 *              every position < N_b of the kept pages, ascending.
 *   stochastic the stochastic index selection the pages evaluate (vAttention: "Technische
 *              Zusammenfassung", sec. 2 "Stochastische Indexierung" and sec. 3A "Stochastisch vs.
 *              Deterministisch"), which they name but do not spell out.  The reading here: per
 *              (b, h) the exact top-k_det rows S_d (as in select), plus m = min(k_samp, |R|) rows
 *              S_s drawn uniformly without replacement from the rest R = [0, N_b) \ S_d; each
 *              sampled row stands for |R| / m rows, i.e. its exp(z) is multiplied by w = |R| / m
 *              in both the numerator and the denominator of the softmax (an inverse-inclusion-
 *              probability estimate of the sums over R).  The draw: every p in R gets the key
 *              u(p) = top 32 bits of SM(SM(SM(seed + step) + r) + p), r = b * Hq + h, where
 *              SM(x) is one output of the SplitMix64 generator from state x (Steele, Lea and
 *              Flood, "Fast splittable pseudorandom number generators", 2014); S_s = the m
 *              positions with the smallest (u, p).  In idx a sampled row carries bit 30
 *              (SAMPLED_FLAG) on its position; attend reads w back from the row as
 *              (N_b - #unflagged) / #flagged.
 *
 * Data layout read here (the paged KV cache the pages describe as a paged-KV backend,
 * "Inference-time context sparsity", sec. 1, "sparsity is usable for systems gains"):
 *   q           bf16 [B][Hq][d]                          (raw 16-bit patterns)
 *   K, V        bf16 [num_pages][P][Hkv][d]              (raw 16-bit patterns)
 *   page_table  int32 [B][max_pages]; logical position p of request b lives in page
 *               page_table[b][p / P], slot p % P
 *   lens        int32 [B]  (N_b)
 *   k           int32 [B]  (k_b; k_b >= N_b selects every row)
 *   idx         int32 [B][Hq][k_max], ascending positions, -1 after the first min(k_b,N_b)
 * Query head h reads KV head h / G with G = Hq / Hkv (contiguous GQA groups).
 *
 * Every entry point returns 0 on success and a negative number for an argument it cannot
 * honour (it never reads outside the buffers it was given).
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SAMPLED_FLAG 0x40000000   /* idx entry: a row drawn by the stochastic selection */
#define POS_MASK 0x3fffffff

/* bf16 -> double is exact: a bf16 is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    int B, Hq, Hkv, d, P, max_pages, k_max, num_pages;
} oshape;

static int check_shape(const oshape* s) {
    if (s->B < 0 || s->Hq <= 0 || s->Hkv <= 0 || s->d <= 0 || s->P <= 0) return -1;
    if (s->Hq % s->Hkv != 0) return -1;
    if (s->max_pages < 0 || s->k_max < 0 || s->num_pages < 0) return -1;
    return 0;
}

/* Pointer to row (b, kvh, logical position p) of a paged cache, or NULL if the page table
 * points outside the cache. */
static const uint16_t* cache_row(const oshape* s, const uint16_t* cache, const int32_t* page_table,
                                 int b, int kvh, long p) {
    long page_slot = p / s->P;
    if (page_slot >= s->max_pages) return NULL;
    int32_t page = page_table[(long)b * s->max_pages + page_slot];
    if (page < 0 || page >= s->num_pages) return NULL;
    long slot = p % s->P;
    long row = ((long)page * s->P + slot) * s->Hkv + kvh;
    return cache + row * s->d;
}

static int req_len(const oshape* s, const int32_t* lens, int b) {
    int n = lens[b];
    if (n < 0 || (long)n > (long)s->max_pages * s->P) return -1;
    return n;
}

/* s[i] = q[b,h] . K[b, h/G, i] for i < N_b, in double. */
static int scores_one(const oshape* s, const uint16_t* q, const uint16_t* K, const int32_t* page_table,
                      int b, int h, int n, double* out) {
    int G = s->Hq / s->Hkv;
    int kvh = h / G;
    const uint16_t* qh = q + ((long)b * s->Hq + h) * s->d;
    for (long i = 0; i < n; ++i) {
        const uint16_t* krow = cache_row(s, K, page_table, b, kvh, i);
        if (!krow) return -2;
        double acc = 0.0;
        for (int j = 0; j < s->d; ++j) acc += bf16_to_double(qh[j]) * bf16_to_double(krow[j]);
        out[i] = acc;
    }
    return 0;
}

int oracle_scores(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages,
                  const uint16_t* q, const uint16_t* K, const int32_t* page_table, const int32_t* lens,
                  int b, int h, double* out) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, 0, num_pages};
    if (check_shape(&s) || b < 0 || b >= B || h < 0 || h >= Hq) return -1;
    int n = req_len(&s, lens, b);
    if (n < 0) return -1;
    return scores_one(&s, q, K, page_table, b, h, n, out);
}

/* Order used for selection: larger score first; equal scores -> lower position first.
 * -0.0 and +0.0 compare equal (C's == on doubles). */
typedef struct { double s; int32_t pos; } scored;

static int by_score_then_pos(const void* a, const void* b) {
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int by_pos(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y);
}

/* Exact top-k of one (b, h): writes min(k, n) ascending positions then -1 up to k_max. */
static int topk_one(const oshape* s, const uint16_t* q, const uint16_t* K, const int32_t* page_table,
                    int b, int h, int n, int kb, int32_t* idx_row) {
    int take = kb < n ? kb : n;
    if (take > s->k_max) return -3;
    for (int i = 0; i < s->k_max; ++i) idx_row[i] = -1;
    if (take <= 0) return 0;
    double* sc = (double*)malloc(sizeof(double) * (size_t)n);
    scored* all = (scored*)malloc(sizeof(scored) * (size_t)n);
    if (!sc || !all) { free(sc); free(all); return -4; }
    int rc = scores_one(s, q, K, page_table, b, h, n, sc);
    if (rc == 0) {
        for (int i = 0; i < n; ++i) { all[i].s = sc[i]; all[i].pos = i; }
        qsort(all, (size_t)n, sizeof(scored), by_score_then_pos);
        for (int i = 0; i < take; ++i) idx_row[i] = all[i].pos;
        qsort(idx_row, (size_t)take, sizeof(int32_t), by_pos);
    }
    free(sc);
    free(all);
    return rc;
}

int oracle_topk(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages, int k_max,
                const uint16_t* q, const uint16_t* K, const int32_t* page_table, const int32_t* lens,
                const int32_t* k, int32_t* idx) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, k_max, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b) {
        if (req_len(&s, lens, b) < 0) return -1;
        if (k[b] < 1) return -1;
    }
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        int rc = topk_one(&s, q, K, page_table, b, h, lens[b], k[b], idx + bh * (long)k_max);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* The two sums of softmax attention of one (b, h) over the listed rows (order irrelevant), each
 * exp taken relative to zref:  z_i = s_i / sqrt(d),  e_i = c_i exp(z_i - zref),
 * num = sum e_i V_i (d doubles),  den = sum e_i,  with c_i = 1 for a plain entry and
 * c_i = w = (N_b - #plain) / #sampled for an entry that carries SAMPLED_FLAG.
 * zref < -1e300 asks for zref = max z_i (the numerically safe choice). */
static int attention_sums(const oshape* s, const uint16_t* q, const uint16_t* K, const uint16_t* V,
                          const int32_t* page_table, int b, int h, int n, const int32_t* sel, int nsel,
                          double zref, double* num, double* den) {
    int G = s->Hq / s->Hkv;
    int kvh = h / G;
    const uint16_t* qh = q + ((long)b * s->Hq + h) * s->d;
    for (int j = 0; j < s->d; ++j) num[j] = 0.0;
    *den = 0.0;
    if (nsel == 0) return 0;
    int nsamp = 0;
    for (int t = 0; t < nsel; ++t) nsamp += (sel[t] & SAMPLED_FLAG) != 0;
    double w = nsamp > 0 ? (double)(n - (nsel - nsamp)) / (double)nsamp : 1.0;
    double* z = (double*)malloc(sizeof(double) * (size_t)nsel);
    if (!z) return -4;
    double scale = 1.0 / sqrt((double)s->d);
    double zmax = -INFINITY;
    for (int t = 0; t < nsel; ++t) {
        int32_t p = sel[t] & POS_MASK;
        if (p >= n) { free(z); return -2; }
        const uint16_t* krow = cache_row(s, K, page_table, b, kvh, p);
        if (!krow) { free(z); return -2; }
        double acc = 0.0;
        for (int j = 0; j < s->d; ++j) acc += bf16_to_double(qh[j]) * bf16_to_double(krow[j]);
        z[t] = acc * scale;
        if (z[t] > zmax) zmax = z[t];
    }
    if (zref < -1e300) zref = zmax;
    for (int t = 0; t < nsel; ++t) {
        double e = exp(z[t] - zref) * ((sel[t] & SAMPLED_FLAG) ? w : 1.0);
        const uint16_t* vrow = cache_row(s, V, page_table, b, kvh, sel[t] & POS_MASK);
        if (!vrow) { free(z); return -2; }
        *den += e;
        for (int j = 0; j < s->d; ++j) num[j] += e * bf16_to_double(vrow[j]);
    }
    free(z);
    return 0;
}

/* Softmax attention of one (b, h) over the listed rows: out = num / den (an empty list gives 0). */
static int attend_one(const oshape* s, const uint16_t* q, const uint16_t* K, const uint16_t* V,
                      const int32_t* page_table, int b, int h, int n, const int32_t* sel, int nsel,
                      double* out) {
    double den = 0.0;
    int rc = attention_sums(s, q, K, V, page_table, b, h, n, sel, nsel, -INFINITY, out, &den);
    if (rc != 0 || nsel == 0) return rc;
    for (int j = 0; j < s->d; ++j) out[j] /= den;
    return 0;
}

/* Attention over the rows each (b, h) lists in idx (entries < 0 are padding and are skipped;
 * entries with SAMPLED_FLAG are weighted as described at the top).  out is double [B][Hq][d]. */
int oracle_attend(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages, int k_max,
                  const uint16_t* q, const uint16_t* K, const uint16_t* V, const int32_t* page_table,
                  const int32_t* lens, const int32_t* idx, double* out) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, k_max, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b)
        if (req_len(&s, lens, b) < 0) return -1;
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        const int32_t* row = idx + bh * (long)k_max;
        int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k_max > 0 ? k_max : 1));
        int nsel = 0;
        int rc = sel ? 0 : -4;
        if (sel) {
            for (int t = 0; t < k_max; ++t)
                if (row[t] >= 0) sel[nsel++] = row[t];
            rc = attend_one(&s, q, K, V, page_table, b, h, lens[b], sel, nsel, out + bh * (long)d);
        }
        free(sel);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* Dense decode: attention over every position 0..N_b-1.  out is double [B][Hq][d]. */
int oracle_dense(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages,
                 const uint16_t* q, const uint16_t* K, const uint16_t* V, const int32_t* page_table,
                 const int32_t* lens, double* out) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, 0, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b)
        if (req_len(&s, lens, b) < 0) return -1;
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        int n = lens[b];
        int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        int rc = sel ? 0 : -4;
        if (sel) {
            for (int i = 0; i < n; ++i) sel[i] = i;
            rc = attend_one(&s, q, K, V, page_table, b, h, n, sel, n, out + bh * (long)d);
        }
        free(sel);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* The unnormalised sums of attend, every exp taken relative to 0 (so that sums from different
 * row lists are comparable): num double [B][Hq][d], den double [B][Hq]. */
int oracle_attend_parts(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages, int k_max,
                        const uint16_t* q, const uint16_t* K, const uint16_t* V, const int32_t* page_table,
                        const int32_t* lens, const int32_t* idx, double* num, double* den) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, k_max, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b)
        if (req_len(&s, lens, b) < 0) return -1;
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        const int32_t* row = idx + bh * (long)k_max;
        int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k_max > 0 ? k_max : 1));
        int nsel = 0;
        int rc = sel ? 0 : -4;
        if (sel) {
            for (int t = 0; t < k_max; ++t)
                if (row[t] >= 0) sel[nsel++] = row[t];
            rc = attention_sums(&s, q, K, V, page_table, b, h, lens[b], sel, nsel, 0.0, num + bh * (long)d, den + bh);
        }
        free(sel);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* One output of the SplitMix64 generator whose state is x before the step: the state advances by
 * the golden-ratio increment 0x9E3779B97F4A7C15 and is then mixed (Steele, Lea and Flood 2014). */
static uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t oracle_splitmix64(uint64_t x) { return splitmix64(x); }

/* Sampling key of position p in row r: the top 32 bits of SM(SM(SM(seed + step) + r) + p). */
static uint32_t sample_key(uint64_t seed, uint32_t step, long r, long p) {
    uint64_t c = splitmix64(splitmix64(splitmix64(seed + (uint64_t)step) + (uint64_t)r) + (uint64_t)p);
    return (uint32_t)(c >> 32);
}

typedef struct { uint32_t key; int32_t pos; } keyed;

static int by_key_then_pos(const void* a, const void* b) {
    const keyed* x = (const keyed*)a;
    const keyed* y = (const keyed*)b;
    if (x->key != y->key) return (x->key < y->key) ? -1 : 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

/* Stochastic selection of one (b, h) (see the top): S_d = exact top-k_det, S_s = the min(k_samp, |R|)
 * positions of R = [0, N_b) \ S_d with the smallest sampling keys; both ascending together in
 * idx_row, sampled ones with SAMPLED_FLAG, then -1. */
static int stochastic_one(const oshape* s, const uint16_t* q, const uint16_t* K, const int32_t* page_table,
                          int b, int h, int n, int kdet, int ksamp, uint64_t seed, uint32_t step, int32_t* idx_row) {
    int rc = topk_one(s, q, K, page_table, b, h, n, kdet, idx_row);
    if (rc != 0 || n <= 0) return rc;
    int ndet = 0;   /* the rows top-k returned */
    while (ndet < s->k_max && idx_row[ndet] >= 0) ++ndet;
    long nrest = (long)n - ndet;
    long m = ksamp < nrest ? ksamp : nrest;
    if (m <= 0) return 0;
    if (ndet + m > s->k_max) return -3;
    char* in_det = (char*)calloc((size_t)n, 1);
    keyed* rest = (keyed*)malloc(sizeof(keyed) * (size_t)n);
    int32_t* merged = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ndet + m));
    if (!in_det || !rest || !merged) { free(in_det); free(rest); free(merged); return -4; }
    for (int t = 0; t < ndet; ++t)
        if (idx_row[t] < n) in_det[idx_row[t]] = 1;
    long r = (long)b * s->Hq + h, c = 0;
    for (long p = 0; p < n; ++p)
        if (!in_det[p]) { rest[c].key = sample_key(seed, step, r, p); rest[c].pos = (int32_t)p; ++c; }
    qsort(rest, (size_t)c, sizeof(keyed), by_key_then_pos);
    for (int t = 0; t < ndet; ++t) merged[t] = idx_row[t];
    for (long t = 0; t < m; ++t) merged[ndet + t] = rest[t].pos | SAMPLED_FLAG;
    /* ascending by position (the flag bit does not take part in the order) */
    for (long i = 1; i < ndet + m; ++i) {
        int32_t v = merged[i];
        long j = i - 1;
        while (j >= 0 && (merged[j] & POS_MASK) > (v & POS_MASK)) { merged[j + 1] = merged[j]; --j; }
        merged[j + 1] = v;
    }
    for (long t = 0; t < ndet + m; ++t) idx_row[t] = merged[t];
    free(in_det);
    free(rest);
    free(merged);
    return 0;
}

int oracle_stochastic_topk(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages, int k_max,
                           const uint16_t* q, const uint16_t* K, const int32_t* page_table, const int32_t* lens,
                           const int32_t* k_det, const int32_t* k_samp, uint64_t seed, uint32_t step,
                           int32_t* idx) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, k_max, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b) {
        if (req_len(&s, lens, b) < 0) return -1;
        if (k_det[b] < 1 || k_samp[b] < 0) return -1;
        if ((long)lens[b] > (long)POS_MASK) return -1;
    }
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        int rc = stochastic_one(&s, q, K, page_table, b, h, lens[b], k_det[b], k_samp[b], seed, step,
                                idx + bh * (long)k_max);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* Quest page representation of logical page j of request b, KV head kvh: the per-dimension minimum
 * and maximum over the page's positions that exist (those < N_b), in double. */
static int quest_box(const oshape* s, const uint16_t* K, const int32_t* page_table, int b, int kvh, int n, long j,
                     double* mn, double* mx) {
    long p0 = j * s->P, p1 = p0 + s->P;
    if (p1 > n) p1 = n;
    for (long p = p0; p < p1; ++p) {
        const uint16_t* krow = cache_row(s, K, page_table, b, kvh, p);
        if (!krow) return -2;
        for (int e = 0; e < s->d; ++e) {
            double v = bf16_to_double(krow[e]);
            if (p == p0 || v < mn[e]) mn[e] = v;
            if (p == p0 || v > mx[e]) mx[e] = v;
        }
    }
    return 0;
}

/* r_j = sum_d max(q_d * min_d, q_d * max_d) for every page j < ceil(N_b / P) of (b, h). */
static int quest_scores_one(const oshape* s, const uint16_t* q, const uint16_t* K, const int32_t* page_table,
                            int b, int h, int n, double* out) {
    int G = s->Hq / s->Hkv;
    int kvh = h / G;
    const uint16_t* qh = q + ((long)b * s->Hq + h) * s->d;
    long np = ((long)n + s->P - 1) / s->P;
    double* mn = (double*)malloc(sizeof(double) * (size_t)s->d);
    double* mx = (double*)malloc(sizeof(double) * (size_t)s->d);
    if (!mn || !mx) { free(mn); free(mx); return -4; }
    int rc = 0;
    for (long j = 0; j < np && rc == 0; ++j) {
        rc = quest_box(s, K, page_table, b, kvh, n, j, mn, mx);
        double r = 0.0;
        for (int e = 0; e < s->d && rc == 0; ++e) {
            double qe = bf16_to_double(qh[e]);
            double lo = qe * mn[e], hi = qe * mx[e];
            r += lo > hi ? lo : hi;
        }
        out[j] = r;
    }
    free(mn);
    free(mx);
    return rc;
}

int oracle_quest_scores(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages,
                        const uint16_t* q, const uint16_t* K, const int32_t* page_table, const int32_t* lens,
                        int b, int h, double* out) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, 0, num_pages};
    if (check_shape(&s) || b < 0 || b >= B || h < 0 || h >= Hq) return -1;
    int n = req_len(&s, lens, b);
    if (n < 0) return -1;
    return quest_scores_one(&s, q, K, page_table, b, h, n, out);
}

/* Quest selection of one (b, h): the current page (the last one) plus the ceil(k_b / P) - 1 other
 * pages with the largest r (ties to the lower page); all their positions < N_b, ascending, then -1. */
static int quest_one(const oshape* s, const uint16_t* q, const uint16_t* K, const int32_t* page_table,
                     int b, int h, int n, int kb, int32_t* idx_row) {
    for (int i = 0; i < s->k_max; ++i) idx_row[i] = -1;
    if (n <= 0) return 0;
    long np = ((long)n + s->P - 1) / s->P;
    long kp = ((long)kb + s->P - 1) / s->P;
    if (kp > np) kp = np;
    char* keep = (char*)calloc((size_t)np, 1);
    double* r = (double*)malloc(sizeof(double) * (size_t)np);
    scored* other = (scored*)malloc(sizeof(scored) * (size_t)np);
    if (!keep || !r || !other) { free(keep); free(r); free(other); return -4; }
    int rc = quest_scores_one(s, q, K, page_table, b, h, n, r);
    if (rc == 0) {
        keep[np - 1] = 1;   /* the page of the current position is always kept */
        for (long j = 0; j + 1 < np; ++j) { other[j].s = r[j]; other[j].pos = (int32_t)j; }
        qsort(other, (size_t)(np - 1), sizeof(scored), by_score_then_pos);
        for (long t = 0; t + 1 < kp; ++t) keep[other[t].pos] = 1;
        long w = 0;
        for (long j = 0; j < np && rc == 0; ++j) {
            if (!keep[j]) continue;
            for (long p = j * s->P; p < (j + 1) * s->P && p < n; ++p) {
                if (w >= s->k_max) { rc = -3; break; }
                idx_row[w++] = (int32_t)p;
            }
        }
    }
    free(keep);
    free(r);
    free(other);
    return rc;
}

int oracle_quest_topk(int B, int Hq, int Hkv, int d, int P, int max_pages, int num_pages, int k_max,
                      const uint16_t* q, const uint16_t* K, const int32_t* page_table, const int32_t* lens,
                      const int32_t* k, int32_t* idx) {
    oshape s = {B, Hq, Hkv, d, P, max_pages, k_max, num_pages};
    if (check_shape(&s)) return -1;
    for (int b = 0; b < B; ++b) {
        if (req_len(&s, lens, b) < 0) return -1;
        if (k[b] < 1) return -1;
    }
    int rc_all = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc_all)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        int rc = quest_one(&s, q, K, page_table, b, h, lens[b], k[b], idx + bh * (long)k_max);
        if (rc < rc_all) rc_all = rc;
    }
    return rc_all;
}

/* Number of OpenMP threads the entry points above use (reported beside CPU timings). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
