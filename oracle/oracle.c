/*
 * Plain fp64 CPU oracle for the DSA lightning indexer and its two
 * scan-reducing variants (PIVOT group proxies, HISA hierarchical blocks).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded inputs both are given.
 *
 * Sources (web pages on DeepSeek Sparse Attention indexers):
 *   [MLI]   "Multi-layer Indexer: overlapping selection and attention in
 *            DeepSeek Sparse Attention", abstract: every layer is preceded by
 *            a lightning indexer that scores the whole cache and keeps the
 *            k = 2048 highest-scoring tokens.
 *   [PIVOT] "PIVOT: Efficient Query-Group Indexing for Token-Level Sparse
 *            Attention", abstract: each query scores every preceding token;
 *            a group of nearby queries is aggregated into one proxy query,
 *            one shared prefix scan gives a candidate set, then Reuse (share
 *            the proxy top-k) or Refine (re-score the candidates with each
 *            query's own indexer, take its own top-k).  Groups are fixed-size
 *            runs of consecutive queries in prefill and the queries of one
 *            MTP step in decode.
 *   [HISA]  "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
 *            Attention", abstract: pooled block representations are scored
 *            and irrelevant blocks discarded, then the original indexer runs
 *            only inside the retained blocks, producing the same token-level
 *            top-k pattern.
 *
 * The pages give the indexer only in words.  The score used throughout is
 * the DeepSeek-V3.2 lightning-indexer score with one key per token shared by
 * all indexer heads:
 *       I[t,s] = sum_h w[t,h] * max(0, q[t,h] . k[s])
 * Readings taken where the pages are silent (each listed in the design notes):
 *   - the prefix is inclusive: query t may select keys s <= pos[t]; a position
 *     at or past the sequence end is clamped to its last key, a negative
 *     position leaves the row empty;
 *   - ties in every ranking go to the lower index;
 *   - a row with fewer than k eligible keys returns all of them, then -1;
 *   - the PIVOT proxy is the mean of the group's q (rounded to bf16, since it
 *     feeds a bf16 scan) and the mean of its w; the proxy scans up to the
 *     group's last position and each query then drops keys past its own
 *     position; the candidate count is C;
 *   - HISA pools each block by the mean of its keys; the first block and the
 *     query's own (last) block are always kept, the `keep` best of the blocks
 *     strictly between them are added; blocks are chosen per query.
 *
 * Numerics: inputs arrive as bf16 bit patterns (Q, K) and fp32 (W); every
 * product and sum is formed in double.  Sorting is a full qsort per row.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- helpers */

/* bf16 bit pattern -> value.  A bf16 number is the upper half of an fp32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits, exponent of
 * fp32), ties to even.  Written from the format's definition: scale x by a
 * power of two so that its 8 significant bits sit left of the binary point,
 * round to an integer with ties to even (rint under the default rounding
 * mode), scale back.  Exponents below fp32's normal range use the subnormal
 * spacing 2^-133.  Overflow is not handled (values stay far below 2^127). */
double orc_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x))
        return x;
    int e;
    frexp(x, &e);                 /* x = m * 2^e, 0.5 <= |m| < 1 */
    int lsb = e - 8;              /* weight of the 8th significant bit */
    if (lsb < -133)
        lsb = -133;
    double r = rint(ldexp(x, -lsb));
    return ldexp(r, lsb);
}

typedef struct {
    double v;
    int32_t i;
} scored_t;

/* Ranking order of every selection: higher score first, then lower index. */
static int cmp_scored(const void* pa, const void* pb)
{
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

/* The indexer score of one query (H heads x d) against one key (d). */
static double indexer_score(const double* q, const double* w, const double* key, int H, int d)
{
    double total = 0.0;
    for (int h = 0; h < H; ++h) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i)
            dot += q[(size_t)h * d + i] * key[i];
        double relu = dot > 0.0 ? dot : 0.0;
        total += w[h] * relu;
    }
    return total;
}

static void load_query(const uint16_t* Q, const float* W, int64_t row, int H, int d, double* q, double* w)
{
    for (int64_t j = 0; j < (int64_t)H * d; ++j)
        q[j] = bf16_value(Q[row * H * d + j]);
    for (int h = 0; h < H; ++h)
        w[h] = (double)W[row * H + h];
}

static void load_key(const uint16_t* K, int64_t row, int d, double* key)
{
    for (int i = 0; i < d; ++i)
        key[i] = bf16_value(K[row * d + i]);
}

/* Sequence that owns query row t: the b with q_off[b] <= t < q_off[b+1]. */
static int seq_of_row(const int32_t* q_off, int n_seqs, int64_t t)
{
    for (int b = 0; b < n_seqs; ++b)
        if (t >= q_off[b] && t < q_off[b + 1])
            return b;
    return -1;
}

/* Number of eligible keys of a query: keys 0..pos, clamped to the sequence. */
static int64_t eligible_count(int32_t pos, int64_t L)
{
    if (pos < 0) return 0;
    int64_t n = (int64_t)pos + 1;
    return n < L ? n : L;
}

/* ------------------------------------------------------------- threading */

typedef void (*row_fn)(void* ctx, int64_t i);
typedef struct {
    row_fn fn;
    void* ctx;
    int64_t n;
    int tid, nthreads;
} worker_t;

static void* worker_main(void* p)
{
    worker_t* w = (worker_t*)p;
    for (int64_t i = w->tid; i < w->n; i += w->nthreads)
        w->fn(w->ctx, i);
    return NULL;
}

/* Run fn(ctx, i) for i in [0, n) on `nthreads` threads (rows are independent). */
static void parallel_rows(row_fn fn, void* ctx, int64_t n, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    worker_t wk[256];
    for (int t = 0; t < nthreads; ++t) {
        wk[t].fn = fn; wk[t].ctx = ctx; wk[t].n = n; wk[t].tid = t; wk[t].nthreads = nthreads;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, worker_main, &wk[t]);
    worker_main(&wk[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
}

/* ----------------------------------------------------------- dense indexer */

typedef struct {
    const uint16_t *Q, *K;
    const float* W;
    int H, d, n_seqs, k;
    const int32_t *q_off, *k_off, *q_pos, *rows;
    int64_t ld;                /* row stride of all_scores */
    int32_t* idx;              /* [n_rows, k] or NULL */
    double* top;               /* [n_rows, k] or NULL */
    double* all_scores;        /* [n_rows, ld] or NULL: score of every key, -inf if ineligible */
    int32_t* n_elig;           /* [n_rows] or NULL */
} dense_ctx;

static void dense_row(void* p, int64_t r)
{
    dense_ctx* c = (dense_ctx*)p;
    int64_t t = c->rows[r];
    int b = seq_of_row(c->q_off, c->n_seqs, t);
    int64_t L = b < 0 ? 0 : (int64_t)c->k_off[b + 1] - c->k_off[b];
    int64_t n = b < 0 ? 0 : eligible_count(c->q_pos[t], L);
    double* q = (double*)malloc(sizeof(double) * ((size_t)c->H * c->d + c->H + c->d));
    double* w = q + (size_t)c->H * c->d;
    double* key = w + c->H;
    scored_t* row = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    load_query(c->Q, c->W, t, c->H, c->d, q, w);
    for (int64_t s = 0; s < n; ++s) {
        load_key(c->K, (int64_t)c->k_off[b] + s, c->d, key);
        row[s].v = indexer_score(q, w, key, c->H, c->d);
        row[s].i = (int32_t)s;
    }
    if (c->all_scores) {
        double* out = c->all_scores + r * c->ld;
        for (int64_t s = 0; s < c->ld; ++s)
            out[s] = s < n ? row[s].v : -INFINITY;
    }
    if (c->n_elig)
        c->n_elig[r] = (int32_t)n;
    if (c->idx) {
        qsort(row, (size_t)n, sizeof(scored_t), cmp_scored);
        for (int j = 0; j < c->k; ++j) {
            c->idx[r * c->k + j] = j < n ? row[j].i : -1;
            if (c->top)
                c->top[r * c->k + j] = j < n ? row[j].v : NAN;
        }
    }
    free(row);
    free(q);
}

/* Dense indexer for the listed query rows: every eligible key is scored and
 * the row is fully sorted by (score desc, index asc) [MLI abstract; PIVOT
 * abstract].  Outputs (each optional): top-k indices and scores in ranking
 * order (-1 / NaN padding), every key's score (-inf where ineligible), and
 * the eligible count. */
int orc_dense(const uint16_t* Q, const uint16_t* K, const float* W, int H, int d,
              int n_seqs, const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
              int n_rows, const int32_t* rows, int k,
              int32_t* idx, double* top, double* all_scores, int64_t ld, int32_t* n_elig,
              int nthreads)
{
    dense_ctx c = {Q, K, W, H, d, n_seqs, k, q_off, k_off, q_pos, rows, ld, idx, top, all_scores, n_elig};
    parallel_rows(dense_row, &c, n_rows, nthreads);
    return 0;
}

/* Score arbitrary (query row, sequence-local key) pairs: key s of the query's
 * own sequence, scored by the dense formula.  Pairs are independent; blocks
 * of them run on `nthreads` threads. */
typedef struct {
    const uint16_t *Q, *K;
    const float* W;
    int H, d, n_seqs;
    const int32_t *q_off, *k_off, *rows, *keys;
    int64_t n_pairs;
    double* out;
} pairs_ctx;

enum { PAIR_BLOCK = 1024 };

static void pair_block(void* p, int64_t blk)
{
    pairs_ctx* c = (pairs_ctx*)p;
    double* q = (double*)malloc(sizeof(double) * ((size_t)c->H * c->d + c->H + c->d));
    double* w = q + (size_t)c->H * c->d;
    double* key = w + c->H;
    int64_t end = (blk + 1) * PAIR_BLOCK < c->n_pairs ? (blk + 1) * PAIR_BLOCK : c->n_pairs;
    for (int64_t i = blk * PAIR_BLOCK; i < end; ++i) {
        int b = seq_of_row(c->q_off, c->n_seqs, c->rows[i]);
        load_query(c->Q, c->W, c->rows[i], c->H, c->d, q, w);
        load_key(c->K, (int64_t)c->k_off[b] + c->keys[i], c->d, key);
        c->out[i] = indexer_score(q, w, key, c->H, c->d);
    }
    free(q);
}

int orc_pair_scores(const uint16_t* Q, const uint16_t* K, const float* W, int H, int d,
                    int n_seqs, const int32_t* q_off, const int32_t* k_off,
                    int64_t n_pairs, const int32_t* rows, const int32_t* keys, double* out,
                    int nthreads)
{
    pairs_ctx c = {Q, K, W, H, d, n_seqs, q_off, k_off, rows, keys, n_pairs, out};
    parallel_rows(pair_block, &c, (n_pairs + PAIR_BLOCK - 1) / PAIR_BLOCK, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ PIVOT */

/* Groups: within each sequence, consecutive runs of G query rows (the last
 * run may be shorter); numbered in sequence order [PIVOT abstract]. */
static int64_t count_groups(int n_seqs, const int32_t* q_off, int G)
{
    int64_t n = 0;
    for (int b = 0; b < n_seqs; ++b)
        n += ((int64_t)q_off[b + 1] - q_off[b] + G - 1) / G;
    return n;
}

static void group_info(int n_seqs, const int32_t* q_off, int G, int64_t g, int* seq, int64_t* first, int* size)
{
    for (int b = 0; b < n_seqs; ++b) {
        int64_t nq = (int64_t)q_off[b + 1] - q_off[b];
        int64_t ng = (nq + G - 1) / G;
        if (g < ng) {
            *seq = b;
            *first = q_off[b] + g * G;
            int64_t left = nq - g * G;
            *size = (int)(left < G ? left : G);
            return;
        }
        g -= ng;
    }
    *seq = -1; *first = 0; *size = 0;
}

int64_t orc_pivot_num_groups(int n_seqs, const int32_t* q_off, int G)
{
    return count_groups(n_seqs, q_off, G);
}

typedef struct {
    const uint16_t *Q, *K;
    const float* W;
    int H, d, n_seqs, G, C, k;
    const int32_t *q_off, *k_off, *q_pos, *groups;
    const int32_t* ext_cand;   /* [n_groups_sel, C] ascending, -1 padded, or NULL */
    int32_t* cand;             /* [n_sel, C] ascending, -1 padded */
    double* cand_score;        /* [n_sel, C] proxy score of cand */
    int32_t* reuse_idx;        /* [n_sel*G, k] */
    double* reuse_score;       /* proxy scores of reuse_idx */
    int32_t* refine_idx;       /* [n_sel*G, k] */
    double* refine_score;      /* indexer scores of refine_idx */
    double* proxy_q;           /* [n_sel, H*d] or NULL */
    double* proxy_w;           /* [n_sel, H] or NULL */
} pivot_ctx;

static int cmp_index(const void* pa, const void* pb)
{
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    return (a->i > b->i) - (a->i < b->i);
}

static void pivot_group(void* p, int64_t gi)
{
    pivot_ctx* c = (pivot_ctx*)p;
    int H = c->H, d = c->d, G = c->G, C = c->C, k = c->k;
    int b, size;
    int64_t first;
    group_info(c->n_seqs, c->q_off, G, c->groups[gi], &b, &first, &size);
    int64_t L = (int64_t)c->k_off[b + 1] - c->k_off[b];
    size_t hd = (size_t)H * d;

    /* Proxy query: mean over the group, in double; q rounded to bf16. */
    double* pq = (double*)calloc(hd + H + hd + H + d, sizeof(double));
    double* pw = pq + hd;
    double* q = pw + H;
    double* w = q + hd;
    double* key = w + H;
    int32_t p_last = -1;
    for (int j = 0; j < size; ++j) {
        load_query(c->Q, c->W, first + j, H, d, q, w);
        for (size_t e = 0; e < hd; ++e) pq[e] += q[e];
        for (int h = 0; h < H; ++h) pw[h] += w[h];
        if (c->q_pos[first + j] > p_last) p_last = c->q_pos[first + j];
    }
    for (size_t e = 0; e < hd; ++e) pq[e] = orc_round_bf16(pq[e] / size);
    for (int h = 0; h < H; ++h) pw[h] /= size;
    if (c->proxy_q) memcpy(c->proxy_q + gi * hd, pq, hd * sizeof(double));
    if (c->proxy_w) memcpy(c->proxy_w + gi * H, pw, H * sizeof(double));

    /* One shared scan over the prefix up to the group's last position. */
    int64_t n_scan = eligible_count(p_last, L);
    /* room for the scanned keys, or for C supplied candidates (they may lie past p_last) */
    int64_t n_room = n_scan > C ? n_scan : C;
    scored_t* cand = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_room > 0 ? n_room : 1));
    int64_t n_cand;
    if (c->ext_cand) {
        n_cand = 0;
        for (int j = 0; j < C; ++j) {
            int32_t s = c->ext_cand[gi * C + j];
            if (s < 0) break;
            load_key(c->K, (int64_t)c->k_off[b] + s, d, key);
            cand[n_cand].v = indexer_score(pq, pw, key, H, d);
            cand[n_cand].i = s;
            ++n_cand;
        }
    } else {
        for (int64_t s = 0; s < n_scan; ++s) {
            load_key(c->K, (int64_t)c->k_off[b] + s, d, key);
            cand[s].v = indexer_score(pq, pw, key, H, d);
            cand[s].i = (int32_t)s;
        }
        qsort(cand, (size_t)n_scan, sizeof(scored_t), cmp_scored);
        n_cand = n_scan < C ? n_scan : C;
    }
    /* Candidate set, reported in ascending index order. */
    scored_t* by_idx = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_cand > 0 ? n_cand : 1));
    memcpy(by_idx, cand, sizeof(scored_t) * (size_t)n_cand);
    qsort(by_idx, (size_t)n_cand, sizeof(scored_t), cmp_index);
    for (int j = 0; j < C; ++j) {
        c->cand[gi * C + j] = j < n_cand ? by_idx[j].i : -1;
        if (c->cand_score) c->cand_score[gi * C + j] = j < n_cand ? by_idx[j].v : NAN;
    }
    /* Ranking order of the candidates by proxy score. */
    qsort(cand, (size_t)n_cand, sizeof(scored_t), cmp_scored);

    scored_t* mine = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_cand > 0 ? n_cand : 1));
    for (int j = 0; j < G; ++j) {
        int64_t out = (gi * G + j) * (int64_t)k;
        if (j >= size) {
            for (int x = 0; x < k; ++x) {
                if (c->reuse_idx) c->reuse_idx[out + x] = -1;
                if (c->refine_idx) c->refine_idx[out + x] = -1;
            }
            continue;
        }
        int64_t t = first + j;
        int64_t lim = eligible_count(c->q_pos[t], L);   /* keys s < lim */
        /* Reuse: the proxy ranking, keeping only keys inside this query's prefix. */
        int taken = 0;
        for (int64_t x = 0; x < n_cand && taken < k; ++x)
            if (cand[x].i < lim) {
                if (c->reuse_idx) c->reuse_idx[out + taken] = cand[x].i;
                if (c->reuse_score) c->reuse_score[out + taken] = cand[x].v;
                ++taken;
            }
        for (; taken < k; ++taken) {
            if (c->reuse_idx) c->reuse_idx[out + taken] = -1;
            if (c->reuse_score) c->reuse_score[out + taken] = NAN;
        }
        /* Refine: this query's own indexer over its eligible candidates. */
        if (c->refine_idx) {
            load_query(c->Q, c->W, t, H, d, q, w);
            int64_t m = 0;
            for (int64_t x = 0; x < n_cand; ++x)
                if (by_idx[x].i < lim) {
                    load_key(c->K, (int64_t)c->k_off[b] + by_idx[x].i, d, key);
                    mine[m].v = indexer_score(q, w, key, H, d);
                    mine[m].i = by_idx[x].i;
                    ++m;
                }
            qsort(mine, (size_t)m, sizeof(scored_t), cmp_scored);
            for (int x = 0; x < k; ++x) {
                c->refine_idx[out + x] = x < m ? mine[x].i : -1;
                if (c->refine_score) c->refine_score[out + x] = x < m ? mine[x].v : NAN;
            }
        }
    }
    free(mine);
    free(by_idx);
    free(cand);
    free(pq);
}

/* PIVOT for the listed groups (global group numbers).  Query rows of group gi
 * occupy output rows gi*G .. gi*G+G-1 (rows past the group's size are -1).
 * ext_cand, when given, replaces the oracle's own candidate set (used to
 * check a second stage on another implementation's first-stage result). */
int orc_pivot(const uint16_t* Q, const uint16_t* K, const float* W, int H, int d,
              int n_seqs, const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
              int G, int C, int k, int n_sel, const int32_t* groups, const int32_t* ext_cand,
              int32_t* cand, double* cand_score, int32_t* reuse_idx, double* reuse_score,
              int32_t* refine_idx, double* refine_score, double* proxy_q, double* proxy_w,
              int nthreads)
{
    pivot_ctx c = {Q, K, W, H, d, n_seqs, G, C, k, q_off, k_off, q_pos, groups, ext_cand,
                   cand, cand_score, reuse_idx, reuse_score, refine_idx, refine_score, proxy_q, proxy_w};
    parallel_rows(pivot_group, &c, n_sel, nthreads);
    return 0;
}

/* ------------------------------------------------------------------- HISA */

/* Pooled block keys [HISA abstract: "pooled block representations"]: block j
 * of sequence b covers keys [j*B, min((j+1)*B, L_b)); its pooled key is the
 * mean of those keys.  Blocks of all sequences are stacked in sequence order. */
int orc_hisa_pool(const uint16_t* K, int d, int n_seqs, const int32_t* k_off, int B, double* pooled)
{
    double* key = (double*)malloc(sizeof(double) * d);
    int64_t out = 0;
    for (int b = 0; b < n_seqs; ++b) {
        int64_t L = (int64_t)k_off[b + 1] - k_off[b];
        for (int64_t j0 = 0; j0 < L; j0 += B, ++out) {
            int64_t j1 = j0 + B < L ? j0 + B : L;
            for (int i = 0; i < d; ++i) pooled[out * d + i] = 0.0;
            for (int64_t s = j0; s < j1; ++s) {
                load_key(K, (int64_t)k_off[b] + s, d, key);
                for (int i = 0; i < d; ++i) pooled[out * d + i] += key[i];
            }
            for (int i = 0; i < d; ++i) pooled[out * d + i] /= (double)(j1 - j0);
        }
    }
    free(key);
    return 0;
}

typedef struct {
    const uint16_t *Q, *K;
    const float* W;
    const double* pooled;
    int H, d, n_seqs, B, keep, k;
    const int32_t *q_off, *k_off, *q_pos, *rows;
    const int32_t* ext_kept;   /* [n_rows, keep+2] ascending, -1 padded, or NULL */
    int32_t* kept;             /* [n_rows, keep+2] ascending, -1 padded */
    double* block_scores;      /* [n_rows, max_blocks]: score of each middle block, NaN otherwise */
    int64_t max_blocks;
    int32_t* idx;              /* [n_rows, k] */
    double* top;               /* [n_rows, k] */
} hisa_ctx;

static void hisa_row(void* p, int64_t r)
{
    hisa_ctx* c = (hisa_ctx*)p;
    int H = c->H, d = c->d, B = c->B, k = c->k, n_keep = c->keep + 2;
    int64_t t = c->rows[r];
    int b = seq_of_row(c->q_off, c->n_seqs, t);
    int64_t L = (int64_t)c->k_off[b + 1] - c->k_off[b];
    int64_t n = eligible_count(c->q_pos[t], L);
    int64_t block_base = 0;   /* first pooled block of sequence b */
    for (int x = 0; x < b; ++x)
        block_base += ((int64_t)c->k_off[x + 1] - c->k_off[x] + B - 1) / B;

    double* q = (double*)malloc(sizeof(double) * ((size_t)H * d + H + d));
    double* w = q + (size_t)H * d;
    double* key = w + H;
    load_query(c->Q, c->W, t, H, d, q, w);

    int32_t* kept = c->kept + r * n_keep;
    for (int j = 0; j < n_keep; ++j) kept[j] = -1;
    if (c->block_scores)
        for (int64_t j = 0; j < c->max_blocks; ++j) c->block_scores[r * c->max_blocks + j] = NAN;
    int n_kept = 0;
    if (n > 0) {
        int64_t last = (n - 1) / B;
        int64_t n_mid = last > 1 ? last - 1 : 0;
        scored_t* mid = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_mid > 0 ? n_mid : 1));
        for (int64_t j = 0; j < n_mid; ++j) {
            mid[j].v = indexer_score(q, w, c->pooled + (block_base + 1 + j) * d, H, d);
            mid[j].i = (int32_t)(1 + j);
            if (c->block_scores) c->block_scores[r * c->max_blocks + 1 + j] = mid[j].v;
        }
        if (c->ext_kept) {
            for (int j = 0; j < n_keep; ++j) {
                if (c->ext_kept[r * n_keep + j] < 0) break;
                kept[n_kept++] = c->ext_kept[r * n_keep + j];
            }
        } else {
            qsort(mid, (size_t)n_mid, sizeof(scored_t), cmp_scored);
            int64_t n_sel = n_mid < c->keep ? n_mid : c->keep;
            kept[n_kept++] = 0;
            for (int64_t j = 0; j < n_sel; ++j) kept[n_kept++] = mid[j].i;
            if (last > 0) kept[n_kept++] = (int32_t)last;
            /* ascending block order */
            for (int a = 1; a < n_kept; ++a)
                for (int z = a; z > 0 && kept[z - 1] > kept[z]; --z) {
                    int32_t tmp = kept[z]; kept[z] = kept[z - 1]; kept[z - 1] = tmp;
                }
        }
        free(mid);
    }
    /* Token-level refinement: the indexer inside the kept blocks only. */
    scored_t* row = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_kept * (int64_t)B + 1));
    int64_t m = 0;
    for (int j = 0; j < n_kept; ++j) {
        int64_t s0 = (int64_t)kept[j] * B, s1 = s0 + B < n ? s0 + B : n;
        for (int64_t s = s0; s < s1; ++s) {
            load_key(c->K, (int64_t)c->k_off[b] + s, d, key);
            row[m].v = indexer_score(q, w, key, H, d);
            row[m].i = (int32_t)s;
            ++m;
        }
    }
    qsort(row, (size_t)m, sizeof(scored_t), cmp_scored);
    for (int j = 0; j < k; ++j) {
        c->idx[r * k + j] = j < m ? row[j].i : -1;
        if (c->top) c->top[r * k + j] = j < m ? row[j].v : NAN;
    }
    free(row);
    free(q);
}

/* HISA for the listed query rows.  pooled: output of orc_hisa_pool. */
int orc_hisa(const uint16_t* Q, const uint16_t* K, const float* W, const double* pooled, int H, int d,
             int n_seqs, const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
             int B, int keep, int k, int n_rows, const int32_t* rows, const int32_t* ext_kept,
             int32_t* kept, double* block_scores, int64_t max_blocks, int32_t* idx, double* top,
             int nthreads)
{
    hisa_ctx c = {Q, K, W, pooled, H, d, n_seqs, B, keep, k, q_off, k_off, q_pos, rows, ext_kept,
                  kept, block_scores, max_blocks, idx, top};
    parallel_rows(hisa_row, &c, n_rows, nthreads);
    return 0;
}
