/*
 * HISA CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header or table with the CUDA path.
 *
 * It computes, slowly and in double precision, what the HISA indexer computes:
 *
 *   HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse Attention
 *   (gptget.net summary, "Methodology"; Chinese summary, "方法详解" / method
 *   details; arXiv abstract):
 *     1. split the length-L prefix into contiguous blocks of size B and
 *        mean-pool each block's keys into one block representative;
 *     2. score every representative with the original indexer and keep the
 *        top-m blocks (block-level coarse filter);
 *     3. score every token of the kept blocks with the original indexer
 *        (token-level refinement);
 *     4. keep the final top-k tokens; their indices go to the sparse
 *        attention operator.
 *   The flat DSA scan (blog "Hierarchical Indexing Makes Sparse Attention
 *   Actually Fast", "How Fine-Grained Sparse Attention Works Today") scores
 *   every prefix token and keeps the top-k.  The multi-level search (same
 *   blog, "HISA's Approach") repeats steps 1-2 from the coarsest level of
 *   a tree of growing units down, each level scoring only the units inside
 *   the ones kept above it, before steps 3-4.
 *
 * The indexer score of a key x for one query row is
 *     score(q, x) = sum_h w_h * max(0, q_h . x)      over the H indexer heads,
 * the lightning-indexer form (the pages only call it a lightweight
 * dot-product scorer).  Readings where the pages are silent:
 *   - causal: a key at position s is visible to a query at t iff s <= t;
 *   - the trailing block is pooled over its visible tokens only;
 *   - the query's own block is always kept and counts inside m;
 *   - ties go to the lower index (tokens) and the lower block id (blocks);
 *   - output: the selected indices in ascending order, then -1 padding;
 *   - e4m3 keys are dequantised as fl32(e4m3 value * scale), the fp32
 *     product, and used in double from there.
 *
 * Parity pins: the tests check this file against exact rational brute force
 * on tiny inputs, closed-form pooled means, the B = 1 identity, one-hot score
 * cases and the m >= #blocks == flat-scan identity.
 *
 * Rows are independent; they are spread over POSIX threads.  A library sort
 * (qsort) is the only borrowed step.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { KEY_BF16 = 0, KEY_E4M3 = 1 };

typedef struct {
    const void* keys;    /* [batch, cap, d] bf16 bits or e4m3 codes */
    const float* scale;  /* [batch, cap] (e4m3 only) */
    int dtype, batch, cap, d;
} cache_t;

/* ---------------------------------------------------------------- values */

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP e4m3 ("fn"): 1 sign, 4 exponent (bias 7), 3 mantissa bits, no inf. */
static double e4m3_value(uint8_t c) {
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* Key row s of sequence b as the indexer sees it. */
static void key_row(const cache_t* c, int b, long s, double* x) {
    size_t base = ((size_t)b * c->cap + (size_t)s) * c->d;
    if (c->dtype == KEY_BF16) {
        const uint16_t* k = (const uint16_t*)c->keys + base;
        for (int e = 0; e < c->d; ++e) x[e] = bf16_value(k[e]);
    } else {
        const uint8_t* k = (const uint8_t*)c->keys + base;
        float sc = c->scale[(size_t)b * c->cap + (size_t)s];
        for (int e = 0; e < c->d; ++e) {
            /* one fp32 rounding of the exact product, then double */
            float v = (float)(e4m3_value(k[e]) * (double)sc);
            x[e] = (double)v;
        }
    }
}

/* ---------------------------------------------------------- the indexer */

/* q_h . x with four interleaved partial sums (fixed order, double). */
static double dot(const double* a, const double* x, int d) {
    double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
    int e = 0;
    for (; e + 4 <= d; e += 4) {
        s0 += a[e] * x[e];
        s1 += a[e + 1] * x[e + 1];
        s2 += a[e + 2] * x[e + 2];
        s3 += a[e + 3] * x[e + 3];
    }
    for (; e < d; ++e) s0 += a[e] * x[e];
    return (s0 + s1) + (s2 + s3);
}

/* score(q, x) = sum_h w_h * ReLU(q_h . x) */
static double indexer_score(const double* q, const double* w, int H, int d, const double* x) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h) {
        double z = dot(q + (size_t)h * d, x, d);
        acc += w[h] * (z > 0.0 ? z : 0.0);
    }
    return acc;
}

enum { POOL_MEAN = 0, POOL_MAX = 1 };

/* Step 1: block representative = mean of the block's visible keys
 * (tokens j*B .. min((j+1)*B, n) - 1), or, with POOL_MAX, their elementwise
 * maximum (blog "Hierarchical Indexing Makes Sparse Attention Actually Fast",
 * "HISA's Approach": summary nodes pool their token group by mean or by max). */
static void pool_block(const cache_t* c, int b, int B, long j, long n, double* mu, double* tmp,
                       int mode) {
    long s0 = j * (long)B, s1 = s0 + B < n ? s0 + B : n;
    if (mode == POOL_MAX) {
        for (long s = s0; s < s1; ++s) {
            key_row(c, b, s, tmp);
            for (int e = 0; e < c->d; ++e) mu[e] = (s == s0 || tmp[e] > mu[e]) ? tmp[e] : mu[e];
        }
        return;
    }
    for (int e = 0; e < c->d; ++e) mu[e] = 0.0;
    for (long s = s0; s < s1; ++s) {
        key_row(c, b, s, tmp);
        for (int e = 0; e < c->d; ++e) mu[e] += tmp[e];
    }
    for (int e = 0; e < c->d; ++e) mu[e] /= (double)(s1 - s0);
}

/* ------------------------------------------------------------ selection */

typedef struct { double v; long i; } scored_t;

/* higher value first; equal values: lower index first */
static int by_value_then_index(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int by_index(const void* pa, const void* pb) {
    long a = ((const scored_t*)pa)->i, b = ((const scored_t*)pb)->i;
    return (a > b) - (a < b);
}

/* Keep the first k of `items` under (value desc, index asc); write them in
 * ascending index order into idx/val (padding -1 / NaN up to k). */
static void keep_top(scored_t* items, long n, int k, int32_t* idx, double* val) {
    qsort(items, (size_t)n, sizeof(scored_t), by_value_then_index);
    long kept = n < k ? n : k;
    qsort(items, (size_t)kept, sizeof(scored_t), by_index);
    for (long r = 0; r < k; ++r) {
        idx[r] = r < kept ? (int32_t)items[r].i : -1;
        if (val) val[r] = r < kept ? items[r].v : NAN;
    }
}

/* ------------------------------------------------------------ threading */

typedef void (*row_fn)(void* ctx, int row, void* scratch);

typedef struct {
    row_fn fn;
    void* ctx;
    int n_rows, n_threads, tid;
    size_t scratch_bytes;
    int failed;
} worker_t;

static void* worker_main(void* p) {
    worker_t* w = (worker_t*)p;
    void* scratch = malloc(w->scratch_bytes);
    if (!scratch) { w->failed = 1; return NULL; }
    for (int r = w->tid; r < w->n_rows; r += w->n_threads) w->fn(w->ctx, r, scratch);
    free(scratch);
    return NULL;
}

static int for_rows(row_fn fn, void* ctx, int n_rows, int n_threads, size_t scratch_bytes) {
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_rows) n_threads = n_rows > 0 ? n_rows : 1;
    worker_t* ws = (worker_t*)calloc((size_t)n_threads, sizeof(worker_t));
    pthread_t* th = (pthread_t*)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!ws || !th) { free(ws); free(th); return 3; }
    int rc = 0;
    for (int t = 0; t < n_threads; ++t) {
        ws[t] = (worker_t){fn, ctx, n_rows, n_threads, t, scratch_bytes, 0};
        if (pthread_create(&th[t], NULL, worker_main, &ws[t]) != 0) {
            worker_main(&ws[t]);   /* run inline if a thread cannot start */
            th[t] = 0;
        }
    }
    for (int t = 0; t < n_threads; ++t) {
        if (th[t]) pthread_join(th[t], NULL);
        if (ws[t].failed) rc = 3;
    }
    free(ws);
    free(th);
    return rc;
}

/* ---------------------------------------------------------- query rows */

typedef struct {
    cache_t c;
    int B;
    const int32_t* lens;
    const uint16_t* Q;    /* [n_q, H, d] bf16 */
    const float* w;       /* [n_q, H] */
    const int32_t* q_seq;
    const int32_t* q_pos; /* NULL: last position of the sequence */
    int n_q, H, m, k, nbmax;
    /* HISA outputs */
    int32_t* idx; double* score;
    int32_t* blocks; int32_t* nblocks; double* block_scores; int64_t* counts;
    /* refine inputs */
    const int32_t* in_blocks; const int32_t* in_nblocks; int mm;
    double* cand_scores;
    /* flat output */
    double* all_scores;
    int bad;
    int pool_mode;
    /* tree: branching factor, superblocks kept, outputs */
    int bf, W;
    int32_t* sblocks; int32_t* nsblocks;
    /* search of any depth: levels finest first (level 0 = blocks of B) */
    int n_lv;
    const int* lv_B; const int* lv_W;
    int32_t* lv_kept; int32_t* lv_nkept; int lv_ld; int maxW; long lv_items;
} job_t;

static long row_position(const job_t* J, int i, int* b_out) {
    int b = J->q_seq[i];
    *b_out = b;
    if (b < 0 || b >= J->c.batch) return -1;
    long t = J->q_pos ? J->q_pos[i] : (long)J->lens[b] - 1;
    if (t < 0 || t >= J->lens[b] || J->lens[b] > J->c.cap) return -1;
    return t;
}

static void load_query(const job_t* J, int i, double* q, double* w) {
    const uint16_t* Qi = J->Q + (size_t)i * J->H * J->c.d;
    for (int x = 0; x < J->H * J->c.d; ++x) q[x] = bf16_value(Qi[x]);
    for (int h = 0; h < J->H; ++h) w[h] = (double)J->w[(size_t)i * J->H + h];
}

static size_t row_scratch_bytes(int H, int d, long n_items) {
    return sizeof(double) * ((size_t)H * d + H + 2 * (size_t)d) + sizeof(scored_t) * (size_t)n_items;
}

/* Token-level refinement on a given set of blocks (steps 3-4). */
static void refine_blocks(const job_t* J, int i, int b, long t, const double* q, const double* w,
                          const int32_t* blk, int nblk, scored_t* items, double* x,
                          int32_t* idx, double* val, double* cand) {
    (void)i;
    long n = 0;
    for (int r = 0; r < nblk; ++r) {
        for (int o = 0; o < J->B; ++o) {
            long s = (long)blk[r] * J->B + o;
            double v = NAN;
            if (blk[r] >= 0 && s <= t) {
                key_row(&J->c, b, s, x);
                v = indexer_score(q, w, J->H, J->c.d, x);
                items[n].v = v;
                items[n].i = s;
                ++n;
            }
            if (cand) cand[(size_t)r * J->B + o] = v;
        }
    }
    keep_top(items, n, J->k, idx, val);
}

static void hisa_row(void* ctx, int i, void* scratch) {
    job_t* J = (job_t*)ctx;
    int H = J->H, d = J->c.d, B = J->B, b;
    long t = row_position(J, i, &b);
    int32_t* idx = J->idx + (size_t)i * J->k;
    double* val = J->score ? J->score + (size_t)i * J->k : NULL;
    int32_t* blocks = J->blocks ? J->blocks + (size_t)i * J->m : NULL;
    if (t < 0) {
        J->bad = 1;
        for (int r = 0; r < J->k; ++r) { idx[r] = -1; if (val) val[r] = NAN; }
        return;
    }
    double* q = (double*)scratch;
    double* w = q + (size_t)H * d;
    double* mu = w + H;
    double* x = mu + d;
    scored_t* items = (scored_t*)(x + d);

    load_query(J, i, q, w);
    long n_t = t + 1;
    long nb = (n_t + B - 1) / B;

    /* steps 1-2: pool every visible block, score the representatives */
    double* S = J->block_scores ? J->block_scores + (size_t)i * J->nbmax : NULL;
    if (S) for (int j = 0; j < J->nbmax; ++j) S[j] = NAN;
    for (long j = 0; j < nb; ++j) {
        pool_block(&J->c, b, B, j, n_t, mu, x, J->pool_mode);
        double sj = indexer_score(q, w, H, d, mu);
        if (S) S[j] = sj;
        items[j].v = sj;
        items[j].i = j;
    }
    /* keep the own block (nb-1) plus the best m-1 of the others */
    int32_t chosen[4096];
    int n_chosen;
    if (nb <= J->m) {
        n_chosen = (int)nb;
        for (int j = 0; j < n_chosen; ++j) chosen[j] = j;
    } else {
        qsort(items, (size_t)(nb - 1), sizeof(scored_t), by_value_then_index);
        n_chosen = J->m;
        for (int r = 0; r < J->m - 1; ++r) chosen[r] = (int32_t)items[r].i;
        chosen[J->m - 1] = (int32_t)(nb - 1);
        /* ascending block order */
        for (int a = 1; a < n_chosen; ++a)
            for (int c2 = a; c2 > 0 && chosen[c2 - 1] > chosen[c2]; --c2) {
                int32_t tmp = chosen[c2]; chosen[c2] = chosen[c2 - 1]; chosen[c2 - 1] = tmp;
            }
    }
    if (blocks) for (int r = 0; r < J->m; ++r) blocks[r] = r < n_chosen ? chosen[r] : -1;
    if (J->nblocks) J->nblocks[i] = n_chosen;
    if (J->counts) {
        J->counts[2 * (size_t)i] = nb;                          /* block scores */
        J->counts[2 * (size_t)i + 1] = (int64_t)n_chosen * B;   /* token slots */
    }
    /* steps 3-4 */
    refine_blocks(J, i, b, t, q, w, chosen, n_chosen, items, x, idx, val, NULL);
}

/* Three-level search (blog "Hierarchical Indexing Makes Sparse Attention
 * Actually Fast", "HISA's Approach": a multi-level summary searched top down,
 * keeping the best branches at each level).  Superblocks of bf blocks
 * (bf * B tokens) are pooled and scored; the own superblock plus the best
 * W - 1 others are kept; the visible blocks under them are pooled and scored;
 * the own block plus the best m - 1 of those are kept; their tokens are
 * refined as in the two-stage search. */
static void tree_row(void* ctx, int i, void* scratch) {
    job_t* J = (job_t*)ctx;
    int H = J->H, d = J->c.d, B = J->B, bf = J->bf, b;
    long B2 = (long)B * bf;
    long t = row_position(J, i, &b);
    int32_t* idx = J->idx + (size_t)i * J->k;
    double* val = J->score ? J->score + (size_t)i * J->k : NULL;
    int32_t* sblocks = J->sblocks ? J->sblocks + (size_t)i * J->W : NULL;
    int32_t* blocks = J->blocks ? J->blocks + (size_t)i * J->m : NULL;
    if (t < 0) {
        J->bad = 1;
        for (int r = 0; r < J->k; ++r) { idx[r] = -1; if (val) val[r] = NAN; }
        return;
    }
    double* q = (double*)scratch;
    double* w = q + (size_t)H * d;
    double* mu = w + H;
    double* x = mu + d;
    scored_t* items = (scored_t*)(x + d);
    load_query(J, i, q, w);
    long n_t = t + 1;
    long nb = (n_t + B - 1) / B;
    long ns = (n_t + B2 - 1) / B2;

    /* level 2: superblocks */
    for (long j = 0; j < ns; ++j) {
        pool_block(&J->c, b, (int)B2, j, n_t, mu, x, J->pool_mode);
        items[j].v = indexer_score(q, w, H, d, mu);
        items[j].i = j;
    }
    int32_t skept[4096];
    int n_s;
    if (ns <= J->W) {
        n_s = (int)ns;
        for (int j = 0; j < n_s; ++j) skept[j] = j;
    } else {
        qsort(items, (size_t)(ns - 1), sizeof(scored_t), by_value_then_index);
        n_s = J->W;
        for (int r = 0; r < J->W - 1; ++r) skept[r] = (int32_t)items[r].i;
        skept[J->W - 1] = (int32_t)(ns - 1);
        for (int a = 1; a < n_s; ++a)
            for (int c2 = a; c2 > 0 && skept[c2 - 1] > skept[c2]; --c2) {
                int32_t tmp = skept[c2]; skept[c2] = skept[c2 - 1]; skept[c2 - 1] = tmp;
            }
    }
    if (sblocks) for (int r = 0; r < J->W; ++r) sblocks[r] = r < n_s ? skept[r] : -1;
    if (J->nsblocks) J->nsblocks[i] = n_s;

    /* level 1: the visible blocks under the kept superblocks, own block apart */
    long nc = 0;
    for (int r = 0; r < n_s; ++r)
        for (long j = (long)skept[r] * bf; j < (long)(skept[r] + 1) * bf && j < nb - 1; ++j) {
            pool_block(&J->c, b, B, j, n_t, mu, x, J->pool_mode);
            items[nc].v = indexer_score(q, w, H, d, mu);
            items[nc].i = j;
            ++nc;
        }
    int32_t chosen[4096];
    int n_chosen;
    if (nc + 1 <= J->m) {
        n_chosen = (int)nc + 1;
        for (long r = 0; r < nc; ++r) chosen[r] = (int32_t)items[r].i;
    } else {
        qsort(items, (size_t)nc, sizeof(scored_t), by_value_then_index);
        n_chosen = J->m;
        for (int r = 0; r < J->m - 1; ++r) chosen[r] = (int32_t)items[r].i;
    }
    chosen[n_chosen - 1] = (int32_t)(nb - 1);
    for (int a = 1; a < n_chosen; ++a)
        for (int c2 = a; c2 > 0 && chosen[c2 - 1] > chosen[c2]; --c2) {
            int32_t tmp = chosen[c2]; chosen[c2] = chosen[c2 - 1]; chosen[c2 - 1] = tmp;
        }
    if (blocks) for (int r = 0; r < J->m; ++r) blocks[r] = r < n_chosen ? chosen[r] : -1;
    if (J->nblocks) J->nblocks[i] = n_chosen;
    if (J->counts) {
        J->counts[3 * (size_t)i] = ns;                              /* superblock scores */
        J->counts[3 * (size_t)i + 1] = nc + 1;                      /* block scores */
        J->counts[3 * (size_t)i + 2] = (int64_t)n_chosen * B;       /* token slots */
    }
    refine_blocks(J, i, b, t, q, w, chosen, n_chosen, items, x, idx, val, NULL);
}

/* Search of any depth (blog "Hierarchical Indexing Makes Sparse Attention
 * Actually Fast", "HISA's Approach" and "The Complexity Win": the summary is
 * a tree searched from the root down, the best branches kept at each level).
 * Level l groups the keys into units of lv_B[l] tokens (lv_B[0] = B, each
 * size a multiple of the one below), pooled from the keys like blocks.  From
 * the coarsest level down: the candidates are every visible unit (coarsest
 * level) or the visible units inside the units kept one level up; the own
 * unit, the one holding the query position, is kept without being compared,
 * together with the best lv_W[l] - 1 candidates by (score desc, id asc).
 * The tokens of the kept level-0 blocks are then refined as in the
 * two-stage search.  counts[l] is the units of level l scored (candidates
 * plus the own unit), counts[n_lv] the token slots scored. */
static void levels_row(void* ctx, int i, void* scratch) {
    job_t* J = (job_t*)ctx;
    int H = J->H, d = J->c.d, b;
    long t = row_position(J, i, &b);
    int32_t* idx = J->idx + (size_t)i * J->k;
    double* val = J->score ? J->score + (size_t)i * J->k : NULL;
    if (t < 0) {
        J->bad = 1;
        for (int r = 0; r < J->k; ++r) { idx[r] = -1; if (val) val[r] = NAN; }
        return;
    }
    double* q = (double*)scratch;
    double* w = q + (size_t)H * d;
    double* mu = w + H;
    double* x = mu + d;
    scored_t* items = (scored_t*)(x + d);
    int32_t* cur = (int32_t*)(items + J->lv_items);
    int32_t* up = cur + J->maxW;                   /* the kept units one level up */
    load_query(J, i, q, w);
    long n_t = t + 1;
    int n_up = 0;
    for (int l = J->n_lv - 1; l >= 0; --l) {
        long Bl = J->lv_B[l];
        long nu = (n_t + Bl - 1) / Bl;             /* visible units; the own one is nu - 1 */
        long nc = 0;
        if (l == J->n_lv - 1) {
            for (long j = 0; j < nu - 1; ++j) {
                pool_block(&J->c, b, (int)Bl, j, n_t, mu, x, J->pool_mode);
                items[nc].v = indexer_score(q, w, H, d, mu);
                items[nc].i = j;
                ++nc;
            }
        } else {
            long bf = J->lv_B[l + 1] / Bl;         /* units of this level per unit above */
            for (int r = 0; r < n_up; ++r)
                for (long j = (long)up[r] * bf; j < (long)(up[r] + 1) * bf && j < nu - 1; ++j) {
                    pool_block(&J->c, b, (int)Bl, j, n_t, mu, x, J->pool_mode);
                    items[nc].v = indexer_score(q, w, H, d, mu);
                    items[nc].i = j;
                    ++nc;
                }
        }
        int W = J->lv_W[l], n_keep;
        if (nc + 1 <= W) {
            n_keep = (int)nc + 1;
            for (long r = 0; r < nc; ++r) cur[r] = (int32_t)items[r].i;
        } else {
            qsort(items, (size_t)nc, sizeof(scored_t), by_value_then_index);
            n_keep = W;
            for (int r = 0; r < W - 1; ++r) cur[r] = (int32_t)items[r].i;
        }
        cur[n_keep - 1] = (int32_t)(nu - 1);
        for (int a = 1; a < n_keep; ++a)
            for (int c2 = a; c2 > 0 && cur[c2 - 1] > cur[c2]; --c2) {
                int32_t tmp = cur[c2]; cur[c2] = cur[c2 - 1]; cur[c2 - 1] = tmp;
            }
        if (J->lv_kept) {
            int32_t* o = J->lv_kept + (size_t)i * J->lv_ld;
            for (int j = 0; j < l; ++j) o += J->lv_W[j];
            for (int r = 0; r < W; ++r) o[r] = r < n_keep ? cur[r] : -1;
        }
        if (J->lv_nkept) J->lv_nkept[(size_t)i * J->n_lv + l] = n_keep;
        if (J->counts) J->counts[(size_t)i * (J->n_lv + 1) + l] = nc + 1;
        int32_t* tmp = up; up = cur; cur = tmp;
        n_up = n_keep;
    }
    if (J->counts) J->counts[(size_t)i * (J->n_lv + 1) + J->n_lv] = (int64_t)n_up * J->B;
    refine_blocks(J, i, b, t, q, w, up, n_up, items, x, idx, val, NULL);
}

static void refine_row(void* ctx, int i, void* scratch) {
    job_t* J = (job_t*)ctx;
    int H = J->H, d = J->c.d, b;
    long t = row_position(J, i, &b);
    int32_t* idx = J->idx + (size_t)i * J->k;
    double* val = J->score ? J->score + (size_t)i * J->k : NULL;
    double* cand = J->cand_scores ? J->cand_scores + (size_t)i * J->mm * J->B : NULL;
    int nblk = J->in_nblocks[i];
    if (t < 0 || nblk < 0 || nblk > J->mm) {
        J->bad = 1;
        for (int r = 0; r < J->k; ++r) { idx[r] = -1; if (val) val[r] = NAN; }
        return;
    }
    double* q = (double*)scratch;
    double* w = q + (size_t)H * d;
    double* x = w + H + d;
    scored_t* items = (scored_t*)(x + d);
    load_query(J, i, q, w);
    if (cand) for (long s = 0; s < (long)J->mm * J->B; ++s) cand[s] = NAN;
    refine_blocks(J, i, b, t, q, w, J->in_blocks + (size_t)i * J->mm, nblk, items, x, idx, val, cand);
}

/* Flat scan: every visible token is a candidate. */
static void flat_row(void* ctx, int i, void* scratch) {
    job_t* J = (job_t*)ctx;
    int H = J->H, d = J->c.d, b;
    long t = row_position(J, i, &b);
    int32_t* idx = J->idx + (size_t)i * J->k;
    double* val = J->score ? J->score + (size_t)i * J->k : NULL;
    double* all = J->all_scores ? J->all_scores + (size_t)i * J->c.cap : NULL;
    if (t < 0) {
        J->bad = 1;
        for (int r = 0; r < J->k; ++r) { idx[r] = -1; if (val) val[r] = NAN; }
        return;
    }
    double* q = (double*)scratch;
    double* w = q + (size_t)H * d;
    double* x = w + H + d;
    scored_t* items = (scored_t*)(x + d);
    load_query(J, i, q, w);
    if (all) for (long s = 0; s < J->c.cap; ++s) all[s] = NAN;
    for (long s = 0; s <= t; ++s) {
        key_row(&J->c, b, s, x);
        items[s].v = indexer_score(q, w, H, d, x);
        items[s].i = s;
        if (all) all[s] = items[s].v;
    }
    keep_top(items, t + 1, J->k, idx, val);
}

static int check_cache(const void* keys, const float* scale, int dtype, int batch, int cap, int d) {
    if (!keys || batch < 1 || cap < 1 || d < 1) return 1;
    if (dtype != KEY_BF16 && dtype != KEY_E4M3) return 1;
    if (dtype == KEY_E4M3 && !scale) return 1;
    return 0;
}

/* ------------------------------------------------------------- exports */

/* Cache-level pooling: pooled[b, j, :] = mean (or max) of keys j*B .. min((j+1)B, len[b]) - 1;
 * blocks at or past len[b] are left untouched. */
int hisa_oracle_pool(const void* keys, const float* scale, int dtype, int batch, int cap, int d,
                     int B, int pool_mode, const int32_t* lens, double* pooled) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || B < 1 || !lens || !pooled ||
        (pool_mode != POOL_MEAN && pool_mode != POOL_MAX))
        return 1;
    cache_t c = {keys, scale, dtype, batch, cap, d};
    long nblk = (cap + B - 1) / B;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)d);
    if (!tmp) return 3;
    for (int b = 0; b < batch; ++b) {
        long n = lens[b];
        if (n < 0 || n > cap) { free(tmp); return 1; }
        for (long j = 0; j * B < n; ++j)
            pool_block(&c, b, B, j, n, pooled + ((size_t)b * nblk + (size_t)j) * d, tmp, pool_mode);
    }
    free(tmp);
    return 0;
}

int hisa_oracle_select(const void* keys, const float* scale, int dtype, int batch, int cap, int d,
                       int B, int pool_mode, const int32_t* lens, const uint16_t* Q, const float* w,
                       const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m, int k,
                       int n_threads, int32_t* idx, double* score, int32_t* blocks,
                       int32_t* nblocks, double* block_scores, int64_t* counts) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || B < 1 || !lens || !Q || !w || !q_seq ||
        n_q < 0 || H < 1 || m < 1 || m > 4096 || k < 1 || !idx ||
        (pool_mode != POOL_MEAN && pool_mode != POOL_MAX))
        return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.c = (cache_t){keys, scale, dtype, batch, cap, d};
    J.pool_mode = pool_mode;
    J.B = B; J.lens = lens; J.Q = Q; J.w = w; J.q_seq = q_seq; J.q_pos = q_pos;
    J.n_q = n_q; J.H = H; J.m = m; J.k = k; J.nbmax = (cap + B - 1) / B;
    J.idx = idx; J.score = score; J.blocks = blocks; J.nblocks = nblocks;
    J.block_scores = block_scores; J.counts = counts;
    long items = J.nbmax > (long)m * B ? J.nbmax : (long)m * B;
    int rc = for_rows(hisa_row, &J, n_q, n_threads, row_scratch_bytes(H, d, items));
    return rc ? rc : (J.bad ? 2 : 0);
}

int hisa_oracle_tree_select(const void* keys, const float* scale, int dtype, int batch, int cap,
                            int d, int B, int bf, int pool_mode, const int32_t* lens,
                            const uint16_t* Q, const float* w, const int32_t* q_seq,
                            const int32_t* q_pos, int n_q, int H, int W, int m, int k,
                            int n_threads, int32_t* idx, double* score, int32_t* sblocks,
                            int32_t* nsblocks, int32_t* blocks, int32_t* nblocks, int64_t* counts) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || B < 1 || bf < 1 || !lens || !Q || !w ||
        !q_seq || n_q < 0 || H < 1 || W < 1 || W > 4096 || m < 1 || m > 4096 || k < 1 || !idx ||
        (pool_mode != POOL_MEAN && pool_mode != POOL_MAX))
        return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.c = (cache_t){keys, scale, dtype, batch, cap, d};
    J.pool_mode = pool_mode;
    J.B = B; J.bf = bf; J.W = W; J.lens = lens; J.Q = Q; J.w = w; J.q_seq = q_seq; J.q_pos = q_pos;
    J.n_q = n_q; J.H = H; J.m = m; J.k = k; J.nbmax = (cap + B - 1) / B;
    J.idx = idx; J.score = score; J.sblocks = sblocks; J.nsblocks = nsblocks;
    J.blocks = blocks; J.nblocks = nblocks; J.counts = counts;
    long items = J.nbmax > (long)m * B ? J.nbmax : (long)m * B;
    int rc = for_rows(tree_row, &J, n_q, n_threads, row_scratch_bytes(H, d, items));
    return rc ? rc : (J.bad ? 2 : 0);
}

int hisa_oracle_levels_select(const void* keys, const float* scale, int dtype, int batch, int cap,
                              int d, int n_levels, const int* level_B, const int* keep,
                              int pool_mode, const int32_t* lens, const uint16_t* Q, const float* w,
                              const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int k,
                              int n_threads, int32_t* idx, double* score, int32_t* kept,
                              int32_t* nkept, int64_t* counts) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || n_levels < 1 || n_levels > 8 || !level_B ||
        !keep || !lens || !Q || !w || !q_seq || n_q < 0 || H < 1 || k < 1 || !idx ||
        (pool_mode != POOL_MEAN && pool_mode != POOL_MAX))
        return 1;
    int ld = 0, maxW = 0;
    for (int l = 0; l < n_levels; ++l) {
        if (level_B[l] < 1 || keep[l] < 1 || keep[l] > (1 << 20)) return 1;
        if (l > 0 && level_B[l] % level_B[l - 1] != 0) return 1;
        ld += keep[l];
        if (keep[l] > maxW) maxW = keep[l];
    }
    job_t J;
    memset(&J, 0, sizeof J);
    J.c = (cache_t){keys, scale, dtype, batch, cap, d};
    J.pool_mode = pool_mode;
    J.B = level_B[0]; J.lens = lens; J.Q = Q; J.w = w; J.q_seq = q_seq; J.q_pos = q_pos;
    J.n_q = n_q; J.H = H; J.m = keep[0]; J.k = k; J.nbmax = (cap + J.B - 1) / J.B;
    J.idx = idx; J.score = score; J.counts = counts;
    J.n_lv = n_levels; J.lv_B = level_B; J.lv_W = keep;
    J.lv_kept = kept; J.lv_nkept = nkept; J.lv_ld = ld; J.maxW = maxW;
    /* candidates at any level are at most the level-0 blocks; the tokens at most m * B */
    J.lv_items = J.nbmax > (long)keep[0] * J.B ? J.nbmax : (long)keep[0] * J.B;
    size_t bytes = row_scratch_bytes(H, d, J.lv_items) + 2 * sizeof(int32_t) * (size_t)maxW;
    int rc = for_rows(levels_row, &J, n_q, n_threads, bytes);
    return rc ? rc : (J.bad ? 2 : 0);
}

int hisa_oracle_refine(const void* keys, const float* scale, int dtype, int batch, int cap, int d,
                       int B, const int32_t* lens, const uint16_t* Q, const float* w,
                       const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int k,
                       const int32_t* in_blocks, const int32_t* in_nblocks, int mm, int n_threads,
                       int32_t* idx, double* score, double* cand_scores) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || B < 1 || !lens || !Q || !w || !q_seq ||
        n_q < 0 || H < 1 || k < 1 || mm < 1 || !in_blocks || !in_nblocks || !idx)
        return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.c = (cache_t){keys, scale, dtype, batch, cap, d};
    J.B = B; J.lens = lens; J.Q = Q; J.w = w; J.q_seq = q_seq; J.q_pos = q_pos;
    J.n_q = n_q; J.H = H; J.k = k; J.in_blocks = in_blocks; J.in_nblocks = in_nblocks;
    J.mm = mm; J.idx = idx; J.score = score; J.cand_scores = cand_scores;
    int rc = for_rows(refine_row, &J, n_q, n_threads, row_scratch_bytes(H, d, (long)mm * B));
    return rc ? rc : (J.bad ? 2 : 0);
}

int hisa_oracle_flat(const void* keys, const float* scale, int dtype, int batch, int cap, int d,
                     const int32_t* lens, const uint16_t* Q, const float* w, const int32_t* q_seq,
                     const int32_t* q_pos, int n_q, int H, int k, int n_threads, int32_t* idx,
                     double* score, double* all_scores) {
    if (check_cache(keys, scale, dtype, batch, cap, d) || !lens || !Q || !w || !q_seq || n_q < 0 ||
        H < 1 || k < 1 || !idx)
        return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.c = (cache_t){keys, scale, dtype, batch, cap, d};
    J.B = 1; J.lens = lens; J.Q = Q; J.w = w; J.q_seq = q_seq; J.q_pos = q_pos;
    J.n_q = n_q; J.H = H; J.k = k; J.idx = idx; J.score = score; J.all_scores = all_scores;
    int rc = for_rows(flat_row, &J, n_q, n_threads, row_scratch_bytes(H, d, cap));
    return rc ? rc : (J.bad ? 2 : 0);
}

/* The selection rule alone, on given fp32 values: per row keep the k largest
 * (ties: lower index), indices ascending, -1 padded.  Both sides decide on
 * the same fp32 numbers here, so the result is exact. */
int hisa_oracle_topk_f32(const float* x, int rows, int n, int k, int32_t* idx) {
    if (!x || rows < 0 || n < 0 || k < 1 || !idx) return 1;
    scored_t* items = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    if (!items) return 3;
    for (int r = 0; r < rows; ++r) {
        for (int s = 0; s < n; ++s) {
            items[s].v = (double)x[(size_t)r * n + s];
            items[s].i = s;
        }
        keep_top(items, n, k, idx + (size_t)r * k, NULL);
    }
    free(items);
    return 0;
}

/* ----------------------------------------------------- sparse attention */

/* The consumer of the selection (blog "Hierarchical Indexing Makes Sparse
 * Attention Actually Fast", "How Fine-Grained Sparse Attention Works Today":
 * the second stage attends to the selected top-K tokens only).  A synthetic
 * multi-query operator, by its definition: for row i (sequence b) and head h,
 * over the list entries j whose index s_j satisfies 0 <= s_j < len[b],
 *     a_j = scale * Qa[i,h] . K[b, s_j]
 *     out[i,h] = sum_j exp(a_j) V[b, s_j] / sum_j exp(a_j)
 *     lse[i,h] = log sum_j exp(a_j)
 * in double (the exponentials are taken relative to the largest a_j, which
 * changes nothing but the range).  No valid entry: out = 0, lse = -inf. */
typedef struct {
    const uint16_t* Qa; const uint16_t* K; const uint16_t* V;
    const int32_t* lens; const int32_t* q_seq; const int32_t* idx;
    int Ha, batch, cap, d, k;
    double scale;
    double* out; double* lse;
} attn_job_t;

static void attn_row(void* ctx, int i, void* scratch) {
    const attn_job_t* J = (const attn_job_t*)ctx;
    double* a = (double*)scratch;             /* [k] */
    double* x = a + J->k;                     /* [d] */
    const int b = J->q_seq[i];
    const int n = (b >= 0 && b < J->batch) ? J->lens[b] : 0;
    for (int h = 0; h < J->Ha; ++h) {
        double* o = J->out + ((size_t)i * J->Ha + h) * J->d;
        for (int e = 0; e < J->d; ++e) o[e] = 0.0;
        const uint16_t* q = J->Qa + ((size_t)i * J->Ha + h) * J->d;
        double amax = -INFINITY;
        for (int j = 0; j < J->k; ++j) {
            const int s = J->idx[(size_t)i * J->k + j];
            if (s < 0 || s >= n) { a[j] = NAN; continue; }
            const uint16_t* kr = J->K + ((size_t)b * J->cap + s) * J->d;
            double z = 0.0;
            for (int e = 0; e < J->d; ++e) z += bf16_value(q[e]) * bf16_value(kr[e]);
            a[j] = J->scale * z;
            if (a[j] > amax) amax = a[j];
        }
        if (amax == -INFINITY) {
            if (J->lse) J->lse[(size_t)i * J->Ha + h] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int e = 0; e < J->d; ++e) x[e] = 0.0;
        for (int j = 0; j < J->k; ++j) {
            if (isnan(a[j])) continue;
            const int s = J->idx[(size_t)i * J->k + j];
            const double p = exp(a[j] - amax);
            const uint16_t* vr = J->V + ((size_t)b * J->cap + s) * J->d;
            sum += p;
            for (int e = 0; e < J->d; ++e) x[e] += p * bf16_value(vr[e]);
        }
        for (int e = 0; e < J->d; ++e) o[e] = x[e] / sum;
        if (J->lse) J->lse[(size_t)i * J->Ha + h] = amax + log(sum);
    }
}

int hisa_oracle_sparse_attn(const uint16_t* Qa, int Ha, const uint16_t* K, const uint16_t* V,
                            const int32_t* lens, int batch, int cap, int d, const int32_t* q_seq,
                            const int32_t* idx, int n_q, int k, double scale, int n_threads,
                            double* out, double* lse) {
    if (!Qa || !K || !V || !lens || !q_seq || !idx || !out || Ha < 1 || batch < 1 || cap < 1 ||
        d < 1 || n_q < 0 || k < 1)
        return 1;
    attn_job_t J = {Qa, K, V, lens, q_seq, idx, Ha, batch, cap, d, k, scale, out, lse};
    return for_rows(attn_row, &J, n_q, n_threads, sizeof(double) * ((size_t)k + (size_t)d));
}
