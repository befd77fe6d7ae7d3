/*
 * fa_oracle.c -- plain, slow, fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (the plain definition, written out, no blocking, no
 * online softmax, no fusion):
 *
 *   Standard attention is softmax(Q K^T / sqrt(d_k)) V
 *     ("optimizing-attention-flash", Workflow 1 / Step 2, the "standard
 *      attention" snippet it replaces; Step 4, the accuracy check at
 *      scale 1/8 for d = 64).
 *   The tiled method computes exactly this, with no approximation
 *     ("Что такое FlashAttention…", section "Основной механизм простыми
 *      словами" and section "Структурная корректность и фактическая
 *      правильность").
 *   causal=True hides future keys; window_size=(left,right) keeps only keys
 *   within `left` before and `right` after the query, -1 meaning unbounded;
 *   K/V may carry fewer heads than Q (MQA/GQA)
 *     ("optimizing-attention-flash", Workflow 2, Steps 2 and 3).
 *
 * Readings taken where the pages are silent (each listed in the design
 * notes of the repository):
 *   - scale tau is passed explicitly (the caller maps "auto" to 1/sqrt(d));
 *   - mask alignment for Nq != Nk is bottom-right: query i sits at key
 *     position i + (Nk - Nq);
 *   - window bounds are inclusive: i' - left <= j <= i' + right;
 *   - causal together with a window intersects both constraints;
 *   - GQA maps query head h to kv head h / (Hq / Hkv) (consecutive groups);
 *   - LSE is the natural log of sum_j exp(S_ij) over visible keys;
 *   - a row with no visible key has O = 0, LSE = -inf, and zero gradients;
 *   - dropout (optional) multiplies P_ij by s M_ij before P V, where M_ij is
 *     a keep bit and s = 256 / T the rescale, and leaves LSE alone; M_ij is
 *     read from Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
 *     random numbers: as easy as 1, 2, 3", SC 2011) with key = the 64-bit seed
 *     and counter (j / 4, i / 4, b Hq + h, offset): the byte (j mod 4) of
 *     output word (i mod 4) keeps the element iff it is below T = round(256
 *     (1 - p)) ("optimizing-attention-flash", the dropout_p argument of
 *     flash_attn_func; "Что такое FlashAttention…", versions section: dropout
 *     among the features);
 *   - backward is the textbook gradient of the definition:
 *       dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij,
 *       dS = P o (dP - D), dQ = tau dS K, dK = tau dS^T Q
 *     with query heads of one group summed into their shared kv head.
 *
 * Layout: every tensor is dense row-major [batch, seq, heads, head_dim] in
 * fp64; LSE is [batch, q_heads, seq_q].  Work is split over rows (forward,
 * dQ) or key rows (dK, dV) with POSIX threads; each output element is
 * written by exactly one thread, with a fixed summation order, so results
 * are deterministic for any thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int B, Nq, Nk, Hq, Hkv, d;
    double tau;
    int causal, wl, wr;
    /* dropout: keep threshold T in [1, 255] (0 = no dropout), Philox key and
     * counter offset */
    int drop_T;
    uint64_t drop_seed;
    uint32_t drop_offset;
} shape_t;

/* Philox4x32-10 (SC 2011): ten rounds of two 32 x 32 -> 64-bit products
 * with multipliers 0xD2511F53 and 0xCD9E8D57; between rounds the key is
 * bumped by the Weyl constants 0x9E3779B9 and 0xBB67AE85. */
int oracle_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * x2;
        uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        uint32_t y1 = (uint32_t)p1;
        uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        uint32_t y3 = (uint32_t)p0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
    return 0;
}

/* Keep bit of element (i, j) of (batch, query head) bh: 1 or 0. */
int oracle_dropout_keep(uint64_t seed, uint32_t offset, long bh, long i, long j, int T) {
    uint32_t ctr[4] = {(uint32_t)(j / 4), (uint32_t)(i / 4), (uint32_t)bh, offset};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    uint32_t byte = (w[i % 4] >> (8 * (j % 4))) & 0xFFu;
    return byte < (uint32_t)T;
}

/* Multiplier of P_ij in P V: s M_ij with dropout, 1 without. */
static double drop_mult(const shape_t* s, int b, int h, long i, long j) {
    if (s->drop_T <= 0) return 1.0;
    long bh = (long)b * s->Hq + h;
    return oracle_dropout_keep(s->drop_seed, s->drop_offset, bh, i, j, s->drop_T)
               ? 256.0 / s->drop_T
               : 0.0;
}

/* Is key j visible to query i?  (mask definition, see header) */
static int key_visible(const shape_t* s, long i, long j) {
    long ip = i + (long)s->Nk - (long)s->Nq; /* bottom-right aligned position */
    if (s->causal && j > ip) return 0;
    if (s->wl >= 0 && j < ip - s->wl) return 0;
    if (s->wr >= 0 && j > ip + s->wr) return 0;
    return 1;
}

static const double* q_row(const double* q, const shape_t* s, int b, int i, int h) {
    return q + (((size_t)b * s->Nq + i) * s->Hq + h) * s->d;
}
static const double* kv_row(const double* k, const shape_t* s, int b, int j, int g) {
    return k + (((size_t)b * s->Nk + j) * s->Hkv + g) * s->d;
}

static double dot(const double* a, const double* b, int n) {
    double acc = 0.0;
    for (int c = 0; c < n; ++c) acc += a[c] * b[c];
    return acc;
}

/* Full score row S_i. = tau * q_i . k_j for every key j (masked ones too). */
static void score_row(const shape_t* s, const double* q, const double* k, int b, int h,
                      int i, double* srow) {
    int g = h / (s->Hq / s->Hkv);
    const double* qi = q_row(q, s, b, i, h);
    for (int j = 0; j < s->Nk; ++j) srow[j] = s->tau * dot(qi, kv_row(k, s, b, j, g), s->d);
}

/* LSE of the visible part of one score row: m + log sum exp(S - m). */
static double row_lse(const shape_t* s, long i, const double* srow) {
    double m = -INFINITY;
    for (long j = 0; j < s->Nk; ++j)
        if (key_visible(s, i, j) && srow[j] > m) m = srow[j];
    if (m == -INFINITY) return -INFINITY;
    double sum = 0.0;
    for (long j = 0; j < s->Nk; ++j)
        if (key_visible(s, i, j)) sum += exp(srow[j] - m);
    return m + log(sum);
}

/* P_i. = exp(S_ij - LSE_i) on visible keys, 0 elsewhere. */
static void prob_row(const shape_t* s, long i, const double* srow, double lse, double* prow) {
    for (long j = 0; j < s->Nk; ++j)
        prow[j] = (lse != -INFINITY && key_visible(s, i, j)) ? exp(srow[j] - lse) : 0.0;
}

/* ------------------------------------------------------------------ */
/* a tiny work-stealing pool over integer work items                    */
/* ------------------------------------------------------------------ */
typedef struct {
    void (*fn)(void* ctx, long item, double* scratch);
    void* ctx;
    long n_items;
    long next;
    size_t scratch_len;
    pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    double* scratch = (double*)malloc(sizeof(double) * (p->scratch_len ? p->scratch_len : 1));
    if (!scratch) return (void*)1;
    for (;;) {
        pthread_mutex_lock(&p->lock);
        long it = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (it >= p->n_items) break;
        p->fn(p->ctx, it, scratch);
    }
    free(scratch);
    return NULL;
}

static int run_pool(void (*fn)(void*, long, double*), void* ctx, long n_items,
                    size_t scratch_len, int nthreads) {
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > n_items) nthreads = (int)(n_items > 0 ? n_items : 1);
    pool_t p;
    p.fn = fn; p.ctx = ctx; p.n_items = n_items; p.next = 0; p.scratch_len = scratch_len;
    pthread_mutex_init(&p.lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -1;
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, pool_worker, &p) == 0) ++started;
    }
    if (started == 0) { pool_worker(&p); }
    for (int t = 0; t < started; ++t) {
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = -1;
    }
    free(th);
    pthread_mutex_destroy(&p.lock);
    return rc;
}

static int check_shape(const shape_t* s) {
    if (s->B < 1 || s->Nq < 1 || s->Nk < 1 || s->Hq < 1 || s->Hkv < 1 || s->d < 1) return -1;
    if (s->Hq % s->Hkv != 0) return -1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* forward                                                              */
/* ------------------------------------------------------------------ */
typedef struct {
    shape_t s;
    const double *q, *k, *v;
    double *o, *lse;
    const int64_t* rows; /* optional list of (b, h, i) triples */
} fwd_ctx;

static void fwd_one_row(const fwd_ctx* c, int b, int h, int i, double* out_o, double* out_lse,
                        double* scratch) {
    const shape_t* s = &c->s;
    int g = h / (s->Hq / s->Hkv);
    double* srow = scratch;
    double* prow = scratch + s->Nk;
    score_row(s, c->q, c->k, b, h, i, srow);
    double lse = row_lse(s, i, srow);
    prob_row(s, i, srow, lse, prow);
    for (int cc = 0; cc < s->d; ++cc) out_o[cc] = 0.0;
    for (int j = 0; j < s->Nk; ++j) {
        if (prow[j] == 0.0) continue;
        const double* vj = kv_row(c->v, s, b, j, g);
        double zij = prow[j] * drop_mult(s, b, h, i, j);
        for (int cc = 0; cc < s->d; ++cc) out_o[cc] += zij * vj[cc];
    }
    *out_lse = lse;
}

static void fwd_item(void* ctx, long item, double* scratch) {
    const fwd_ctx* c = (const fwd_ctx*)ctx;
    const shape_t* s = &c->s;
    int i = (int)(item % s->Nq);
    long bh = item / s->Nq;
    int h = (int)(bh % s->Hq);
    int b = (int)(bh / s->Hq);
    double* o = c->o + (((size_t)b * s->Nq + i) * s->Hq + h) * s->d;
    double* lse = c->lse + ((size_t)b * s->Hq + h) * s->Nq + i;
    fwd_one_row(c, b, h, i, o, lse, scratch);
}

int oracle_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
               int B, int Nq, int Nk, int Hq, int Hkv, int d, double tau, int causal,
               int window_left, int window_right, int nthreads) {
    fwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right},
                 q, k, v, o, lse, NULL};
    if (check_shape(&c.s)) return -1;
    return run_pool(fwd_item, &c, (long)B * Hq * Nq, 2 * (size_t)Nk, nthreads);
}

/* ------------------------------------------------------------------ */
/* forward over a paged KV cache                                        */
/* ------------------------------------------------------------------ */
/* The keys and values of sequence b are the first cache_seqlens[b] rows of
 * a cache made of fixed-size pages ("optimizing-attention-flash", the list of
 * advanced features, which names a paged KV cache; "FlashAttention V3
 * 原理与…实战指南", section 四 on inference, where the KV cache is kept in
 * pages and the vLLM example sets a page of 16 tokens): logical key j of
 * sequence b is row j % P of page block_table[b][j / P], and a page is laid
 * out [P, Hkv, d].  With the keys gathered that way the result is the
 * definition above, the mask aligned bottom-right against cache_seqlens[b]
 * (decode: the Nq new queries are the last Nq positions of the sequence). */
typedef struct {
    int B, Nq, Hq, Hkv, d, P, max_pages;
    double tau;
    int causal, wl, wr;
    const double *q, *kc, *vc;
    const int *block_table, *seqlens;
    double *o, *lse;
} paged_ctx;

/* Row of the cache holding logical key j of sequence b, kv head g. */
static const double* paged_key(const paged_ctx* c, const double* cache, int b, long j, int g) {
    long page = c->block_table[(size_t)b * c->max_pages + j / c->P];
    long row = j % c->P;
    return cache + (((size_t)page * c->P + row) * c->Hkv + g) * c->d;
}

static void paged_item(void* ctx, long item, double* scratch) {
    const paged_ctx* c = (const paged_ctx*)ctx;
    int i = (int)(item % c->Nq);
    long bh = item / c->Nq;
    int h = (int)(bh % c->Hq);
    int b = (int)(bh / c->Hq);
    int kv_head = h / (c->Hq / c->Hkv);
    int nk = c->seqlens[b];
    /* the sequence's own shape, for the shared mask and LSE definitions */
    shape_t s = {1, c->Nq, nk, c->Hq, c->Hkv, c->d, c->tau, c->causal, c->wl, c->wr};
    double* srow = scratch;
    double* prow = scratch + (nk > 0 ? nk : 1);
    const double* qi = c->q + (((size_t)b * c->Nq + i) * c->Hq + h) * c->d;
    for (long j = 0; j < nk; ++j)
        srow[j] = c->tau * dot(qi, paged_key(c, c->kc, b, j, kv_head), c->d);
    double l = row_lse(&s, i, srow);
    prob_row(&s, i, srow, l, prow);
    double* oi = c->o + (((size_t)b * c->Nq + i) * c->Hq + h) * c->d;
    for (int cc = 0; cc < c->d; ++cc) oi[cc] = 0.0;
    for (long j = 0; j < nk; ++j) {
        if (prow[j] == 0.0) continue;
        const double* vrow = paged_key(c, c->vc, b, j, kv_head);
        for (int cc = 0; cc < c->d; ++cc) oi[cc] += prow[j] * vrow[cc];
    }
    c->lse[((size_t)b * c->Hq + h) * c->Nq + i] = l;
}

int oracle_fwd_paged(const double* q, const double* k_cache, const double* v_cache,
                     const int* block_table, const int* cache_seqlens, double* o, double* lse,
                     int B, int Nq, int Hq, int Hkv, int d, int page_size, int num_pages,
                     int max_pages_per_seq, double tau, int causal, int window_left,
                     int window_right, int nthreads) {
    if (B < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv) return -1;
    if (page_size < 1 || num_pages < 1 || max_pages_per_seq < 1) return -1;
    long longest = 0;
    for (int b = 0; b < B; ++b) {
        long nk = cache_seqlens[b];
        if (nk < 0 || nk > (long)max_pages_per_seq * page_size) return -1;
        for (long pg = 0; pg * page_size < nk; ++pg) {
            int id = block_table[(size_t)b * max_pages_per_seq + pg];
            if (id < 0 || id >= num_pages) return -1;
        }
        if (nk > longest) longest = nk;
    }
    paged_ctx c = {B, Nq, Hq, Hkv, d, page_size, max_pages_per_seq, tau, causal,
                   window_left, window_right, q, k_cache, v_cache, block_table,
                   cache_seqlens, o, lse};
    return run_pool(paged_item, &c, (long)B * Hq * Nq, 2 * (size_t)(longest > 0 ? longest : 1),
                    nthreads);
}

static void fwd_rows_item(void* ctx, long item, double* scratch) {
    const fwd_ctx* c = (const fwd_ctx*)ctx;
    int b = (int)c->rows[3 * item], h = (int)c->rows[3 * item + 1], i = (int)c->rows[3 * item + 2];
    fwd_one_row(c, b, h, i, c->o + (size_t)item * c->s.d, c->lse + item, scratch);
}

/* Forward for a list of rows only: rows[3r..3r+2] = (b, h, i); o_rows is
 * [nrows, d], lse_rows is [nrows]. */
int oracle_fwd_rows(const double* q, const double* k, const double* v, const int64_t* rows,
                    long nrows, double* o_rows, double* lse_rows, int B, int Nq, int Nk, int Hq,
                    int Hkv, int d, double tau, int causal, int window_left, int window_right,
                    int nthreads) {
    fwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right},
                 q, k, v, o_rows, lse_rows, rows};
    if (check_shape(&c.s)) return -1;
    for (long r = 0; r < nrows; ++r) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= Hq ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Nq)
            return -1;
    }
    return run_pool(fwd_rows_item, &c, nrows, 2 * (size_t)Nk, nthreads);
}

/* The whole probability matrix P[Nq, Nk] of one (b, h). */
int oracle_probs(const double* q, const double* k, int b, int h, double* p, int B, int Nq, int Nk,
                 int Hq, int Hkv, int d, double tau, int causal, int window_left,
                 int window_right) {
    shape_t s = {B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right};
    if (check_shape(&s) || b < 0 || b >= B || h < 0 || h >= Hq) return -1;
    double* srow = (double*)malloc(sizeof(double) * Nk);
    if (!srow) return -1;
    for (int i = 0; i < Nq; ++i) {
        score_row(&s, q, k, b, h, i, srow);
        prob_row(&s, i, srow, row_lse(&s, i, srow), p + (size_t)i * Nk);
    }
    free(srow);
    return 0;
}

/* ------------------------------------------------------------------ */
/* backward                                                             */
/* ------------------------------------------------------------------ */
typedef struct {
    shape_t s;
    const double *q, *k, *v, *dout;
    double *dq, *dk, *dv;
    double *lse, *Dvec; /* per (b, h, i): filled by pass 1, read by pass 2 */
} bwd_ctx;

/* Pass 1, one query row: LSE_i, D_i = sum_j P_ij dP_ij, and
 * dQ_i = tau * sum_j dS_ij k_j. */
static void bwd_row_item(void* ctx, long item, double* scratch) {
    const bwd_ctx* c = (const bwd_ctx*)ctx;
    const shape_t* s = &c->s;
    int i = (int)(item % s->Nq);
    long bh = item / s->Nq;
    int h = (int)(bh % s->Hq);
    int b = (int)(bh / s->Hq);
    int g = h / (s->Hq / s->Hkv);
    double* srow = scratch;
    double* prow = scratch + s->Nk;
    double* dprow = scratch + 2 * (size_t)s->Nk;
    score_row(s, c->q, c->k, b, h, i, srow);
    double lse = row_lse(s, i, srow);
    prob_row(s, i, srow, lse, prow);
    const double* doi = c->dout + (((size_t)b * s->Nq + i) * s->Hq + h) * s->d;
    double Di = 0.0;
    for (int j = 0; j < s->Nk; ++j) {
        /* gradient w.r.t. P_ij: dO_i . V_j through the dropout multiplier */
        dprow[j] = dot(doi, kv_row(c->v, s, b, j, g), s->d) * drop_mult(s, b, h, i, j);
        Di += prow[j] * dprow[j];
    }
    double* dqi = c->dq + (((size_t)b * s->Nq + i) * s->Hq + h) * s->d;
    for (int cc = 0; cc < s->d; ++cc) dqi[cc] = 0.0;
    for (int j = 0; j < s->Nk; ++j) {
        if (prow[j] == 0.0) continue;
        double dS = prow[j] * (dprow[j] - Di);
        const double* kj = kv_row(c->k, s, b, j, g);
        for (int cc = 0; cc < s->d; ++cc) dqi[cc] += s->tau * dS * kj[cc];
    }
    size_t li = ((size_t)b * s->Hq + h) * s->Nq + i;
    c->lse[li] = lse;
    c->Dvec[li] = Di;
}

/* Pass 2, one key row j of kv head g: dK_j and dV_j summed over every query
 * head of the group and every query row. */
static void bwd_key_item(void* ctx, long item, double* scratch) {
    (void)scratch;
    const bwd_ctx* c = (const bwd_ctx*)ctx;
    const shape_t* s = &c->s;
    int j = (int)(item % s->Nk);
    long bg = item / s->Nk;
    int g = (int)(bg % s->Hkv);
    int b = (int)(bg / s->Hkv);
    int G = s->Hq / s->Hkv;
    const double* kj = kv_row(c->k, s, b, j, g);
    const double* vj = kv_row(c->v, s, b, j, g);
    double* dkj = c->dk + (((size_t)b * s->Nk + j) * s->Hkv + g) * s->d;
    double* dvj = c->dv + (((size_t)b * s->Nk + j) * s->Hkv + g) * s->d;
    for (int cc = 0; cc < s->d; ++cc) { dkj[cc] = 0.0; dvj[cc] = 0.0; }
    for (int h = g * G; h < (g + 1) * G; ++h) {
        for (int i = 0; i < s->Nq; ++i) {
            size_t li = ((size_t)b * s->Hq + h) * s->Nq + i;
            double lse = c->lse[li];
            if (lse == -INFINITY || !key_visible(s, i, j)) continue;
            const double* qi = q_row(c->q, s, b, i, h);
            const double* doi = c->dout + (((size_t)b * s->Nq + i) * s->Hq + h) * s->d;
            double Sij = s->tau * dot(qi, kj, s->d);
            double Pij = exp(Sij - lse);
            double mult = drop_mult(s, b, h, i, j);
            double Zij = Pij * mult; /* the weight of V_j in O_i */
            double dPij = dot(doi, vj, s->d) * mult;
            double dSij = Pij * (dPij - c->Dvec[li]);
            for (int cc = 0; cc < s->d; ++cc) {
                dkj[cc] += s->tau * dSij * qi[cc];
                dvj[cc] += Zij * doi[cc];
            }
        }
    }
}

/* Gradients of L = sum(dout o O) w.r.t. q, k, v.  lse_out and D_out
 * ([B, Hq, Nq], may be NULL) receive the oracle's own LSE and D. */
int oracle_bwd(const double* q, const double* k, const double* v, const double* dout, double* dq,
               double* dk, double* dv, double* lse_out, double* D_out, int B, int Nq, int Nk,
               int Hq, int Hkv, int d, double tau, int causal, int window_left, int window_right,
               int nthreads) {
    bwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right},
                 q, k, v, dout, dq, dk, dv, NULL, NULL};
    if (check_shape(&c.s)) return -1;
    size_t nrow = (size_t)B * Hq * Nq;
    c.lse = lse_out ? lse_out : (double*)malloc(sizeof(double) * nrow);
    c.Dvec = D_out ? D_out : (double*)malloc(sizeof(double) * nrow);
    int rc = -1;
    if (c.lse && c.Dvec) {
        rc = run_pool(bwd_row_item, &c, (long)nrow, 3 * (size_t)Nk, nthreads);
        if (rc == 0) rc = run_pool(bwd_key_item, &c, (long)B * Hkv * Nk, 1, nthreads);
    }
    if (!lse_out) free(c.lse);
    if (!D_out) free(c.Dvec);
    return rc;
}

/* The forward and backward with dropout at keep threshold T (1..255). */
/* Selected rows of the forward with dropout (rows as in oracle_fwd_rows):
 * the same per-row definition, for checking long sequences one row at a time. */
int oracle_fwd_rows_dropout(const double* q, const double* k, const double* v,
                            const int64_t* rows, long nrows, double* o_rows, double* lse_rows,
                            int B, int Nq, int Nk, int Hq, int Hkv, int d, double tau, int causal,
                            int window_left, int window_right, int T, uint64_t seed,
                            uint32_t offset, int nthreads) {
    if (T < 1 || T > 255) return -1;
    fwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right, T, seed, offset},
                 q, k, v, o_rows, lse_rows, rows};
    if (check_shape(&c.s)) return -1;
    for (long r = 0; r < nrows; ++r) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= Hq ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Nq)
            return -1;
    }
    return run_pool(fwd_rows_item, &c, nrows, 2 * (size_t)Nk, nthreads);
}

int oracle_fwd_dropout(const double* q, const double* k, const double* v, double* o, double* lse,
                       int B, int Nq, int Nk, int Hq, int Hkv, int d, double tau, int causal,
                       int window_left, int window_right, int T, uint64_t seed, uint32_t offset,
                       int nthreads) {
    if (T < 1 || T > 255) return -1;
    fwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right, T, seed, offset},
                 q, k, v, o, lse, NULL};
    if (check_shape(&c.s)) return -1;
    return run_pool(fwd_item, &c, (long)B * Hq * Nq, 2 * (size_t)Nk, nthreads);
}

int oracle_bwd_dropout(const double* q, const double* k, const double* v, const double* dout,
                       double* dq, double* dk, double* dv, double* lse_out, double* D_out, int B,
                       int Nq, int Nk, int Hq, int Hkv, int d, double tau, int causal,
                       int window_left, int window_right, int T, uint64_t seed, uint32_t offset,
                       int nthreads) {
    if (T < 1 || T > 255) return -1;
    bwd_ctx c = {{B, Nq, Nk, Hq, Hkv, d, tau, causal, window_left, window_right, T, seed, offset},
                 q, k, v, dout, dq, dk, dv, NULL, NULL};
    if (check_shape(&c.s)) return -1;
    size_t nrow = (size_t)B * Hq * Nq;
    c.lse = lse_out ? lse_out : (double*)malloc(sizeof(double) * nrow);
    c.Dvec = D_out ? D_out : (double*)malloc(sizeof(double) * nrow);
    int rc = -1;
    if (c.lse && c.Dvec) {
        rc = run_pool(bwd_row_item, &c, (long)nrow, 3 * (size_t)Nk, nthreads);
        if (rc == 0) rc = run_pool(bwd_key_item, &c, (long)B * Hkv * Nk, 1, nthreads);
    }
    if (!lse_out) free(c.lse);
    if (!D_out) free(c.Dvec);
    return rc;
}

/* Number of threads a call with nthreads <= 0 would use. */
int oracle_default_threads(void) {
    long nc = sysconf(_SC_NPROCESSORS_ONLN);
    return nc > 0 ? (int)nc : 1;
}
