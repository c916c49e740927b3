/*
 * sa_oracle.c -- CPU fp64 oracle for fine-grained top-K sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow restatement of what
 * the method computes, written from the pages' definitions.  Only the tests,
 * __graft_entry__.smoke() and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA library
 * (fine_grained_top_b200/csrc): the two meet only on the seeded inputs.
 *
 * Every value is a double; bf16 inputs are widened exactly by the Python
 * wrapper before they arrive here.  Rows are independent, so the heavy loops
 * are split over POSIX threads by row; nothing else is reordered.
 *
 * Sources (page title, section):
 *  - indexer: "Sparse Attention for Long-Context LLM Inference" (Baidu),
 *    section "Where Sparse Attention Is Actually Sparse" (lightweight indexer
 *    scores history, outputs candidate indices, no positional encoding);
 *    "Sparse Attention in 2026" (Acing AI), "The designs that shipped"
 *    (lightning indexer: few heads, low precision, top-k 2048);
 *    "Sparse Attention" (completesystemdesign.dev), DSA list ("ReLU + top-k").
 *    Score: I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s]); no 1/sqrt(D), no
 *    softmax, one key head shared by all indexer heads.
 *  - top-K: Baidu long-context page, same section (Top-K caps the candidate
 *    count).  Ties go to the lower position; output ascending; -1 padding.
 *  - window: "Sparse Attention" (completesystemdesign.dev) mask diagrams
 *    ("always the local window"); Window(t) = {max(0,t-W+1) .. t}.
 *  - coarse pass: "Why fine-grained sparse attention ..." (mg6.net),
 *    "What Fine-Grained Means" (coarse block pass, then fine top-K inside the
 *    candidates) and section 2 "Learned Block Routing" (blocks mean-pooled
 *    over complete blocks, dot product, top-k).
 *  - FP8 indexer operands: "Sparse Attention in 2026", "The designs that
 *    shipped" (the lightning indexer is a small FP8 network).  The pages name
 *    no FP8 layout; this file takes e4m3 as the OCP 8-bit float format defines
 *    it (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at
 *    exponent field 0, no infinities, exponent 15 with mantissa 7 is NaN),
 *    with round-to-nearest-even and saturation of finite overflow to +-448.
 *  - attention: "A Guide to Sparse Attention in Large Models" (Baidu),
 *    section 2: Attention = softmax(QK^T/sqrt(d)) V and its masked form
 *    softmax(QK^T * Mask + (1-Mask)(-inf)) V with Mask[i,j] = 1 iff j in S(i).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* row-parallel driver                                                 */
/* ------------------------------------------------------------------ */
typedef void (*row_fn)(void *ctx, int64_t r);
typedef struct { row_fn fn; void *ctx; int64_t first, R, stride; } span_t;

/* thread i takes rows i, i+n, i+2n, ... so that causal rows, whose cost grows
 * with the position, spread evenly over the threads */
static void *run_span(void *p) {
    span_t *s = (span_t *)p;
    for (int64_t r = s->first; r < s->R; r += s->stride) s->fn(s->ctx, r);
    return NULL;
}

static void for_rows(int64_t R, int nthreads, row_fn fn, void *ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (R < nthreads) nthreads = (int)(R > 0 ? R : 1);
    if (nthreads == 1) {
        span_t one = {fn, ctx, 0, R, 1};
        run_span(&one);
        return;
    }
    pthread_t th[256];
    span_t sp[256];
    for (int i = 0; i < nthreads; ++i) {
        sp[i].fn = fn; sp[i].ctx = ctx;
        sp[i].first = i; sp[i].R = R; sp[i].stride = nthreads;
        pthread_create(&th[i], NULL, run_span, &sp[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------ */
/* indexer score of one (query row, key row) pair                      */
/* ------------------------------------------------------------------ */
static double index_score(int H, int D, const double *qI_row /*[H,D]*/,
                          const double *w_row /*[H]*/, const double *key /*[D]*/) {
    double total = 0.0;
    for (int j = 0; j < H; ++j) {
        double dot = 0.0;
        for (int c = 0; c < D; ++c) dot += qI_row[j * D + c] * key[c];
        double relu = dot > 0.0 ? dot : 0.0;
        total += w_row[j] * relu;
    }
    return total;
}

/* I[r, s] for 0 <= s < S.  Column s is scored iff s <= lim[r]; every other
 * column is -inf (causal: lim[r] = position of query r). */
typedef struct {
    int S, H, D; const double *qI, *w, *kI; const int64_t *lim; double *out;
} idx_ctx;

static void indexer_row(void *p, int64_t r) {
    idx_ctx *c = (idx_ctx *)p;
    const double *q = c->qI + r * (int64_t)c->H * c->D;
    const double *w = c->w + r * (int64_t)c->H;
    double *o = c->out + r * (int64_t)c->S;
    for (int64_t s = 0; s < c->S; ++s)
        o[s] = (s <= c->lim[r]) ? index_score(c->H, c->D, q, w, c->kI + s * c->D)
                                : -INFINITY;
}

void oracle_indexer(int64_t R, int S, int H, int D, const double *qI,
                    const double *w, const double *kI, const int64_t *lim,
                    double *out, int nthreads) {
    idx_ctx c = {S, H, D, qI, w, kI, lim, out};
    for_rows(R, nthreads, indexer_row, &c);
}

/* ------------------------------------------------------------------ */
/* e4m3 (OCP FP8) values and codes                                     */
/* ------------------------------------------------------------------ */
/* The value of a code: (-1)^s * (1 + M/8) * 2^(E-7) for E > 0, and
 * (-1)^s * (M/8) * 2^-6 for E = 0; E = 15, M = 7 is NaN. */
static double e4m3_value(uint8_t c) {
    const int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
    if (E == 15 && M == 7) return NAN;
    const double v = (E == 0) ? ldexp((double)M, -9) : ldexp((double)(8 + M), E - 10);
    return s ? -v : v;
}

/* The nearest code (ties to the even mantissa).  Within the binade
 * [2^e, 2^(e+1)), e >= -6, the representable values are spaced 2^(e-3);
 * below 2^-6 the subnormals keep the spacing 2^-9.  Counting the value in
 * units of that spacing and rounding gives the code directly: a subnormal's
 * code is its unit count, a normal's is (e+7)*8 + (units - 8), and a round-up
 * to the next binade lands on that binade's first code. */
static uint8_t e4m3_code(double x) {
    if (isnan(x)) return signbit(x) ? 0xFF : 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;          /* largest finite value */
    int e = -6;
    if (a >= ldexp(1.0, -6)) {
        int ex;
        frexp(a, &ex);                           /* a = m 2^ex, m in [0.5, 1) */
        e = ex - 1;
    }
    const double units = rint(ldexp(a, 3 - e));  /* exact scaling; rint: ties to even */
    const int code = (e + 7) * 8 + (int)units - 8;
    return sign | (uint8_t)code;
}

void oracle_e4m3_encode(int64_t n, const double *x, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(x[i]);
}

void oracle_e4m3_decode(int64_t n, const uint8_t *c, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(c[i]);
}

/* ------------------------------------------------------------------ */
/* top-K among candidate positions                                     */
/* ------------------------------------------------------------------ */
typedef struct { double score; int64_t pos; } cand_t;

/* order: higher score first; equal scores -> lower position first */
static int by_score_then_pos(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int by_pos(const void *a, const void *b) {
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x < y) ? -1 : (x > y);
}

/* Keep the min(K, n) best of n candidates, emit their positions ascending,
 * pad with -1 up to K.  `work` has room for n candidates. */
static void topk_of(int64_t n, cand_t *work, int K, int64_t *out) {
    qsort(work, (size_t)n, sizeof(cand_t), by_score_then_pos);
    int64_t m = n < K ? n : K;
    for (int64_t i = 0; i < m; ++i) out[i] = work[i].pos;
    qsort(out, (size_t)m, sizeof(int64_t), by_pos);
    for (int64_t i = m; i < K; ++i) out[i] = -1;
}

/* Row r holds scores[r, 0 .. n_valid[r]-1]; its candidate positions are the
 * column indices, or cand[r, col] when cand is given. */
typedef struct {
    int64_t L; const double *scores; const int64_t *n_valid; const int64_t *cand;
    int K; int64_t *out;
} topk_ctx;

static void topk_row(void *p, int64_t r) {
    topk_ctx *c = (topk_ctx *)p;
    int64_t n = c->n_valid[r];
    cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        work[i].score = c->scores[r * c->L + i];
        work[i].pos = c->cand ? c->cand[r * c->L + i] : i;
    }
    topk_of(n, work, c->K, c->out + r * (int64_t)c->K);
    free(work);
}

void oracle_topk(int64_t R, int64_t L, const double *scores,
                 const int64_t *n_valid, const int64_t *cand, int K,
                 int64_t *out, int nthreads) {
    topk_ctx c = {L, scores, n_valid, cand, K, out};
    for_rows(R, nthreads, topk_row, &c);
}

/* ------------------------------------------------------------------ */
/* coarse pass: mean-pooled complete blocks                            */
/* ------------------------------------------------------------------ */
/* kB[b, c] = mean over the blk rows of block b (only complete blocks; a
 * partial tail block is dropped, as the block router truncates). */
void oracle_pool_mean(int64_t S, int D, int blk, const double *kI, double *kB) {
    int64_t nb = S / blk;
    for (int64_t b = 0; b < nb; ++b)
        for (int c = 0; c < D; ++c) {
            double sum = 0.0;
            for (int i = 0; i < blk; ++i) sum += kI[(b * blk + i) * D + c];
            kB[b * D + c] = sum / blk;
        }
}

/* Two-stage selection for query rows at positions t_pos[r]:
 *   1. blocks eligible for t: complete blocks entirely before t's own block,
 *      b < floor(t / blk);
 *   2. coarse score of block b = indexer score against the pooled key kB[b];
 *      keep the min(keep, #eligible) best (ties -> lower block);
 *   3. candidates = tokens of the kept blocks, plus t's own block up to t;
 *   4. fine score = indexer score against kI[s]; keep the top K candidates
 *      (ties -> lower position), ascending, -1 padded.
 * blocks_out[r, :] receives the kept blocks ascending, -1 padded. */
typedef struct {
    const int64_t *t_pos; int H, D; const double *qI, *w, *kI, *kB;
    int blk, keep, K; int64_t *topk_out, *blocks_out;
} two_ctx;

static void two_stage_row(void *p, int64_t r) {
    two_ctx *c = (two_ctx *)p;
    int64_t t = c->t_pos[r];
    const double *q = c->qI + r * (int64_t)c->H * c->D;
    const double *w = c->w + r * (int64_t)c->H;
    int64_t own = t / c->blk;            /* t's own block */
    int64_t n_elig = own;                /* blocks 0 .. own-1 */
    cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_elig + 1));
    for (int64_t b = 0; b < n_elig; ++b) {
        work[b].score = index_score(c->H, c->D, q, w, c->kB + b * c->D);
        work[b].pos = b;
    }
    int64_t *blocks = c->blocks_out + r * (int64_t)c->keep;
    topk_of(n_elig, work, c->keep, blocks);
    free(work);
    int64_t n_kept = n_elig < c->keep ? n_elig : c->keep;

    int64_t n_cand = n_kept * c->blk + (t - own * c->blk + 1);
    cand_t *cw = (cand_t *)malloc(sizeof(cand_t) * (size_t)n_cand);
    int64_t n = 0;
    for (int64_t i = 0; i < n_kept; ++i)
        for (int j = 0; j < c->blk; ++j) {
            int64_t s = blocks[i] * c->blk + j;
            cw[n].score = index_score(c->H, c->D, q, w, c->kI + s * c->D);
            cw[n++].pos = s;
        }
    for (int64_t s = own * c->blk; s <= t; ++s) {
        cw[n].score = index_score(c->H, c->D, q, w, c->kI + s * c->D);
        cw[n++].pos = s;
    }
    topk_of(n, cw, c->K, c->topk_out + r * (int64_t)c->K);
    free(cw);
}

void oracle_two_stage(int64_t R, const int64_t *t_pos, int H, int D,
                      const double *qI, const double *w, int64_t S,
                      const double *kI, int blk, int keep, int K,
                      int64_t *topk_out, int64_t *blocks_out, int nthreads) {
    double *kB = (double *)malloc(sizeof(double) * (size_t)((S / blk) * D + 1));
    oracle_pool_mean(S, D, blk, kI, kB);
    two_ctx c = {t_pos, H, D, qI, w, kI, kB, blk, keep, K, topk_out, blocks_out};
    for_rows(R, nthreads, two_stage_row, &c);
    free(kB);
}

/* ------------------------------------------------------------------ */
/* selection set and exact attention over it                           */
/* ------------------------------------------------------------------ */
/* S(t) = TopK(t) U {max(0, t-W+1) .. t} as a sorted set without repeats.
 * Returns |S(t)|; `out` has room for K + W entries. */
int64_t oracle_selection(int K, const int64_t *topk_row, int W, int64_t t,
                         int64_t *out) {
    int64_t n = 0;
    for (int i = 0; i < K; ++i)
        if (topk_row[i] >= 0) out[n++] = topk_row[i];
    int64_t w0 = t - W + 1 > 0 ? t - W + 1 : 0;
    for (int64_t s = w0; s <= t; ++s) out[n++] = s;
    qsort(out, (size_t)n, sizeof(int64_t), by_pos);
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (m == 0 || out[i] != out[m - 1]) out[m++] = out[i];
    return m;
}

/* O[r, h, :] = sum_{s in S_r} softmax_s(q[r,h] . k[s] * scale) v[s]
 * with S_r = sel_idx[sel_ptr[r] .. sel_ptr[r+1]).  lse[r, h] is the natural
 * log of the softmax denominator, sum_s exp(q[r,h].k[s]*scale). */
typedef struct {
    int Hq, d; const double *q, *k, *v; const int64_t *sel_ptr, *sel_idx;
    double scale; double *out, *lse;
} attn_ctx;

static void attn_row(void *p, int64_t r) {
    attn_ctx *c = (attn_ctx *)p;
    int64_t b = c->sel_ptr[r], n = c->sel_ptr[r + 1] - b;
    const int64_t *S = c->sel_idx + b;
    double *logit = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int h = 0; h < c->Hq; ++h) {
        const double *qh = c->q + (r * c->Hq + h) * (int64_t)c->d;
        double mx = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            double dot = 0.0;
            for (int e = 0; e < c->d; ++e) dot += qh[e] * c->k[S[i] * c->d + e];
            logit[i] = dot * c->scale;
            if (logit[i] > mx) mx = logit[i];
        }
        double denom = 0.0;
        for (int64_t i = 0; i < n; ++i) { logit[i] = exp(logit[i] - mx); denom += logit[i]; }
        double *oh = c->out + (r * c->Hq + h) * (int64_t)c->d;
        for (int e = 0; e < c->d; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < n; ++i) acc += (logit[i] / denom) * c->v[S[i] * c->d + e];
            oh[e] = acc;
        }
        if (c->lse) c->lse[r * c->Hq + h] = mx + log(denom);
    }
    free(logit);
}

void oracle_sparse_attention(int64_t R, int Hq, int d, const double *q,
                             const double *k, const double *v,
                             const int64_t *sel_ptr, const int64_t *sel_idx,
                             double scale, double *out, double *lse,
                             int nthreads) {
    attn_ctx c = {Hq, d, q, k, v, sel_ptr, sel_idx, scale, out, lse};
    for_rows(R, nthreads, attn_row, &c);
}
