/*
 * sa_oracle.c -- plain, slow, fp64 CPU reference for head-aware sparse
 * attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; it reads the same input
 * layouts and nothing else.
 *
 * Every floating-point quantity is computed in fp64 from the exact stored
 * input values (bf16 cache entries and bf16/fp32 queries widened to double).
 * Loops follow the definitions literally: no blocking, no online softmax, no
 * radix tricks.  Work is spread over plain pthreads by independent output
 * (one (sequence, head) or one query row per task); that changes no
 * arithmetic.
 *
 * Sources (titles of the pages the method is read from):
 *  [Kascade] "Kascade稀疏注意力：让长上下文大模型更快落地物流供应链"
 *            sections "核心机制：Anchor + Reuse", "头部感知（head-aware）是精度关键".
 *  [DA-1]    "语言模型能自己决定该看哪里吗？" section on the DA state machine and
 *            block-aligned masks in vLLM.
 *  [RBS]     "RBS-Attention: Radius-Bounded Sparse Prefill ..." blog, section
 *            "关键技术点" items 1 (双分支选择机制) and 2 (独立阈值 + mask 合并).
 *  [DA-2]    "百万上下文，模型终于会挑重点了", section "三种模式，背后是三种推理状态".
 *  [LoZA]    "稀疏注意力机制创新：美团新技术如何提升大模型的效率与成本控制？"
 *            sections "二、ZigZag架构" (1024-token streaming window) and
 *            "四、从外卖到AI" (SplitKV-and-Combine).
 *
 * Parity pins: every function below is pinned by the CPU tests in
 * tests/test_oracle_*.py against closed forms, brute force or library routines.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* input layouts                                                             */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *k;          /* bf16 bits [num_pages][Hkv][P][d] */
    const uint16_t *v;          /* bf16 bits [num_pages][Hkv][P][d] */
    const int32_t *page_table;  /* [B][max_pages] */
    const int32_t *seq_lens;    /* [B] */
    int32_t batch, num_kv_heads, head_dim, page_size, max_pages, num_pages;
} or_cache;

static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Row of token t (logical position in sequence b) of kv head g. */
static const uint16_t *cache_row(const or_cache *c, const uint16_t *base, int b, int g, long t)
{
    long logical_page = t / c->page_size;
    long page = c->page_table[(long)b * c->max_pages + logical_page];
    long slot = t % c->page_size;
    return base + ((page * c->num_kv_heads + g) * c->page_size + slot) * c->head_dim;
}

static void widen_row(const uint16_t *src, int d, double *dst)
{
    for (int i = 0; i < d; ++i) dst[i] = widen_bf16(src[i]);
}

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += a[i] * b[i];
    return s;
}

/* ------------------------------------------------------------------------ */
/* a trivial dynamic parallel-for                                            */
/* ------------------------------------------------------------------------ */
typedef void (*task_fn)(void *ctx, long i);
typedef struct { task_fn fn; void *ctx; long n; long next; } pool_t;

static void *pool_worker(void *arg)
{
    pool_t *p = (pool_t *)arg;
    for (;;) {
        long i = __atomic_fetch_add(&p->next, 1, __ATOMIC_RELAXED);
        if (i >= p->n) break;
        p->fn(p->ctx, i);
    }
    return NULL;
}

int or_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void parallel_for(long n, int nthreads, task_fn fn, void *ctx)
{
    if (nthreads <= 0) nthreads = or_default_threads();
    if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    pool_t p = {fn, ctx, n, 0};
    if (nthreads <= 1) { pool_worker(&p); return; }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pool_worker, &p);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
}

/* ------------------------------------------------------------------------ */
/* 1. masked softmax attention over an explicit token set                   */
/*    [Kascade] "只对这 k 个位置做注意力计算"; [DA-1] block-aligned masks;     */
/*    [RBS] block-sparse FlashAttention path.  Definition:                   */
/*      s_t = scale * q.k_t ; m = max s_t ; w_t = exp(s_t - m)               */
/*      out = sum w_t v_t / sum w_t ; lse = m + ln sum w_t                   */
/*    Two passes (max, then sums).  Empty set: out = 0, lse = -inf.          */
/* ------------------------------------------------------------------------ */
static void attend_tokens(const or_cache *c, int b, int g, const double *q, double scale,
                          const int64_t *tok, long n, double *out, double *lse,
                          double *m_out, double *l_out, double *acc_out)
{
    int d = c->head_dim;
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (n <= 0) {
        if (lse) *lse = -INFINITY;
        if (m_out) *m_out = -INFINITY;
        if (l_out) *l_out = 0.0;
        if (acc_out) for (int i = 0; i < d; ++i) acc_out[i] = 0.0;
        return;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double *row = (double *)malloc(sizeof(double) * (size_t)d);
    double *acc = (double *)calloc((size_t)d, sizeof(double));
    double m = -INFINITY;
    for (long i = 0; i < n; ++i) {
        widen_row(cache_row(c, c->k, b, g, tok[i]), d, row);
        s[i] = scale * dot(q, row, d);
        if (s[i] > m) m = s[i];
    }
    double l = 0.0;
    for (long i = 0; i < n; ++i) {
        double w = exp(s[i] - m);
        l += w;
        widen_row(cache_row(c, c->v, b, g, tok[i]), d, row);
        for (int j = 0; j < d; ++j) acc[j] += w * row[j];
    }
    for (int j = 0; j < d; ++j) out[j] = acc[j] / l;
    if (lse) *lse = m + log(l);
    if (m_out) *m_out = m;
    if (l_out) *l_out = l;
    if (acc_out) for (int j = 0; j < d; ++j) acc_out[j] = acc[j];
    free(s); free(row); free(acc);
}

/* ------------------------------------------------------------------------ */
/* 2. anchor-layer exact top-k, per query head                               */
/*    [Kascade] "核心机制": exact Top-k key indices on anchor layers;         */
/*    "头部感知": selection per head.  r_t = q_h . k_{g(h),t} for t < L_b;   */
/*    keep the min(k, L_b) largest, ordered by (r desc, t asc) with a full  */
/*    sort; output ascending by position, padded with -1.                    */
/* ------------------------------------------------------------------------ */
typedef struct { double r; int64_t t; } scored_t;

static int cmp_score_desc(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->r > y->r) return -1;
    if (x->r < y->r) return 1;
    return (x->t > y->t) - (x->t < y->t);
}

static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

typedef struct {
    const or_cache *c; const double *q; int Hq; int k;
    int32_t *idx; int32_t *count; double *scores; long score_stride;
} topk_ctx;

static void topk_task(void *vctx, long bh)
{
    topk_ctx *x = (topk_ctx *)vctx;
    const or_cache *c = x->c;
    int d = c->head_dim;
    int b = (int)(bh / x->Hq), h = (int)(bh % x->Hq);
    int g = h / (x->Hq / c->num_kv_heads);
    long L = c->seq_lens[b];
    const double *q = x->q + ((long)b * x->Hq + h) * d;
    double *row = (double *)malloc(sizeof(double) * (size_t)d);
    scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)(L > 0 ? L : 1));
    for (long t = 0; t < L; ++t) {
        widen_row(cache_row(c, c->k, b, g, t), d, row);
        sc[t].r = dot(q, row, d);
        sc[t].t = t;
        if (x->scores) x->scores[bh * x->score_stride + t] = sc[t].r;
    }
    if (x->idx) {
        long m = L < x->k ? L : x->k;
        qsort(sc, (size_t)L, sizeof(scored_t), cmp_score_desc);
        int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(m > 0 ? m : 1));
        for (long i = 0; i < m; ++i) pos[i] = sc[i].t;
        qsort(pos, (size_t)m, sizeof(int64_t), cmp_i64);
        int32_t *out = x->idx + bh * (long)x->k;
        for (long i = 0; i < x->k; ++i) out[i] = i < m ? (int32_t)pos[i] : -1;
        x->count[bh] = (int32_t)m;
        free(pos);
    }
    free(row); free(sc);
}

/* raw anchor scores r[b][h][t] (t < L_b; rest untouched) */
void or_topk_scores(const or_cache *c, const double *q, int Hq, double *scores, long score_stride,
                    int nthreads)
{
    topk_ctx x = {c, q, Hq, 0, NULL, NULL, scores, score_stride};
    parallel_for((long)c->batch * Hq, nthreads, topk_task, &x);
}

void or_select_topk(const or_cache *c, const double *q, int Hq, int k, int32_t *idx, int32_t *count,
                    int nthreads)
{
    topk_ctx x = {c, q, Hq, k, idx, count, NULL, 0};
    parallel_for((long)c->batch * Hq, nthreads, topk_task, &x);
}

/* ------------------------------------------------------------------------ */
/* 3. decode attention over a per-head token-index set (anchor and reuse     */
/*    layers use the same idx; [Kascade] "复用这个 Top-k 索引")             */
/* ------------------------------------------------------------------------ */
typedef struct {
    const or_cache *c; const double *q; int Hq; const int32_t *idx; int kcap;
    const int32_t *count; const uint8_t *member; long member_stride;
    double scale; double *out; double *lse; const int64_t *rows; int num_splits;
    double *part_m, *part_l, *part_acc;
} dec_ctx;

static void decode_task(void *vctx, long r)
{
    dec_ctx *x = (dec_ctx *)vctx;
    const or_cache *c = x->c;
    int d = c->head_dim;
    long bh = x->rows ? x->rows[r] : r;
    int b = (int)(bh / x->Hq), h = (int)(bh % x->Hq);
    int g = h / (x->Hq / c->num_kv_heads);
    const double *q = x->q + bh * d;
    long n = 0;
    int64_t *tok;
    if (x->member) {
        long L = c->seq_lens[b];
        tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
        for (long t = 0; t < L; ++t)
            if (x->member[(long)b * x->member_stride + t]) tok[n++] = t;
    } else {
        n = x->count[bh];
        tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        for (long i = 0; i < n; ++i) tok[i] = x->idx[bh * (long)x->kcap + i];
    }
    attend_tokens(c, b, g, q, x->scale, tok, n, x->out + r * d, x->lse ? x->lse + r : NULL,
                  NULL, NULL, NULL);
    if (x->num_splits > 0) {
        /* split s covers list positions [s*chunk, min((s+1)*chunk, n)), chunk = ceil(n/S) */
        int S = x->num_splits;
        long chunk = (n + S - 1) / S;
        double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
        for (int s = 0; s < S; ++s) {
            long lo = s * chunk, hi = lo + chunk;
            if (lo > n) lo = n;
            if (hi > n) hi = n;
            long o = r * S + s;
            attend_tokens(c, b, g, q, x->scale, tok + lo, hi - lo, tmp, NULL,
                          x->part_m + o, x->part_l + o, x->part_acc + o * d);
        }
        free(tmp);
    }
    free(tok);
}

/* out[r][d], lse[r] for rows r (all B*Hq rows if rows == NULL, else n_rows listed (b*Hq+h)) */
void or_decode_tokens(const or_cache *c, const double *q, int Hq, const int32_t *idx, int kcap,
                      const int32_t *count, double scale, double *out, double *lse,
                      const int64_t *rows, long n_rows, int nthreads)
{
    dec_ctx x = {c, q, Hq, idx, kcap, count, NULL, 0, scale, out, lse, rows, 0, NULL, NULL, NULL};
    parallel_for(rows ? n_rows : (long)c->batch * Hq, nthreads, decode_task, &x);
}

/* the same attention with per-split partial states (m_s, l_s, unnormalised acc_s) */
void or_decode_tokens_split(const or_cache *c, const double *q, int Hq, const int32_t *idx, int kcap,
                            const int32_t *count, double scale, int num_splits, double *out,
                            double *lse, double *part_m, double *part_l, double *part_acc,
                            int nthreads)
{
    dec_ctx x = {c, q, Hq, idx, kcap, count, NULL, 0, scale, out, lse, NULL, num_splits,
                 part_m, part_l, part_acc};
    parallel_for((long)c->batch * Hq, nthreads, decode_task, &x);
}

/* decode attention over a per-sequence token membership mask (shared by all heads) */
void or_decode_members(const or_cache *c, const double *q, int Hq, const uint8_t *member,
                       long member_stride, double scale, double *out, double *lse,
                       const int64_t *rows, long n_rows, int nthreads)
{
    dec_ctx x = {c, q, Hq, NULL, 0, NULL, member, member_stride, scale, out, lse, rows, 0,
                 NULL, NULL, NULL};
    parallel_for(rows ? n_rows : (long)c->batch * Hq, nthreads, decode_task, &x);
}

/* ------------------------------------------------------------------------ */
/* 4. SplitKV-and-Combine ([LoZA] "四、从外卖到AI"): merge S partial states  */
/*    m = max m_s over non-empty parts; l = sum l_s e^{m_s-m};               */
/*    out = sum e^{m_s-m} acc_s / l ; lse = m + ln l.  Empty parts skipped.  */
/* ------------------------------------------------------------------------ */
void or_combine(int S, int d, const double *m_s, const double *l_s, const double *acc_s,
                double *out, double *lse)
{
    double m = -INFINITY;
    for (int s = 0; s < S; ++s)
        if (l_s[s] > 0.0 && m_s[s] > m) m = m_s[s];
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }
    double l = 0.0;
    for (int s = 0; s < S; ++s) {
        if (!(l_s[s] > 0.0)) continue;
        double w = exp(m_s[s] - m);
        l += l_s[s] * w;
        for (int j = 0; j < d; ++j) out[j] += w * acc_s[(long)s * d + j];
    }
    for (int j = 0; j < d; ++j) out[j] /= l;
    *lse = m + log(l);
}

/* ------------------------------------------------------------------------ */
/* 5. RBS block statistics ([RBS] "关键技术点" 1):                            */
/*    block j = tokens [j*bs, min((j+1)*bs, L)), n_j of them;                 */
/*    c_j = (1/n_j) sum k_t ; r_j = max_t ||k_t - c_j||_2                     */
/* ------------------------------------------------------------------------ */
typedef struct { const or_cache *c; int b; int bs; int nB; double *cen; double *rad; } bstat_ctx;

static void bstat_task(void *vctx, long gj)
{
    bstat_ctx *x = (bstat_ctx *)vctx;
    const or_cache *c = x->c;
    int d = c->head_dim;
    int g = (int)(gj / x->nB), j = (int)(gj % x->nB);
    long L = c->seq_lens[x->b];
    long lo = (long)j * x->bs, hi = lo + x->bs;
    if (hi > L) hi = L;
    double *cen = x->cen + gj * d;
    double *row = (double *)malloc(sizeof(double) * (size_t)d);
    for (int i = 0; i < d; ++i) cen[i] = 0.0;
    long n = hi - lo;
    for (long t = lo; t < hi; ++t) {
        widen_row(cache_row(c, c->k, x->b, g, t), d, row);
        for (int i = 0; i < d; ++i) cen[i] += row[i];
    }
    for (int i = 0; i < d; ++i) cen[i] /= (double)n;
    double r = 0.0;
    for (long t = lo; t < hi; ++t) {
        widen_row(cache_row(c, c->k, x->b, g, t), d, row);
        double e = 0.0;
        for (int i = 0; i < d; ++i) e += (row[i] - cen[i]) * (row[i] - cen[i]);
        e = sqrt(e);
        if (e > r) r = e;
    }
    x->rad[gj] = r;
    free(row);
}

void or_block_stats(const or_cache *c, int b, int bs, double *centroid, double *radius, int nthreads)
{
    long L = c->seq_lens[b];
    int nB = (int)((L + bs - 1) / bs);
    bstat_ctx x = {c, b, bs, nB, centroid, radius};
    parallel_for((long)c->num_kv_heads * nB, nthreads, bstat_task, &x);
}

/* ------------------------------------------------------------------------ */
/* 6. query pooling: qbar_i = mean of the queries of block i (bs rows, fewer */
/*    in a partial last block); qnorm_i = ||qbar_i||_2                        */
/* ------------------------------------------------------------------------ */
void or_pool_q(const uint16_t *q, long T, int Hq, int d, int bs, double *qbar, double *qnorm)
{
    long nB = (T + bs - 1) / bs;
    for (int h = 0; h < Hq; ++h)
        for (long i = 0; i < nB; ++i) {
            double *qb = qbar + ((long)h * nB + i) * d;
            long lo = i * bs, hi = lo + bs;
            if (hi > T) hi = T;
            for (int e = 0; e < d; ++e) qb[e] = 0.0;
            for (long t = lo; t < hi; ++t)
                for (int e = 0; e < d; ++e) qb[e] += widen_bf16(q[(t * Hq + h) * d + e]);
            double nrm = 0.0;
            for (int e = 0; e < d; ++e) { qb[e] /= (double)(hi - lo); nrm += qb[e] * qb[e]; }
            qnorm[(long)h * nB + i] = sqrt(nrm);
        }
}

/* ------------------------------------------------------------------------ */
/* 7. two-branch block-pair scores ([RBS] "关键技术点" 1) over causal pairs  */
/*    j <= i, pair index i(i+1)/2 + j:                                      */
/*      S_c = scale * qbar_i.c_j  ;  S_r = scale * (qbar_i.c_j + ||qbar_i|| r_j) */
/*    head h reads kv head g(h) = h / (Hq/Hkv)'s statistics.                 */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *qbar, *qnorm, *cen, *rad; int Hq, Hkv, nB, d; double scale; double *Sc, *Sr;
} pair_ctx;

static void pair_task(void *vctx, long hi_)
{
    pair_ctx *x = (pair_ctx *)vctx;
    int h = (int)(hi_ / x->nB), i = (int)(hi_ % x->nB);
    int g = h / (x->Hq / x->Hkv);
    long nP = (long)x->nB * (x->nB + 1) / 2;
    const double *qb = x->qbar + ((long)h * x->nB + i) * x->d;
    double qn = x->qnorm[(long)h * x->nB + i];
    for (int j = 0; j <= i; ++j) {
        const double *cj = x->cen + ((long)g * x->nB + j) * x->d;
        double qc = dot(qb, cj, x->d);
        long p = (long)h * nP + (long)i * (i + 1) / 2 + j;
        x->Sc[p] = x->scale * qc;
        x->Sr[p] = x->scale * (qc + qn * x->rad[(long)g * x->nB + j]);
    }
}

void or_pair_scores(const double *qbar, const double *qnorm, const double *centroid,
                    const double *radius, int Hq, int Hkv, int nB, int d, double scale,
                    double *Sc, double *Sr, int nthreads)
{
    pair_ctx x = {qbar, qnorm, centroid, radius, Hq, Hkv, nB, d, scale, Sc, Sr};
    parallel_for((long)Hq * nB, nthreads, pair_task, &x);
}

/* ------------------------------------------------------------------------ */
/* 8. thresholds and mask ([RBS] "关键技术点" 2: independent thresholds,     */
/*    masks OR'd).  Quantile: sorted_asc(x)[floor(p*(n-1))].                */
/*    keep = score > tau (strict);  M = keep_c | keep_r | [j=i] | [j=0].      */
/* ------------------------------------------------------------------------ */
static int cmp_f64(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

double or_quantile(const double *x, long n, double p)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    memcpy(s, x, sizeof(double) * (size_t)n);
    qsort(s, (size_t)n, sizeof(double), cmp_f64);
    long r = (long)floor(p * (double)(n - 1));
    double v = s[r];
    free(s);
    return v;
}

/* sorted copy (ascending), used by the tests to place thresholds in gaps */
void or_sort(double *x, long n) { qsort(x, (size_t)n, sizeof(double), cmp_f64); }

void or_rbs_mask(const double *Sc, const double *Sr, int Hq, int nB, const double *tau_c,
                 const double *tau_r, int force_diag, int force_first, uint8_t *mask)
{
    long nP = (long)nB * (nB + 1) / 2;
    for (int h = 0; h < Hq; ++h)
        for (int i = 0; i < nB; ++i)
            for (int j = 0; j <= i; ++j) {
                long p = (long)h * nP + (long)i * (i + 1) / 2 + j;
                int keep = (Sc[p] > tau_c[h]) || (Sr[p] > tau_r[h]) ||
                           (force_diag && j == i) || (force_first && j == 0);
                mask[p] = (uint8_t)keep;
            }
}

/* ------------------------------------------------------------------------ */
/* 9. block-sparse causal prefill: row t of head h (query block i = t/bs)    */
/*    attends to the tokens t' <= t whose block t'/bs is selected in row i. */
/* ------------------------------------------------------------------------ */
typedef struct {
    const or_cache *c; int b; const uint16_t *q; int Hq; int bs; int nB; const uint8_t *mask;
    double scale; const int64_t *rows; double *out; double *lse;
} pre_ctx;

static void prefill_task(void *vctx, long r)
{
    pre_ctx *x = (pre_ctx *)vctx;
    const or_cache *c = x->c;
    int d = c->head_dim;
    long th = x->rows ? x->rows[r] : r;
    long t = th / x->Hq;
    int h = (int)(th % x->Hq);
    int g = h / (x->Hq / c->num_kv_heads);
    long i = t / x->bs;
    long nP = (long)x->nB * (x->nB + 1) / 2;
    double *q = (double *)malloc(sizeof(double) * (size_t)d);
    for (int e = 0; e < d; ++e) q[e] = widen_bf16(x->q[(t * x->Hq + h) * d + e]);
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(t + 1));
    long n = 0;
    for (long u = 0; u <= t; ++u) {
        long j = u / x->bs;
        if (x->mask[(long)h * nP + i * (i + 1) / 2 + j]) tok[n++] = u;
    }
    attend_tokens(c, x->b, g, q, x->scale, tok, n, x->out + r * d, x->lse + r, NULL, NULL, NULL);
    free(q); free(tok);
}

/* rows: list of (t*Hq + h); NULL = every row of [T][Hq] */
void or_prefill(const or_cache *c, int b, const uint16_t *q, int Hq, int bs, const uint8_t *mask,
                double scale, const int64_t *rows, long n_rows, double *out, double *lse,
                int nthreads)
{
    long T = c->seq_lens[b];
    int nB = (int)((T + bs - 1) / bs);
    pre_ctx x = {c, b, q, Hq, bs, nB, mask, scale, rows, out, lse};
    parallel_for(rows ? n_rows : T * Hq, nthreads, prefill_task, &x);
}

/* ------------------------------------------------------------------------ */
/* 10. span membership ([DA-1] block-aligned masks: keep-ranges rounded OUT */
/*     to KV-block edges; [LoZA] streaming window, token-exact):            */
/*     span [a,b) -> [floor(a/P)P, ceil(b/P)P) if rounded, then & [0, L).    */
/* ------------------------------------------------------------------------ */
static long floor_div(long a, long b) { long q = a / b; if ((a % b) && ((a < 0) != (b < 0))) --q; return q; }

void or_span_members(long L, int P, int n_spans, const int64_t *spans, const uint8_t *round_out,
                     uint8_t *member)
{
    for (long t = 0; t < L; ++t) member[t] = 0;
    for (int s = 0; s < n_spans; ++s) {
        long a = spans[2 * s], b = spans[2 * s + 1];
        if (round_out[s]) {
            a = floor_div(a, P) * P;
            b = -floor_div(-b, P) * P;
        }
        if (a < 0) a = 0;
        if (b > L) b = L;
        for (long t = a; t < b; ++t) member[t] = 1;
    }
}
