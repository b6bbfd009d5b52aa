/*
 * CPU oracle for MiniMax Sparse Attention (MSA) training hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Every function computes the plain definition, one output row (or one KV
 * block) at a time, in double precision, from the bf16 inputs widened to
 * float.  Where a choice is the oracle's own reading of the pages it is
 * marked READING.
 *
 * Sources (three news pages about Flash-MSA):
 *   [p1] "Flash-MSA: Open-Source Sparse Attention Kernels Debut",
 *        section "How MSA works": KVs are selected in blocks of 128 by
 *        max-pooling proxy scores; the block indices are cached; the main
 *        attention is GQA; each proxy head (one per group) selects its own
 *        subset of KVs.  Section "Verification and limitations": checked in
 *        bf16 by cosine similarity, tolerance 0.01.
 *   [p2] "flash-msa-sparse-attention-training" news post, paragraphs 1-4:
 *        an Index Branch picks the KV blocks each query reads, a Main Branch
 *        runs exact softmax attention over only those blocks; training needs
 *        custom backward kernels; groups of heads keep their own proxy head.
 *
 * Layouts (row-major, last index fastest):
 *   qp, kp   [B][T][Hp][dp]    proxy queries / keys, Hp = Hkv (one per group)
 *   q        [B][T][Hq][d]     main-branch queries
 *   k, v     [B][T][Hkv][d]    main-branch keys / values
 *   idx      [B][Hp][T][topk]  selected block ids, ascending, -1 padded
 *   nsel     [B][Hp][T]        number of valid entries in an idx row
 *   o, dout  [B][T][Hq][d]
 *   lse, D   [B][Hq][T]
 *
 * Query i lives in block bi = i / blk.  It may read block n only if n <= bi,
 * and inside its own block only keys j <= i (causal).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, Hq, Hkv, d, dp, blk, topk;
    double scale;
    int window, dilation;   /* forced block pattern; 1, 1: only the own block */
} odims;

static int nblocks(const odims* m) { return (m->T + m->blk - 1) / m->blk; }

/* ------------------------------------------------------------------ */
/* a tiny pthread parallel-for over independent items                  */
/* ------------------------------------------------------------------ */
typedef void (*item_fn)(void* ctx, int64_t item);
typedef struct {
    item_fn fn;
    void* ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
} pfor_state;

static void* pfor_worker(void* arg)
{
    pfor_state* st = (pfor_state*)arg;
    for (;;) {
        pthread_mutex_lock(&st->mu);
        int64_t it = st->next++;
        pthread_mutex_unlock(&st->mu);
        if (it >= st->n) break;
        st->fn(st->ctx, it);
    }
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, item_fn fn, void* ctx)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pfor_state st;
    st.fn = fn; st.ctx = ctx; st.n = n; st.next = 0;
    pthread_mutex_init(&st.mu, NULL);
    pthread_t th[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[started], NULL, pfor_worker, &st) == 0) ++started;
    pfor_worker(&st);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&st.mu);
}

/* ------------------------------------------------------------------ */
/* Index Branch: proxy score, causal block max-pool, selection          */
/* ------------------------------------------------------------------ */

/* pooled[n] for one query row (b, g, i), n = 0..nblk-1.
 * Proxy score s(i, j) = sum_c qp[b,i,g,c] * kp[b,j,g,c]   (READING: a raw dot
 * product, no scale) for causal keys j <= i; pooled[n] = max over the keys of
 * block n that the query may see; -inf for blocks after the query's own.
 * The maximum is taken in double and rounded once to float: the selection is
 * decided on float scores, the precision the GPU kernel decides in. */
static void pool_row(const odims* m, const float* qp, const float* kp,
                     int b, int g, int i, float* pooled)
{
    const int Hp = m->Hkv, dp = m->dp, blk = m->blk, nb = nblocks(m);
    const float* qrow = qp + (((int64_t)b * m->T + i) * Hp + g) * dp;
    for (int n = 0; n < nb; ++n) {
        int j0 = n * blk;
        if (j0 > i) { pooled[n] = -INFINITY; continue; }
        int j1 = j0 + blk - 1;
        if (j1 > i) j1 = i;
        double best = -INFINITY;
        for (int j = j0; j <= j1; ++j) {
            const float* krow = kp + (((int64_t)b * m->T + j) * Hp + g) * dp;
            double s = 0.0;
            for (int c = 0; c < dp; ++c) s += (double)qrow[c] * (double)krow[c];
            if (s > best) best = s;
        }
        pooled[n] = (float)best;
    }
}

typedef struct { float s; int n; } cand;

/* Order used to rank candidate blocks: higher pooled score first; equal
 * scores (including -0 == +0) go to the lower block index. */
static int cand_cmp(const void* pa, const void* pb)
{
    const cand* a = (const cand*)pa;
    const cand* b = (const cand*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->n > b->n) - (a->n < b->n);
}

static int int_cmp(const void* pa, const void* pb)
{
    int a = *(const int*)pa, b = *(const int*)pb;
    return (a > b) - (a < b);
}

/* Forced blocks of a query in block bi under a window of `window` blocks with
 * dilation `dilation` (page "Flash-MSA: Train on a million tokens without
 * breaking the compute bank", section "Under the hood": the block pattern is
 * configurable by window size and dilation; our reading): bi, bi - dilation,
 * ..., bi - (window-1) dilation, those that are >= 0.  window = 1 forces only
 * the own block.  Returns 1 if block n is forced. */
static int is_forced(int n, int bi, int window, int dilation)
{
    const int back = bi - n;
    return back >= 0 && back % dilation == 0 && back / dilation < window;
}

/* Selection for one row: the forced blocks (the query's own block bi, plus the
 * window) are always kept; the remaining slots of the topk go to the best of
 * the other blocks 0..bi in the order above.  If the query has at most topk
 * eligible blocks it takes all of them.  Output is ascending and padded with
 * -1; returns the count. */
static int select_row(const float* pooled, int bi, int topk, int window, int dilation, int32_t* out,
                      cand* scratch)
{
    int cnt = 0;
    int* sel = (int*)out;
    if (bi + 1 <= topk) {
        for (int n = 0; n <= bi; ++n) sel[cnt++] = n;
    } else {
        int nc = 0;
        for (int n = 0; n <= bi; ++n) {
            if (is_forced(n, bi, window, dilation)) {
                sel[cnt++] = n;
            } else {
                scratch[nc].s = pooled[n];
                scratch[nc].n = n;
                ++nc;
            }
        }
        qsort(scratch, (size_t)nc, sizeof(cand), cand_cmp);
        for (int r = 0; cnt < topk && r < nc; ++r) sel[cnt++] = scratch[r].n;
        qsort(sel, (size_t)cnt, sizeof(int), int_cmp);
    }
    for (int r = cnt; r < topk; ++r) out[r] = -1;
    return cnt;
}

typedef struct {
    const odims* m;
    const float *qp, *kp;
    const int64_t* rows;   /* flattened (b*Hp + g)*T + i */
    float* pooled_out;     /* [nrows][nblk] or NULL */
    int32_t *idx, *nsel;   /* full-size [B][Hp][T][topk], [B][Hp][T] */
} sel_ctx;

static void sel_item(void* vctx, int64_t r)
{
    sel_ctx* c = (sel_ctx*)vctx;
    const odims* m = c->m;
    const int nb = nblocks(m), T = m->T;
    int64_t row = c->rows[r];
    int i = (int)(row % T);
    int64_t bg = row / T;
    int g = (int)(bg % m->Hkv), b = (int)(bg / m->Hkv);
    float* pooled = (float*)malloc(sizeof(float) * (size_t)nb);
    cand* scratch = (cand*)malloc(sizeof(cand) * (size_t)nb);
    pool_row(m, c->qp, c->kp, b, g, i, pooled);
    if (c->pooled_out) memcpy(c->pooled_out + r * nb, pooled, sizeof(float) * (size_t)nb);
    int32_t* out = c->idx + row * m->topk;
    c->nsel[row] = select_row(pooled, i / m->blk, m->topk, m->window, m->dilation, out, scratch);
    free(pooled);
    free(scratch);
}

/* Proxy score -> pool -> select for the listed rows. */
int msa_oracle_select(const odims* m, const float* qp, const float* kp,
                      int64_t nrows, const int64_t* rows,
                      float* pooled_out, int32_t* idx, int32_t* nsel, int nthreads)
{
    sel_ctx c = {m, qp, kp, rows, pooled_out, idx, nsel};
    parallel_for(nrows, nthreads, sel_item, &c);
    return 0;
}

/* Selection alone, from given pooled rows [nrows][nblk] with the query's
 * block index per row (used to check a selection rule on fixed scores). */
int msa_oracle_select_from_pooled(int64_t nrows, int nblk, int topk, int window, int dilation,
                                  const float* pooled, const int32_t* bi,
                                  int32_t* idx, int32_t* nsel)
{
    cand* scratch = (cand*)malloc(sizeof(cand) * (size_t)(nblk > 0 ? nblk : 1));
    for (int64_t r = 0; r < nrows; ++r)
        nsel[r] = select_row(pooled + r * nblk, bi[r], topk, window, dilation, idx + r * topk, scratch);
    free(scratch);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Main Branch forward: exact softmax attention over the selected keys  */
/* ------------------------------------------------------------------ */

/* The keys query (b, g, i) reads: every key of each selected block, limited
 * to j <= i (only the own block is cut by this).  Returns the count. */
static int gather_keys(const odims* m, const int32_t* idx, const int32_t* nsel,
                       int b, int g, int i, int* keys)
{
    int64_t row = ((int64_t)b * m->Hkv + g) * m->T + i;
    const int32_t* sel = idx + row * m->topk;
    int ns = nsel[row], cnt = 0;
    for (int r = 0; r < ns; ++r) {
        int n = sel[r];
        for (int j = n * m->blk; j < (n + 1) * m->blk && j < m->T; ++j)
            if (j <= i) keys[cnt++] = j;
    }
    return cnt;
}

/* scores s_j = scale * q_i . k_j for the row's keys; returns the maximum */
static double row_scores(const odims* m, const float* q, const float* k,
                         int b, int h, int i, const int* keys, int nk, double* s)
{
    const int G = m->Hq / m->Hkv, g = h / G, d = m->d;
    const float* qrow = q + (((int64_t)b * m->T + i) * m->Hq + h) * d;
    double mx = -INFINITY;
    for (int t = 0; t < nk; ++t) {
        const float* krow = k + (((int64_t)b * m->T + keys[t]) * m->Hkv + g) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += (double)qrow[c] * (double)krow[c];
        s[t] = m->scale * acc;
        if (s[t] > mx) mx = s[t];
    }
    return mx;
}

typedef struct {
    const odims* m;
    const float *q, *k, *v;
    const int32_t *idx, *nsel;
    const int64_t* rows;     /* flattened (b*Hq + h)*T + i */
    double *o, *lse;         /* full-size outputs; only listed rows written */
} fwd_ctx;

static void fwd_item(void* vctx, int64_t r)
{
    fwd_ctx* c = (fwd_ctx*)vctx;
    const odims* m = c->m;
    const int T = m->T, d = m->d, G = m->Hq / m->Hkv;
    int64_t row = c->rows[r];
    int i = (int)(row % T);
    int64_t bh = row / T;
    int h = (int)(bh % m->Hq), b = (int)(bh / m->Hq), g = h / G;
    int* keys = (int*)malloc(sizeof(int) * (size_t)(m->topk * m->blk + 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(m->topk * m->blk + 1));
    int nk = gather_keys(m, c->idx, c->nsel, b, g, i, keys);
    double* orow = c->o + (((int64_t)b * T + i) * m->Hq + h) * d;
    for (int e = 0; e < d; ++e) orow[e] = 0.0;
    double mx = row_scores(m, c->q, c->k, b, h, i, keys, nk, s);
    double l = 0.0;
    for (int t = 0; t < nk; ++t) l += exp(s[t] - mx);
    double L = mx + log(l);                       /* logsumexp of the row */
    for (int t = 0; t < nk; ++t) {
        double p = exp(s[t] - L);                 /* softmax probability */
        const float* vrow = c->v + (((int64_t)b * T + keys[t]) * m->Hkv + g) * d;
        for (int e = 0; e < d; ++e) orow[e] += p * (double)vrow[e];
    }
    c->lse[((int64_t)b * m->Hq + h) * T + i] = L;
    free(keys);
    free(s);
}

int msa_oracle_fwd(const odims* m, const float* q, const float* k, const float* v,
                   const int32_t* idx, const int32_t* nsel,
                   int64_t nrows, const int64_t* rows, double* o, double* lse, int nthreads)
{
    fwd_ctx c = {m, q, k, v, idx, nsel, rows, o, lse};
    parallel_for(nrows, nthreads, fwd_item, &c);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Main Branch backward                                                */
/* ------------------------------------------------------------------ */
/* For loss terms <dO, O>:  P_ij = exp(s_ij - L_i),  dP_ij = dO_i . v_j,
 * D_i = dO_i . O_i,  dS_ij = P_ij (dP_ij - D_i),
 * dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
 * dV_j = sum_i P_ij dO_i, where dK/dV sum over every head of the group.
 * No gradient reaches the proxy inputs: the selection is piecewise constant. */

typedef struct {
    const odims* m;
    const float *q, *k, *v, *dout;
    const double *o, *lse;
    const int32_t *idx, *nsel;
    const int64_t* rows;     /* flattened (b*Hq + h)*T + i */
    double *dq, *D;
} dq_ctx;

static void dq_item(void* vctx, int64_t r)
{
    dq_ctx* c = (dq_ctx*)vctx;
    const odims* m = c->m;
    const int T = m->T, d = m->d, G = m->Hq / m->Hkv;
    int64_t row = c->rows[r];
    int i = (int)(row % T);
    int64_t bh = row / T;
    int h = (int)(bh % m->Hq), b = (int)(bh / m->Hq), g = h / G;
    int* keys = (int*)malloc(sizeof(int) * (size_t)(m->topk * m->blk + 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(m->topk * m->blk + 1));
    int nk = gather_keys(m, c->idx, c->nsel, b, g, i, keys);
    row_scores(m, c->q, c->k, b, h, i, keys, nk, s);
    const int64_t qoff = (((int64_t)b * T + i) * m->Hq + h) * d;
    const float* dorow = c->dout + qoff;
    const double* orow = c->o + qoff;
    double Di = 0.0;
    for (int e = 0; e < d; ++e) Di += (double)dorow[e] * orow[e];
    double L = c->lse[((int64_t)b * m->Hq + h) * T + i];
    double* dqrow = c->dq + qoff;
    for (int e = 0; e < d; ++e) dqrow[e] = 0.0;
    for (int t = 0; t < nk; ++t) {
        const int64_t koff = (((int64_t)b * T + keys[t]) * m->Hkv + g) * d;
        double p = exp(s[t] - L);
        double dp = 0.0;
        for (int e = 0; e < d; ++e) dp += (double)dorow[e] * (double)c->v[koff + e];
        double ds = p * (dp - Di);
        for (int e = 0; e < d; ++e) dqrow[e] += m->scale * ds * (double)c->k[koff + e];
    }
    c->D[((int64_t)b * m->Hq + h) * T + i] = Di;
    free(keys);
    free(s);
}

/* dQ and D for the listed rows; needs the oracle's own O and L for them. */
int msa_oracle_bwd_dq(const odims* m, const float* q, const float* k, const float* v,
                      const float* dout, const double* o, const double* lse,
                      const int32_t* idx, const int32_t* nsel,
                      int64_t nrows, const int64_t* rows, double* dq, double* D, int nthreads)
{
    dq_ctx c = {m, q, k, v, dout, o, lse, idx, nsel, rows, dq, D};
    parallel_for(nrows, nthreads, dq_item, &c);
    return 0;
}

typedef struct {
    const odims* m;
    const float *q, *k, *v, *dout;
    const double *lse, *D;
    const int32_t *idx, *nsel;
    const int64_t* blocks;   /* flattened (b*Hkv + g)*nblk + n */
    double *dk, *dv;         /* full-size [B][T][Hkv][d]; only listed blocks written */
} kv_ctx;

static void kv_item(void* vctx, int64_t r)
{
    kv_ctx* c = (kv_ctx*)vctx;
    const odims* m = c->m;
    const int T = m->T, d = m->d, G = m->Hq / m->Hkv, nb = nblocks(m), blk = m->blk;
    int64_t bl = c->blocks[r];
    int n = (int)(bl % nb);
    int64_t bg = bl / nb;
    int g = (int)(bg % m->Hkv), b = (int)(bg / m->Hkv);
    int j0 = n * blk, j1 = (n + 1) * blk;
    if (j1 > T) j1 = T;
    for (int j = j0; j < j1; ++j)
        for (int e = 0; e < d; ++e) {
            c->dk[(((int64_t)b * T + j) * m->Hkv + g) * d + e] = 0.0;
            c->dv[(((int64_t)b * T + j) * m->Hkv + g) * d + e] = 0.0;
        }
    /* every query of the group whose selection holds block n */
    for (int i = j0; i < T; ++i) {
        int64_t srow = ((int64_t)b * m->Hkv + g) * T + i;
        const int32_t* sel = c->idx + srow * m->topk;
        int hit = 0;
        for (int t = 0; t < c->nsel[srow]; ++t) if (sel[t] == n) hit = 1;
        if (!hit) continue;
        for (int hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            const int64_t qoff = (((int64_t)b * T + i) * m->Hq + h) * d;
            const float* qrow = c->q + qoff;
            const float* dorow = c->dout + qoff;
            double L = c->lse[((int64_t)b * m->Hq + h) * T + i];
            double Di = c->D[((int64_t)b * m->Hq + h) * T + i];
            for (int j = j0; j < j1 && j <= i; ++j) {
                const int64_t koff = (((int64_t)b * T + j) * m->Hkv + g) * d;
                double sc = 0.0, dp = 0.0;
                for (int e = 0; e < d; ++e) {
                    sc += (double)qrow[e] * (double)c->k[koff + e];
                    dp += (double)dorow[e] * (double)c->v[koff + e];
                }
                double p = exp(m->scale * sc - L);
                double ds = p * (dp - Di);
                for (int e = 0; e < d; ++e) {
                    c->dv[koff + e] += p * (double)dorow[e];
                    c->dk[koff + e] += m->scale * ds * (double)qrow[e];
                }
            }
        }
    }
}

/* dK, dV for the listed KV blocks; needs L and D of every query that
 * selected the block (from msa_oracle_fwd / msa_oracle_bwd_dq). */
int msa_oracle_bwd_dkdv(const odims* m, const float* q, const float* k, const float* v,
                        const float* dout, const double* lse, const double* D,
                        const int32_t* idx, const int32_t* nsel,
                        int64_t nblk_list, const int64_t* blocks, double* dk, double* dv,
                        int nthreads)
{
    kv_ctx c = {m, q, k, v, dout, lse, D, idx, nsel, blocks, dk, dv};
    parallel_for(nblk_list, nthreads, kv_item, &c);
    return 0;
}

typedef struct {
    const odims* m;
    const float *q, *k, *v, *dout;
    const double *lse, *D;
    const int32_t *idx, *nsel;
    const int64_t* rows;     /* flattened (b*Hq + h)*T + i */
    double *dk, *dv;         /* per-row contributions, [nrows][blk*topk][d] */
} kvr_ctx;

static void kvr_item(void* vctx, int64_t r)
{
    kvr_ctx* c = (kvr_ctx*)vctx;
    const odims* m = c->m;
    const int T = m->T, d = m->d, G = m->Hq / m->Hkv;
    int64_t row = c->rows[r];
    int i = (int)(row % T);
    int64_t bh = row / T;
    int h = (int)(bh % m->Hq), b = (int)(bh / m->Hq), g = h / G;
    int* keys = (int*)malloc(sizeof(int) * (size_t)(m->topk * m->blk + 1));
    int nk = gather_keys(m, c->idx, c->nsel, b, g, i, keys);
    const int64_t qoff = (((int64_t)b * T + i) * m->Hq + h) * d;
    const double L = c->lse[((int64_t)b * m->Hq + h) * T + i];
    const double Di = c->D[((int64_t)b * m->Hq + h) * T + i];
    double* dkr = c->dk + r * (int64_t)m->topk * m->blk * d;
    double* dvr = c->dv + r * (int64_t)m->topk * m->blk * d;
    for (int t = 0; t < nk; ++t) {
        const int64_t koff = (((int64_t)b * T + keys[t]) * m->Hkv + g) * d;
        double sc = 0.0, dp = 0.0;
        for (int e = 0; e < d; ++e) {
            sc += (double)c->q[qoff + e] * (double)c->k[koff + e];
            dp += (double)c->dout[qoff + e] * (double)c->v[koff + e];
        }
        double p = exp(m->scale * sc - L);
        double ds = p * (dp - Di);
        for (int e = 0; e < d; ++e) {
            dvr[(int64_t)t * d + e] = p * (double)c->dout[qoff + e];
            dkr[(int64_t)t * d + e] = m->scale * ds * (double)c->q[qoff + e];
        }
    }
    for (int t = nk; t < m->topk * m->blk; ++t)
        for (int e = 0; e < d; ++e) { dvr[(int64_t)t * d + e] = 0.0; dkr[(int64_t)t * d + e] = 0.0; }
    free(keys);
}

/* What one query row (b, h, i) adds to dK and dV of each key it reads, in
 * the order of the row's keys (selected blocks ascending, keys ascending).
 * Output [nrows][topk*blk][d]; needs the row's L and D. */
int msa_oracle_bwd_kv_rows(const odims* m, const float* q, const float* k, const float* v,
                           const float* dout, const double* lse, const double* D,
                           const int32_t* idx, const int32_t* nsel,
                           int64_t nrows, const int64_t* rows, double* dk_rows, double* dv_rows,
                           int nthreads)
{
    kvr_ctx c = {m, q, k, v, dout, lse, D, idx, nsel, rows, dk_rows, dv_rows};
    parallel_for(nrows, nthreads, kvr_item, &c);
    return 0;
}
