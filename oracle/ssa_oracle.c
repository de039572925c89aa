/*
 * ssa_oracle.c -- plain fp64 CPU oracle for the SSA sparse stream.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg call this code.  It shares no code, header or constant
 * with the CUDA library; it includes only the C standard library and pthreads.
 *
 * What it computes, and where the pages define it:
 *
 *  - Block summaries: the mean of the keys of each contiguous 64-token block
 *    ("SSA: Guida a Sparse Sparse Attention per LLM", section "Block-sparse
 *    attention e Receptive Field": the sequence is cut into contiguous blocks
 *    and each query sees a mean representation of the earlier blocks).  The
 *    query side is the mean over the 64 tokens of a query block and over the
 *    G query heads sharing one KV head (GQA-shared support, the reading the
 *    DashAttention page's Stage 1 gives for heads sharing a KV head).
 *
 *  - Selection: per query block i, the diagonal block i plus the k-1 earlier
 *    blocks of highest score qbar_i . kbar_j (same section: keep only the
 *    top-k most relevant blocks); ties go to the lower block index; when
 *    i + 1 <= k every causal block is taken.  The receptive field is then
 *    64 * k tokens (256 or 1024 on the Italian page).
 *
 *  - Attention: exact softmax attention of each query token over the tokens
 *    of its selected blocks with the causal mask s <= t (same section: the
 *    attention is computed only on the tokens inside the selected blocks),
 *    and the dense causal counterpart ("Resumen Tecnico: SSA", section 2,
 *    "Alineacion Bidireccional": the opposite-mode output computed for the
 *    alignment only).
 *
 *  - Dropped mass: delta(t) = the full-softmax weight on the causal tokens that
 *    the sparse stream did not select ("Resumen Tecnico: SSA", section 1:
 *    the attention weight assigned to the tokens the sparse mechanism did not
 *    select).  Also returned by a second route, 1 - exp(LSE_sparse - LSE_full).
 *
 *  - Sparse backward: the gradient of the sparse output with respect to
 *    q, k, v; keys outside the selected blocks receive exactly zero
 *    ("Resumen Tecnico: SSA", section 1, second gap: discarded tokens receive
 *    zero gradient).  No gradient flows into pooling or selection.
 *
 * All arithmetic is fp64.  Inputs are fp64 arrays (the bf16 tensors widened
 * exactly by the Python wrapper).  Work is split over threads by independent
 * output items only; there is no blocking, fusion or reordering of any sum.
 *
 * Layouts (row-major, contiguous):
 *   q, dO        [B][S][Hq][D]
 *   k, v         [B][S][Hkv][D]
 *   kbar, qbar   [B][Hkv][n][D]          n = S / bs
 *   idx          [B][Hkv][n][topk]       ascending, -1 padded
 *   gap          [B][Hkv][n]             NAN where there is no k-th/(k+1)-th boundary
 * Row lists are int64 triples (b, hq, t); block lists are triples (b, kvh, j).
 * Return value: 0 on success, -1 on invalid arguments or allocation failure.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ threads */

typedef void (*ora_item_fn)(void *ctx, int64_t item, double *scratch);

typedef struct {
    ora_item_fn fn;
    void *ctx;
    int64_t n_items;
    int tid, nthreads;
    size_t scratch_len;
    int failed;
} ora_worker;

static void *ora_worker_main(void *arg) {
    ora_worker *w = (ora_worker *)arg;
    double *scratch = NULL;
    if (w->scratch_len) {
        scratch = (double *)malloc(w->scratch_len * sizeof(double));
        if (!scratch) { w->failed = 1; return NULL; }
    }
    for (int64_t it = w->tid; it < w->n_items; it += w->nthreads) w->fn(w->ctx, it, scratch);
    free(scratch);
    return NULL;
}

/* Runs fn(ctx, item, scratch) for item in [0, n_items) on nthreads threads.
 * Each thread owns a private scratch buffer of scratch_len doubles. */
static int ora_parallel_for(ora_item_fn fn, void *ctx, int64_t n_items, int nthreads,
                            size_t scratch_len) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    ora_worker w[256];
    pthread_t th[256];
    int started[256];
    int failed = 0;
    for (int i = 0; i < nthreads; ++i) {
        w[i].fn = fn; w[i].ctx = ctx; w[i].n_items = n_items;
        w[i].tid = i; w[i].nthreads = nthreads; w[i].scratch_len = scratch_len; w[i].failed = 0;
        started[i] = (nthreads > 1) && (pthread_create(&th[i], NULL, ora_worker_main, &w[i]) == 0);
        if (!started[i]) ora_worker_main(&w[i]);
    }
    for (int i = 0; i < nthreads; ++i) {
        if (started[i]) pthread_join(th[i], NULL);
        failed |= w[i].failed;
    }
    return failed ? -1 : 0;
}

/* ------------------------------------------------------------------ pooling */

typedef struct {
    int B, S, Hq, Hkv, D, bs, n, G;
    const double *k, *q;
    double *kbar, *qbar;
} pool_ctx;

/* item = (b, h, j) flattened; writes kbar[b,h,j,:] and qbar[b,h,j,:]. */
static void pool_item(void *vctx, int64_t item, double *scratch) {
    (void)scratch;
    pool_ctx *c = (pool_ctx *)vctx;
    int j = (int)(item % c->n);
    int h = (int)((item / c->n) % c->Hkv);
    int b = (int)(item / ((int64_t)c->n * c->Hkv));
    double *kb = c->kbar + item * c->D;
    for (int d = 0; d < c->D; ++d) {
        double sum = 0.0;
        for (int t = j * c->bs; t < (j + 1) * c->bs; ++t)
            sum += c->k[(((int64_t)b * c->S + t) * c->Hkv + h) * c->D + d];
        kb[d] = sum / (double)c->bs;
    }
    if (c->q && c->qbar) {
        double *qb = c->qbar + item * c->D;
        for (int d = 0; d < c->D; ++d) {
            double sum = 0.0;
            for (int g = 0; g < c->G; ++g) {
                int hq = h * c->G + g;
                for (int t = j * c->bs; t < (j + 1) * c->bs; ++t)
                    sum += c->q[(((int64_t)b * c->S + t) * c->Hq + hq) * c->D + d];
            }
            qb[d] = sum / ((double)c->bs * (double)c->G);
        }
    }
}

int ora_block_pool(int B, int S, int Hq, int Hkv, int D, int bs,
                   const double *k, const double *q, double *kbar, double *qbar, int nthreads) {
    if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || S % bs || Hq % Hkv || !k || !kbar)
        return -1;
    pool_ctx c = {B, S, Hq, Hkv, D, bs, S / bs, Hq / Hkv, k, q, kbar, qbar};
    return ora_parallel_for(pool_item, &c, (int64_t)B * Hkv * c.n, nthreads, 0);
}

/* ---------------------------------------------------------------- selection */

typedef struct {
    int B, Hkv, n, D, topk;
    const double *qbar, *kbar;
    int32_t *idx;
    double *gap;
} select_ctx;

/* "a ranks before b": higher score first, then the lower block index. */
static int ranks_before(double sa, int ja, double sb, int jb) {
    return (sa > sb) || (sa == sb && ja < jb);
}

/* item = (b, h, i); scratch holds 3*n doubles: scores, candidate order (ints),
 * chosen flags (chars). */
static void select_item(void *vctx, int64_t item, double *scratch) {
    select_ctx *c = (select_ctx *)vctx;
    int i = (int)(item % c->n);
    int64_t bh = item / c->n;
    const double *qi = c->qbar + item * c->D;
    double *score = scratch;
    int *order = (int *)(scratch + c->n);
    char *chosen = (char *)(scratch + 2 * (size_t)c->n);

    /* scores of the earlier blocks j < i */
    for (int j = 0; j < i; ++j) {
        const double *kj = c->kbar + (bh * c->n + j) * c->D;
        double s = 0.0;
        for (int d = 0; d < c->D; ++d) s += qi[d] * kj[d];
        score[j] = s;
    }
    /* stable insertion sort of the candidates by rank */
    for (int j = 0; j < i; ++j) {
        int p = j;
        while (p > 0 && ranks_before(score[j], j, score[order[p - 1]], order[p - 1])) {
            order[p] = order[p - 1];
            --p;
        }
        order[p] = j;
    }
    int take = c->topk - 1 < i ? c->topk - 1 : i;
    /* chosen set = first `take` candidates plus the diagonal, ascending */
    memset(chosen, 0, (size_t)c->n);
    for (int r = 0; r < take; ++r) chosen[order[r]] = 1;
    chosen[i] = 1;
    int32_t *out = c->idx + item * c->topk;
    int w = 0;
    for (int j = 0; j <= i && w < c->topk; ++j)
        if (chosen[j]) out[w++] = j;
    for (; w < c->topk; ++w) out[w] = -1;
    /* the k-1-th and k-th ranked candidates exist only when i > k - 1 */
    if (c->gap)
        c->gap[item] = (c->topk >= 2 && i > c->topk - 1)
                           ? score[order[c->topk - 2]] - score[order[c->topk - 1]]
                           : NAN;
}

int ora_block_select(int B, int Hkv, int n, int D, int topk, const double *qbar,
                     const double *kbar, int32_t *idx, double *gap, int nthreads) {
    if (B < 1 || Hkv < 1 || n < 1 || D < 1 || topk < 1 || !qbar || !kbar || !idx) return -1;
    select_ctx c = {B, Hkv, n, D, topk, qbar, kbar, idx, gap};
    return ora_parallel_for(select_item, &c, (int64_t)B * Hkv * n, nthreads, 3 * (size_t)n);
}

/* ------------------------------------------------------- forward attention */

typedef struct {
    int B, S, Hq, Hkv, D, bs, n, G, topk;
    double scale;
    const double *q, *k, *v;
    const int32_t *idx;
    const int64_t *rows;
    int want_full;
    double *o_sp, *lse_sp, *o_full, *lse_full, *delta, *delta2;
} attn_ctx;

/* Marks the selected blocks of query block i for (b, kvh) in sel[0..n). */
static void mark_selected(const int32_t *idx, int64_t bh, int n, int topk, int i, char *sel) {
    memset(sel, 0, (size_t)n);
    const int32_t *row = idx + (bh * n + i) * topk;
    for (int r = 0; r < topk; ++r)
        if (row[r] >= 0 && row[r] < n) sel[row[r]] = 1;
}

/* One query row (b, hq, t).  Scratch: S logits + n selection flags. */
static void attn_row(const attn_ctx *c, int64_t r, double *scratch) {
    int b = (int)c->rows[3 * r], hq = (int)c->rows[3 * r + 1], t = (int)c->rows[3 * r + 2];
    int h = hq / c->G, i = t / c->bs;
    int64_t bh = (int64_t)b * c->Hkv + h;
    double *logit = scratch;
    char *sel = (char *)(scratch + c->S);
    mark_selected(c->idx, bh, c->n, c->topk, i, sel);
    const double *qt = c->q + (((int64_t)b * c->S + t) * c->Hq + hq) * c->D;

    /* logits over every causal key (full) or the selected causal keys (sparse) */
    for (int s = 0; s <= t; ++s) {
        if (!c->want_full && !sel[s / c->bs]) continue;
        const double *ks = c->k + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        double dot = 0.0;
        for (int d = 0; d < c->D; ++d) dot += qt[d] * ks[d];
        logit[s] = c->scale * dot;
    }
    /* log-sum-exp of the sparse set, each with its own maximum */
    double m_sp = -INFINITY;
    for (int s = 0; s <= t; ++s)
        if (sel[s / c->bs] && logit[s] > m_sp) m_sp = logit[s];
    double sum_sp = 0.0;
    for (int s = 0; s <= t; ++s)
        if (sel[s / c->bs]) sum_sp += exp(logit[s] - m_sp);
    double lse_sp = m_sp + log(sum_sp);
    double *osp = c->o_sp + r * c->D;
    for (int d = 0; d < c->D; ++d) osp[d] = 0.0;
    for (int s = 0; s <= t; ++s) {
        if (!sel[s / c->bs]) continue;
        double p = exp(logit[s] - lse_sp);
        const double *vs = c->v + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        for (int d = 0; d < c->D; ++d) osp[d] += p * vs[d];
    }
    c->lse_sp[r] = lse_sp;
    if (!c->want_full) return;

    double m_f = -INFINITY;
    for (int s = 0; s <= t; ++s)
        if (logit[s] > m_f) m_f = logit[s];
    double sum_f = 0.0;
    for (int s = 0; s <= t; ++s) sum_f += exp(logit[s] - m_f);
    double lse_f = m_f + log(sum_f);
    double *of = c->o_full + r * c->D;
    for (int d = 0; d < c->D; ++d) of[d] = 0.0;
    double dropped = 0.0;
    for (int s = 0; s <= t; ++s) {
        double p = exp(logit[s] - lse_f);
        const double *vs = c->v + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        for (int d = 0; d < c->D; ++d) of[d] += p * vs[d];
        if (!sel[s / c->bs]) dropped += p;
    }
    c->lse_full[r] = lse_f;
    c->delta[r] = dropped;
    c->delta2[r] = -expm1(lse_sp - lse_f);
}

static void attn_item(void *vctx, int64_t item, double *scratch) {
    attn_row((const attn_ctx *)vctx, item, scratch);
}

static int check_rows(const int64_t *rows, int64_t nrows, int B, int S, int Hq) {
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B) return -1;
        if (rows[3 * r + 1] < 0 || rows[3 * r + 1] >= Hq) return -1;
        if (rows[3 * r + 2] < 0 || rows[3 * r + 2] >= S) return -1;
    }
    return 0;
}

int ora_attn_rows(int B, int S, int Hq, int Hkv, int D, int bs, int topk, double scale,
                  const double *q, const double *k, const double *v, const int32_t *idx,
                  int64_t nrows, const int64_t *rows, int want_full,
                  double *o_sp, double *lse_sp, double *o_full, double *lse_full,
                  double *delta, double *delta2, int nthreads) {
    if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || S % bs || Hq % Hkv || topk < 1)
        return -1;
    if (!q || !k || !v || !idx || !rows || !o_sp || !lse_sp || nrows < 0) return -1;
    if (want_full && (!o_full || !lse_full || !delta || !delta2)) return -1;
    if (check_rows(rows, nrows, B, S, Hq)) return -1;
    attn_ctx c = {B, S, Hq, Hkv, D, bs, S / bs, Hq / Hkv, topk, scale, q, k, v, idx, rows,
                  want_full, o_sp, lse_sp, o_full, lse_full, delta, delta2};
    size_t scratch = (size_t)S + (size_t)(S / bs) / sizeof(double) + 1;
    return ora_parallel_for(attn_item, &c, nrows, nthreads, scratch);
}

/* ------------------------------------------------------- sparse backward */
/*
 * With P_ts = exp(scale q_t.k_s - LSE_t) over the selected causal keys s of
 * query t, O_t = sum_s P_ts v_s and upstream gradient dO_t:
 *   D_t   = dO_t . O_t
 *   dV_s  = sum_t P_ts dO_t
 *   dS_ts = P_ts (dO_t . v_s - D_t)
 *   dQ_t  = scale sum_s dS_ts k_s
 *   dK_s  = scale sum_t dS_ts q_t
 * summed over the G query heads that share the KV head of s.  These are the
 * derivatives of the softmax-weighted average; unselected pairs contribute 0.
 */
typedef struct {
    int B, S, Hq, Hkv, D, bs, n, G, topk;
    double scale;
    const double *q, *k, *v, *dO;
    const int32_t *idx;
    const int64_t *items;
    double *out_a, *out_b;
} bwd_ctx;

/* Sparse forward quantities for one query row: logits of selected causal keys
 * into logit[], returns LSE and writes O_t into o[D].  sel must be marked. */
static double row_sparse_forward(const bwd_ctx *c, int b, int hq, int t, const char *sel,
                                 double *logit, double *o) {
    int h = hq / c->G;
    const double *qt = c->q + (((int64_t)b * c->S + t) * c->Hq + hq) * c->D;
    double m = -INFINITY;
    for (int s = 0; s <= t; ++s) {
        if (!sel[s / c->bs]) continue;
        const double *ks = c->k + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        double dot = 0.0;
        for (int d = 0; d < c->D; ++d) dot += qt[d] * ks[d];
        logit[s] = c->scale * dot;
        if (logit[s] > m) m = logit[s];
    }
    double sum = 0.0;
    for (int s = 0; s <= t; ++s)
        if (sel[s / c->bs]) sum += exp(logit[s] - m);
    double lse = m + log(sum);
    for (int d = 0; d < c->D; ++d) o[d] = 0.0;
    for (int s = 0; s <= t; ++s) {
        if (!sel[s / c->bs]) continue;
        double p = exp(logit[s] - lse);
        const double *vs = c->v + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        for (int d = 0; d < c->D; ++d) o[d] += p * vs[d];
    }
    return lse;
}

/* dQ for row item (b, hq, t).  Scratch: S logits + D (O) + n flags. */
static void dq_item(void *vctx, int64_t r, double *scratch) {
    const bwd_ctx *c = (const bwd_ctx *)vctx;
    int b = (int)c->items[3 * r], hq = (int)c->items[3 * r + 1], t = (int)c->items[3 * r + 2];
    int h = hq / c->G, i = t / c->bs;
    double *logit = scratch, *o = scratch + c->S;
    char *sel = (char *)(scratch + c->S + c->D);
    mark_selected(c->idx, (int64_t)b * c->Hkv + h, c->n, c->topk, i, sel);
    double lse = row_sparse_forward(c, b, hq, t, sel, logit, o);
    const double *dot_ = c->dO + (((int64_t)b * c->S + t) * c->Hq + hq) * c->D;
    double Dt = 0.0;
    for (int d = 0; d < c->D; ++d) Dt += dot_[d] * o[d];
    double *dq = c->out_a + r * c->D;
    for (int d = 0; d < c->D; ++d) dq[d] = 0.0;
    for (int s = 0; s <= t; ++s) {
        if (!sel[s / c->bs]) continue;
        const double *ks = c->k + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        const double *vs = c->v + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
        double p = exp(logit[s] - lse);
        double dp = 0.0;
        for (int d = 0; d < c->D; ++d) dp += dot_[d] * vs[d];
        double ds = p * (dp - Dt);
        for (int d = 0; d < c->D; ++d) dq[d] += c->scale * ds * ks[d];
    }
}

/* dK, dV for key block item (b, kvh, j): all bs keys of the block.
 * Scratch: S logits + D (O) + n flags. */
static void dkv_item(void *vctx, int64_t r, double *scratch) {
    const bwd_ctx *c = (const bwd_ctx *)vctx;
    int b = (int)c->items[3 * r], h = (int)c->items[3 * r + 1], j = (int)c->items[3 * r + 2];
    double *logit = scratch, *o = scratch + c->S;
    char *sel = (char *)(scratch + c->S + c->D);
    double *dk = c->out_a + r * (int64_t)c->bs * c->D;
    double *dv = c->out_b + r * (int64_t)c->bs * c->D;
    for (int64_t e = 0; e < (int64_t)c->bs * c->D; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
    int64_t bh = (int64_t)b * c->Hkv + h;
    /* every query block i >= j whose selection contains j, every head of the group */
    for (int i = j; i < c->n; ++i) {
        mark_selected(c->idx, bh, c->n, c->topk, i, sel);
        if (!sel[j]) continue;
        for (int g = 0; g < c->G; ++g) {
            int hq = h * c->G + g;
            for (int t = i * c->bs; t < (i + 1) * c->bs; ++t) {
                double lse = row_sparse_forward(c, b, hq, t, sel, logit, o);
                const double *dot_ = c->dO + (((int64_t)b * c->S + t) * c->Hq + hq) * c->D;
                const double *qt = c->q + (((int64_t)b * c->S + t) * c->Hq + hq) * c->D;
                double Dt = 0.0;
                for (int d = 0; d < c->D; ++d) Dt += dot_[d] * o[d];
                for (int s = j * c->bs; s < (j + 1) * c->bs && s <= t; ++s) {
                    const double *vs = c->v + (((int64_t)b * c->S + s) * c->Hkv + h) * c->D;
                    double p = exp(logit[s] - lse);
                    double dp = 0.0;
                    for (int d = 0; d < c->D; ++d) dp += dot_[d] * vs[d];
                    double ds = p * (dp - Dt);
                    int so = s - j * c->bs;
                    for (int d = 0; d < c->D; ++d) {
                        dv[so * c->D + d] += p * dot_[d];
                        dk[so * c->D + d] += c->scale * ds * qt[d];
                    }
                }
            }
        }
    }
}

int ora_sparse_bwd_dq_rows(int B, int S, int Hq, int Hkv, int D, int bs, int topk, double scale,
                           const double *q, const double *k, const double *v, const double *dO,
                           const int32_t *idx, int64_t nrows, const int64_t *rows, double *dq,
                           int nthreads) {
    if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || S % bs || Hq % Hkv || topk < 1)
        return -1;
    if (!q || !k || !v || !dO || !idx || !rows || !dq || nrows < 0) return -1;
    if (check_rows(rows, nrows, B, S, Hq)) return -1;
    bwd_ctx c = {B, S, Hq, Hkv, D, bs, S / bs, Hq / Hkv, topk, scale, q, k, v, dO, idx, rows, dq, NULL};
    size_t scratch = (size_t)S + (size_t)D + (size_t)(S / bs) / sizeof(double) + 1;
    return ora_parallel_for(dq_item, &c, nrows, nthreads, scratch);
}

int ora_sparse_bwd_dkv_blocks(int B, int S, int Hq, int Hkv, int D, int bs, int topk,
                              double scale, const double *q, const double *k, const double *v,
                              const double *dO, const int32_t *idx, int64_t nblocks,
                              const int64_t *blocks, double *dk, double *dv, int nthreads) {
    if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || S % bs || Hq % Hkv || topk < 1)
        return -1;
    if (!q || !k || !v || !dO || !idx || !blocks || !dk || !dv || nblocks < 0) return -1;
    for (int64_t r = 0; r < nblocks; ++r) {
        if (blocks[3 * r] < 0 || blocks[3 * r] >= B) return -1;
        if (blocks[3 * r + 1] < 0 || blocks[3 * r + 1] >= Hkv) return -1;
        if (blocks[3 * r + 2] < 0 || blocks[3 * r + 2] >= S / bs) return -1;
    }
    bwd_ctx c = {B, S, Hq, Hkv, D, bs, S / bs, Hq / Hkv, topk, scale, q, k, v, dO, idx, blocks, dk, dv};
    size_t scratch = (size_t)S + (size_t)D + (size_t)(S / bs) / sizeof(double) + 1;
    return ora_parallel_for(dkv_item, &c, nblocks, nthreads, scratch);
}
