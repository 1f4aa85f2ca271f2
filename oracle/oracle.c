/*
 * CalibAtt oracle: a plain, slow, fp64 CPU statement of what the hot path
 * computes.  TEST INFRASTRUCTURE ONLY: the product library never links,
 * loads or calls this file; only the tests, the package's smoke check and the
 * CPU-baseline leg of the benchmark do.
 *
 * Source: "Accelerating Text-to-Video Generation with Calibrated Sparse
 * Attention" (Yehezkel et al., arXiv 2603.05503), as explained on the
 * zhichai.net page "让视频生成快 1.58 倍 ... CalibAtt" (cited below as
 * "explainer"), sections 二 (observations), 三 (method) and 六 (spatial
 * repetition).
 *
 * Every function follows the plain definition, written out: no tiling, no
 * online softmax, no reordering beyond what the definition states.  Inputs
 * are bf16 bit patterns (the exact values the GPU sees), widened exactly to
 * double.  Threads only split independent output rows.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> exact double */
static double bf16_to_double(uint16_t x) {
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* tiny thread pool: run fn(ctx, i) for i in [0, n) over `threads` workers   */
/* ------------------------------------------------------------------------ */
typedef void (*row_fn)(void *ctx, int64_t i, double *scratch);
typedef struct {
    row_fn fn;
    void *ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t lock;
    size_t scratch_doubles;
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *p = (pool_t *)arg;
    double *scratch = (double *)malloc(sizeof(double) * (p->scratch_doubles ? p->scratch_doubles : 1));
    for (;;) {
        int64_t i;
        pthread_mutex_lock(&p->lock);
        i = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (i >= p->n) break;
        p->fn(p->ctx, i, scratch);
    }
    free(scratch);
    return NULL;
}

static void run_rows(row_fn fn, void *ctx, int64_t n, int threads, size_t scratch_doubles) {
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n = n;
    p.next = 0;
    p.scratch_doubles = scratch_doubles;
    pthread_mutex_init(&p.lock, NULL);
    if (threads < 1) threads = 1;
    if (threads == 1) {
        pool_worker(&p);
    } else {
        pthread_t *t = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)threads);
        for (int i = 0; i < threads; ++i) pthread_create(&t[i], NULL, pool_worker, &p);
        for (int i = 0; i < threads; ++i) pthread_join(t[i], NULL);
        free(t);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------------ */
/* 1. Masked attention (explainer §三, online inference, non-repeated heads: */
/*    the skip list tells the kernel which B x B key blocks to compute).     */
/*    For query i in block-row r the kept key set is the union of the key    */
/*    blocks c with mask[h][r][c] = 1, clipped to [0, n):                    */
/*      s_ij = scale * q_i . k_j                                             */
/*      O_i  = sum_j exp(s_ij - m) v_j / sum_j exp(s_ij - m),  m = max_j s_ij */
/*      LSE_i = m + ln sum_j exp(s_ij - m)                                   */
/*    A row with no kept key gets O = 0 and LSE = -inf.                      */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k, *v;
    int heads, d, B;
    int64_t n, nb;
    double scale;
    const uint8_t *mask;
    const int64_t *rows;
    double *o, *lse;
} attn_ctx;

static void attn_row(void *vctx, int64_t idx, double *s) {
    attn_ctx *c = (attn_ctx *)vctx;
    int64_t gi = c->rows ? c->rows[idx] : idx; /* h * n + i */
    int64_t h = gi / c->n, i = gi % c->n;
    int64_t r = i / c->B;
    const uint16_t *qi = c->q + (h * c->n + i) * c->d;
    const uint8_t *mrow = c->mask + (h * c->nb + r) * c->nb;
    double *oi = c->o + idx * c->d;
    double m = -INFINITY;
    int64_t cnt = 0;
    for (int64_t j = 0; j < c->n; ++j) {
        if (!mrow[j / c->B]) continue;
        const uint16_t *kj = c->k + (h * c->n + j) * c->d;
        double dot = 0.0;
        for (int t = 0; t < c->d; ++t) dot += bf16_to_double(qi[t]) * bf16_to_double(kj[t]);
        s[cnt] = c->scale * dot;
        if (s[cnt] > m) m = s[cnt];
        ++cnt;
    }
    for (int t = 0; t < c->d; ++t) oi[t] = 0.0;
    if (cnt == 0) {
        c->lse[idx] = -INFINITY;
        return;
    }
    double l = 0.0;
    cnt = 0;
    for (int64_t j = 0; j < c->n; ++j) {
        if (!mrow[j / c->B]) continue;
        double p = exp(s[cnt++] - m);
        l += p;
        const uint16_t *vj = c->v + (h * c->n + j) * c->d;
        for (int t = 0; t < c->d; ++t) oi[t] += p * bf16_to_double(vj[t]);
    }
    for (int t = 0; t < c->d; ++t) oi[t] /= l;
    c->lse[idx] = m + log(l);
}

void oracle_masked_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             int heads, int64_t n, int d, int B, double scale,
                             const uint8_t *mask, const int64_t *rows, int64_t n_rows,
                             double *o, double *lse, int threads) {
    attn_ctx c = {q, k, v, heads, d, B, n, (n + B - 1) / B, scale, mask, rows, o, lse};
    if (!rows) n_rows = (int64_t)heads * n;
    run_rows(attn_row, &c, n_rows, threads, (size_t)n);
}

/* ------------------------------------------------------------------------ */
/* 2. Spatially repeated heads (explainer §三 "repeated head: only k = 5     */
/*    anchor rows are computed and broadcast to the other rows of the same   */
/*    frame", and §六 on row-major tokens within an H x W frame).            */
/*    Token t = f*H*W + row*W + col.  The k anchor rows are the centres of k */
/*    equal bands of the H rows: a_j = floor((2j+1)H / (2k)).  Every row     */
/*    takes the output of its nearest anchor (ties -> lower j), same frame,  */
/*    same column.  Anchor queries attend densely to all n keys.             */
/* ------------------------------------------------------------------------ */
void oracle_anchor_rows(int H, int k_anchor, int *anchors) {
    for (int j = 0; j < k_anchor; ++j)
        anchors[j] = (int)(((int64_t)(2 * j + 1) * H) / (2 * (int64_t)k_anchor));
}

void oracle_nearest_anchor(int H, int k_anchor, const int *anchors, int *owner) {
    for (int r = 0; r < H; ++r) {
        int best = 0;
        for (int j = 1; j < k_anchor; ++j)
            if (abs(r - anchors[j]) < abs(r - anchors[best])) best = j;
        owner[r] = best;
    }
}

typedef struct {
    const uint16_t *q, *k, *v;
    int d, F, H, W, k_anchor;
    int64_t n;
    double scale;
    const int *anchors, *owner;
    const int64_t *rows;
    double *o, *lse;
} rep_ctx;

static void rep_row(void *vctx, int64_t idx, double *s) {
    rep_ctx *c = (rep_ctx *)vctx;
    int64_t gi = c->rows ? c->rows[idx] : idx;
    int64_t h = gi / c->n, t = gi % c->n;
    int64_t hw = (int64_t)c->H * c->W;
    int64_t f = t / hw, rem = t % hw;
    int64_t row = rem / c->W, col = rem % c->W;
    int64_t a = c->anchors[c->owner[row]];
    int64_t src = f * hw + a * c->W + col; /* the anchor query this row copies */
    const uint16_t *qi = c->q + (h * c->n + src) * c->d;
    double *oi = c->o + idx * c->d;
    double m = -INFINITY;
    for (int64_t j = 0; j < c->n; ++j) {
        const uint16_t *kj = c->k + (h * c->n + j) * c->d;
        double dot = 0.0;
        for (int u = 0; u < c->d; ++u) dot += bf16_to_double(qi[u]) * bf16_to_double(kj[u]);
        s[j] = c->scale * dot;
        if (s[j] > m) m = s[j];
    }
    for (int u = 0; u < c->d; ++u) oi[u] = 0.0;
    double l = 0.0;
    for (int64_t j = 0; j < c->n; ++j) {
        double p = exp(s[j] - m);
        l += p;
        const uint16_t *vj = c->v + (h * c->n + j) * c->d;
        for (int u = 0; u < c->d; ++u) oi[u] += p * bf16_to_double(vj[u]);
    }
    for (int u = 0; u < c->d; ++u) oi[u] /= l;
    c->lse[idx] = m + log(l);
}

int oracle_repeat_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            int heads, int F, int H, int W, int d, int k_anchor, double scale,
                            const int64_t *rows, int64_t n_rows, double *o, double *lse,
                            int threads) {
    if (k_anchor < 1 || k_anchor > H) return -1;
    int *anchors = (int *)malloc(sizeof(int) * (size_t)k_anchor);
    int *owner = (int *)malloc(sizeof(int) * (size_t)H);
    oracle_anchor_rows(H, k_anchor, anchors);
    oracle_nearest_anchor(H, k_anchor, anchors, owner);
    int64_t n = (int64_t)F * H * W;
    rep_ctx c = {q, k, v, d, F, H, W, k_anchor, n, scale, anchors, owner, rows, o, lse};
    if (!rows) n_rows = (int64_t)heads * n;
    run_rows(rep_row, &c, n_rows, threads, (size_t)n);
    free(anchors);
    free(owner);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 3. Block energy (explainer §三, offline calibration, steps 1-2):          */
/*    P = softmax(scale * Q K^T) over all n keys (the post-softmax matrix),  */
/*    E[r,c] = (1/|I_r|) sum_{i in I_r} sum_{j in J_c} P_ij.                 */
/*    The page writes 1/B; |I_r| = B on every block-row but a ragged last    */
/*    one, where dividing by the rows present keeps every row sum at 1.      */
/*    Also returns LSE_i for each query row visited.                         */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k;
    int d, B;
    int64_t n, nb;
    double scale;
    const int64_t *blockrows;
    double *E, *lse;
} energy_ctx;

static void energy_blockrow(void *vctx, int64_t idx, double *s) {
    energy_ctx *c = (energy_ctx *)vctx;
    int64_t g = c->blockrows ? c->blockrows[idx] : idx; /* h * nb + r */
    int64_t h = g / c->nb, r = g % c->nb;
    int64_t i0 = r * c->B, i1 = i0 + c->B;
    if (i1 > c->n) i1 = c->n;
    double *Er = c->E + idx * c->nb;
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] = 0.0;
    for (int64_t i = i0; i < i1; ++i) {
        const uint16_t *qi = c->q + (h * c->n + i) * c->d;
        double m = -INFINITY;
        for (int64_t j = 0; j < c->n; ++j) {
            const uint16_t *kj = c->k + (h * c->n + j) * c->d;
            double dot = 0.0;
            for (int u = 0; u < c->d; ++u) dot += bf16_to_double(qi[u]) * bf16_to_double(kj[u]);
            s[j] = c->scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < c->n; ++j) l += exp(s[j] - m);
        double lse_i = m + log(l);
        if (c->lse) c->lse[idx * c->B + (i - i0)] = lse_i;
        for (int64_t j = 0; j < c->n; ++j) Er[j / c->B] += exp(s[j] - lse_i);
    }
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] /= (double)(i1 - i0);
}

void oracle_block_energy(const uint16_t *q, const uint16_t *k, int heads, int64_t n, int d,
                         int B, double scale, const int64_t *blockrows, int64_t n_blockrows,
                         double *E, double *lse, int threads) {
    int64_t nb = (n + B - 1) / B;
    energy_ctx c = {q, k, d, B, n, nb, scale, blockrows, E, lse};
    if (!blockrows) n_blockrows = (int64_t)heads * nb;
    run_rows(energy_blockrow, &c, n_blockrows, threads, (size_t)n);
}

/* ------------------------------------------------------------------------ */
/* 4. Greedy selection (explainer §三, step 3): in each block-row keep the   */
/*    fewest key blocks whose cumulative energy reaches eps.  Greedy order:  */
/*    energy descending, equal energies by lower column first.  The kept    */
/*    set is the shortest prefix of that order whose running sum is >= eps. */
/*    If no prefix reaches eps (rounding when eps ~ 1), every block with     */
/*    nonzero energy is kept and no zero-energy block.  At least one block   */
/*    is always kept (eps <= 0).                                             */
/*    Optional outputs describe the cut for tie accounting: the running sum  */
/*    before and at the last kept block, and the energies on both sides.     */
/* ------------------------------------------------------------------------ */
static const double *g_sort_keys;
static int cmp_desc_stable(const void *a, const void *b) {
    int ia = *(const int *)a, ib = *(const int *)b;
    double ea = g_sort_keys[ia], eb = g_sort_keys[ib];
    if (ea > eb) return -1;
    if (ea < eb) return 1;
    return (ia > ib) - (ia < ib);
}

void oracle_select(const double *E, int64_t n_rows, int nb, double eps, uint8_t *mask,
                   int32_t *kept, double *cum_before, double *cum_at, double *e_last,
                   double *e_next) {
    int *order = (int *)malloc(sizeof(int) * (size_t)nb);
    for (int64_t row = 0; row < n_rows; ++row) {
        const double *e = E + row * nb;
        for (int c = 0; c < nb; ++c) order[c] = c;
        g_sort_keys = e; /* single-threaded: the comparator reads this row */
        qsort(order, (size_t)nb, sizeof(int), cmp_desc_stable);
        double run = 0.0, before = 0.0;
        int m = 0;
        for (int i = 0; i < nb; ++i) {
            before = run;
            run += e[order[i]];
            if (run >= eps) {
                m = i + 1;
                break;
            }
        }
        if (m == 0) { /* eps not reached: keep every nonzero-energy block */
            before = 0.0;
            run = 0.0;
            for (int i = 0; i < nb; ++i)
                if (e[order[i]] > 0.0) {
                    before = run;
                    run += e[order[i]];
                    m = i + 1;
                }
        }
        if (m == 0) m = 1; /* at least one block per row */
        uint8_t *mr = mask + row * nb;
        memset(mr, 0, (size_t)nb);
        for (int i = 0; i < m; ++i) mr[order[i]] = 1;
        if (kept) kept[row] = m;
        if (cum_before) cum_before[row] = before;
        if (cum_at) cum_at[row] = run;
        if (e_last) e_last[row] = e[order[m - 1]];
        if (e_next) e_next[row] = (m < nb) ? e[order[m]] : -1.0;
    }
    free(order);
}

/* ------------------------------------------------------------------------ */
/* 5. Aggregation over calibration inputs (explainer §三):                   */
/*    Mbar = (1/|D|) sum_p M_p, kept where Mbar >= rho (rho = 0.5 in the     */
/*    paper).  Also returns the integer counts sum_p M_p.                    */
/* ------------------------------------------------------------------------ */
void oracle_aggregate(const uint8_t *masks, int n_inputs, int64_t cells, double rho,
                      uint8_t *mask_out, int32_t *counts_out) {
    for (int64_t x = 0; x < cells; ++x) {
        int32_t cnt = 0;
        for (int p = 0; p < n_inputs; ++p) cnt += masks[(int64_t)p * cells + x] ? 1 : 0;
        double mbar = (double)cnt / (double)n_inputs;
        mask_out[x] = (mbar >= rho) ? 1 : 0;
        if (counts_out) counts_out[x] = cnt;
    }
}

/* The same binarisation starting from counts (used when the per-input masks
 * are not kept): keep where count / n_inputs >= rho. */
void oracle_binarize_counts(const int32_t *counts, int n_inputs, int64_t cells, double rho,
                            uint8_t *mask_out) {
    for (int64_t x = 0; x < cells; ++x)
        mask_out[x] = ((double)counts[x] / (double)n_inputs >= rho) ? 1 : 0;
}

/* Skip list (explainer §三, online inference): for each (head, block-row),
 * the kept key blocks in ascending column order, as CSR with global offsets:
 * row_ptr[h*nb + r] .. row_ptr[h*nb + r + 1] index col_idx. */
int64_t oracle_mask_to_csr(const uint8_t *mask, int heads, int64_t nb, int32_t *row_ptr,
                           int32_t *col_idx) {
    int64_t nnz = 0;
    for (int64_t row = 0; row < (int64_t)heads * nb; ++row) {
        row_ptr[row] = (int32_t)nnz;
        for (int64_t c = 0; c < nb; ++c)
            if (mask[row * nb + c]) col_idx[nnz++] = (int32_t)c;
    }
    row_ptr[(int64_t)heads * nb] = (int32_t)nnz;
    return nnz;
}

/* The same skip list for any number of mask rows of `cols` columns (for
 * example the anchor-block rows of repeated heads). */
int64_t oracle_mask_rows_to_csr(const uint8_t *mask, int64_t rows, int64_t cols, int32_t *row_ptr,
                                int32_t *col_idx) {
    int64_t nnz = 0;
    for (int64_t row = 0; row < rows; ++row) {
        row_ptr[row] = (int32_t)nnz;
        for (int64_t c = 0; c < cols; ++c)
            if (mask[row * cols + c]) col_idx[nnz++] = (int32_t)c;
    }
    row_ptr[rows] = (int32_t)nnz;
    return nnz;
}

/* ------------------------------------------------------------------------ */
/* 6. Energy threshold schedule (explainer §三): eps(t) = A + (C - A) e^{-kt/T} */
/*    high (C) at the early, high-noise steps, relaxing towards A.           */
/* ------------------------------------------------------------------------ */
double oracle_eps_schedule(double A, double C, double k, double t, double T) {
    return A + (C - A) * exp(-k * t / T);
}

/* ------------------------------------------------------------------------ */
/* 7. Spatial similarity score of a head (explainer §三: a score s^(t,l,h)   */
/*    per head, flagged as spatially repeated when it exceeds gamma = 0.87;  */
/*    §二 observation 4 and §六: the pixel rows of a frame attend alike, so  */
/*    the k anchor rows can stand in for the rest).  The pages give no      */
/*    formula for s.  Reading used here:                                     */
/*      pixel row R = (f, r) holds the W queries i = f*H*W + r*W + c;         */
/*      its block-energy profile over the key blocks J_c' is                 */
/*        Epx[R][c'] = (1/W) sum_{i in R} sum_{j in J_c'} P_ij,              */
/*      P = softmax(scale Q K^T) over all n keys (as for the block energy);   */
/*      s = mean over frames f and non-anchor rows r of                      */
/*          cos(Epx[(f, r)], Epx[(f, a(r))]),  a(r) the row's nearest anchor  */
/*          (the row whose output the repeated head copies to it).           */
/*    A head whose every row is an anchor (k = H) has s = 1; a cosine with a */
/*    zero profile counts as 0.                                              */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k;
    int d, B, W;
    int64_t n, nb, n_prow; /* pixel rows per head = F*H */
    double scale;
    const int64_t *prows;
    double *Epx;
} prow_ctx;

static void prow_energy_row(void *vctx, int64_t idx, double *s) {
    prow_ctx *c = (prow_ctx *)vctx;
    int64_t g = c->prows ? c->prows[idx] : idx; /* h * n_prow + R */
    int64_t h = g / c->n_prow, R = g % c->n_prow;
    double *Er = c->Epx + idx * c->nb;
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] = 0.0;
    for (int64_t i = R * c->W; i < (R + 1) * c->W; ++i) {
        const uint16_t *qi = c->q + (h * c->n + i) * c->d;
        double m = -INFINITY;
        for (int64_t j = 0; j < c->n; ++j) {
            const uint16_t *kj = c->k + (h * c->n + j) * c->d;
            double dot = 0.0;
            for (int u = 0; u < c->d; ++u) dot += bf16_to_double(qi[u]) * bf16_to_double(kj[u]);
            s[j] = c->scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < c->n; ++j) l += exp(s[j] - m);
        double lse_i = m + log(l);
        for (int64_t j = 0; j < c->n; ++j) Er[j / c->B] += exp(s[j] - lse_i);
    }
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] /= (double)c->W;
}

void oracle_pixel_row_energy(const uint16_t *q, const uint16_t *k, int heads, int F, int H, int W, int d,
                             int B, double scale, const int64_t *prows, int64_t n_prows, double *Epx,
                             int threads) {
    int64_t n = (int64_t)F * H * W;
    prow_ctx c = {q, k, d, B, W, n, (n + B - 1) / B, (int64_t)F * H, scale, prows, Epx};
    if (!prows) n_prows = (int64_t)heads * F * H;
    run_rows(prow_energy_row, &c, n_prows, threads, (size_t)n);
}

/* s of one head from its profiles Epx [F*H][nb]. */
double oracle_spatial_score(const double *Epx, int F, int H, int64_t nb, int k_anchor) {
    int *anchors = (int *)malloc(sizeof(int) * (size_t)k_anchor);
    int *owner = (int *)malloc(sizeof(int) * (size_t)H);
    oracle_anchor_rows(H, k_anchor, anchors);
    oracle_nearest_anchor(H, k_anchor, anchors, owner);
    double total = 0.0;
    int64_t count = 0;
    for (int f = 0; f < F; ++f) {
        for (int r = 0; r < H; ++r) {
            int a = anchors[owner[r]];
            if (a == r) continue; /* an anchor row is computed, not copied */
            const double *x = Epx + ((int64_t)f * H + r) * nb;
            const double *y = Epx + ((int64_t)f * H + a) * nb;
            double xy = 0.0, xx = 0.0, yy = 0.0;
            for (int64_t c = 0; c < nb; ++c) {
                xy += x[c] * y[c];
                xx += x[c] * x[c];
                yy += y[c] * y[c];
            }
            total += (xx > 0.0 && yy > 0.0) ? xy / (sqrt(xx) * sqrt(yy)) : 0.0;
            ++count;
        }
    }
    free(anchors);
    free(owner);
    return count ? total / (double)count : 1.0;
}

/* ------------------------------------------------------------------------ */
/* 8. Repeated heads with a block mask on their anchor rows (explainer §三:  */
/*    the two run-time decisions, a skip list for a head's blocks and the    */
/*    spatial repetition of its rows, are both made per (t, l, h); the pages */
/*    do not combine them, and this reading applies both: a repeated head    */
/*    computes only its anchor rows, and those anchor queries attend only to */
/*    the key blocks their own calibrated mask keeps).                       */
/*    The anchor queries of a head are taken in the order frame, anchor,     */
/*    column: packed row a = f*k*W + j*W + c is token f*H*W + a_j*W + c.     */
/*    They are grouped into blocks of B packed rows (the last one ragged),   */
/*    and calibrated exactly like query blocks: the energy of packed block   */
/*    r over key block c is (1/|I_r|) sum_{i in I_r, j in J_c} P_ij.         */
/*    At run time the anchor query in packed block r attends to the keys of  */
/*    the kept blocks mask_b[h][r][*], and every row takes the output of its */
/*    nearest anchor row (same frame, same column), as in section 2.         */
/* ------------------------------------------------------------------------ */
static int64_t packed_to_token(int64_t a, int W, int H, int k_anchor, const int *anchors) {
    int64_t kw = (int64_t)k_anchor * W;
    int64_t f = a / kw, rem = a % kw;
    int64_t j = rem / W, c = rem % W;
    return f * (int64_t)H * W + (int64_t)anchors[j] * W + c;
}

typedef struct {
    const uint16_t *q, *k;
    int d, B, H, W, k_anchor;
    int64_t n, nq, nbq, nb; /* nq = F*k*W packed anchor queries per head */
    double scale;
    const int *anchors;
    const int64_t *blockrows;
    double *E;
} anchor_energy_ctx;

static void anchor_energy_blockrow(void *vctx, int64_t idx, double *s) {
    anchor_energy_ctx *c = (anchor_energy_ctx *)vctx;
    int64_t g = c->blockrows ? c->blockrows[idx] : idx; /* h * nbq + r */
    int64_t h = g / c->nbq, r = g % c->nbq;
    int64_t a0 = r * c->B, a1 = a0 + c->B;
    if (a1 > c->nq) a1 = c->nq;
    double *Er = c->E + idx * c->nb;
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] = 0.0;
    for (int64_t a = a0; a < a1; ++a) {
        int64_t i = packed_to_token(a, c->W, c->H, c->k_anchor, c->anchors);
        const uint16_t *qi = c->q + (h * c->n + i) * c->d;
        double m = -INFINITY;
        for (int64_t j = 0; j < c->n; ++j) {
            const uint16_t *kj = c->k + (h * c->n + j) * c->d;
            double dot = 0.0;
            for (int u = 0; u < c->d; ++u) dot += bf16_to_double(qi[u]) * bf16_to_double(kj[u]);
            s[j] = c->scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < c->n; ++j) l += exp(s[j] - m);
        double lse_i = m + log(l);
        for (int64_t j = 0; j < c->n; ++j) Er[j / c->B] += exp(s[j] - lse_i);
    }
    for (int64_t cc = 0; cc < c->nb; ++cc) Er[cc] /= (double)(a1 - a0);
}

/* E: [n_blockrows][nb] for blockrows h*nbq + r (all of them when NULL). */
int oracle_anchor_block_energy(const uint16_t *q, const uint16_t *k, int heads, int F, int H, int W, int d,
                               int B, int k_anchor, double scale, const int64_t *blockrows,
                               int64_t n_blockrows, double *E, int threads) {
    if (k_anchor < 1 || k_anchor > H) return -1;
    int *anchors = (int *)malloc(sizeof(int) * (size_t)k_anchor);
    oracle_anchor_rows(H, k_anchor, anchors);
    int64_t n = (int64_t)F * H * W, nq = (int64_t)F * k_anchor * W;
    anchor_energy_ctx c = {q, k, d, B, H, W, k_anchor, n, nq, (nq + B - 1) / B, (n + B - 1) / B, scale,
                           anchors, blockrows, E};
    if (!blockrows) n_blockrows = (int64_t)heads * c.nbq;
    run_rows(anchor_energy_blockrow, &c, n_blockrows, threads, (size_t)n);
    free(anchors);
    return 0;
}

typedef struct {
    const uint16_t *q, *k, *v;
    int d, B, H, W, k_anchor;
    int64_t n, nbq, nb;
    double scale;
    const int *anchors, *owner;
    const uint8_t *mask_b; /* [heads][nbq][nb] */
    const int64_t *rows;
    double *o, *lse;
} rep_masked_ctx;

static void rep_masked_row(void *vctx, int64_t idx, double *s) {
    rep_masked_ctx *c = (rep_masked_ctx *)vctx;
    int64_t gi = c->rows ? c->rows[idx] : idx;
    int64_t h = gi / c->n, t = gi % c->n;
    int64_t hw = (int64_t)c->H * c->W;
    int64_t f = t / hw, rem = t % hw;
    int64_t row = rem / c->W, col = rem % c->W;
    int64_t jn = c->owner[row];                         /* nearest anchor */
    int64_t a = f * (int64_t)c->k_anchor * c->W + jn * c->W + col; /* its packed index */
    int64_t src = f * hw + (int64_t)c->anchors[jn] * c->W + col;   /* its token */
    const uint8_t *mrow = c->mask_b + (h * c->nbq + a / c->B) * c->nb;
    const uint16_t *qi = c->q + (h * c->n + src) * c->d;
    double *oi = c->o + idx * c->d;
    double m = -INFINITY;
    int64_t cnt = 0;
    for (int64_t j = 0; j < c->n; ++j) {
        if (!mrow[j / c->B]) continue;
        const uint16_t *kj = c->k + (h * c->n + j) * c->d;
        double dot = 0.0;
        for (int u = 0; u < c->d; ++u) dot += bf16_to_double(qi[u]) * bf16_to_double(kj[u]);
        s[cnt] = c->scale * dot;
        if (s[cnt] > m) m = s[cnt];
        ++cnt;
    }
    for (int u = 0; u < c->d; ++u) oi[u] = 0.0;
    if (cnt == 0) {
        c->lse[idx] = -INFINITY;
        return;
    }
    double l = 0.0;
    cnt = 0;
    for (int64_t j = 0; j < c->n; ++j) {
        if (!mrow[j / c->B]) continue;
        double p = exp(s[cnt++] - m);
        l += p;
        const uint16_t *vj = c->v + (h * c->n + j) * c->d;
        for (int u = 0; u < c->d; ++u) oi[u] += p * bf16_to_double(vj[u]);
    }
    for (int u = 0; u < c->d; ++u) oi[u] /= l;
    c->lse[idx] = m + log(l);
}

int oracle_repeat_attention_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v, int heads, int F,
                                   int H, int W, int d, int B, int k_anchor, double scale,
                                   const uint8_t *mask_b, const int64_t *rows, int64_t n_rows, double *o,
                                   double *lse, int threads) {
    if (k_anchor < 1 || k_anchor > H) return -1;
    int *anchors = (int *)malloc(sizeof(int) * (size_t)k_anchor);
    int *owner = (int *)malloc(sizeof(int) * (size_t)H);
    oracle_anchor_rows(H, k_anchor, anchors);
    oracle_nearest_anchor(H, k_anchor, anchors, owner);
    int64_t n = (int64_t)F * H * W, nq = (int64_t)F * k_anchor * W;
    rep_masked_ctx c = {q, k, v, d, B, H, W, k_anchor, n, (nq + B - 1) / B, (n + B - 1) / B, scale,
                        anchors, owner, mask_b, rows, o, lse};
    if (!rows) n_rows = (int64_t)heads * n;
    run_rows(rep_masked_row, &c, n_rows, threads, (size_t)n);
    free(anchors);
    free(owner);
    return 0;
}
