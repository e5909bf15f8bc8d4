/*
 * mra_oracle.c - plain, slow fp64 CPU oracle of the MRA-2 approximate
 * self-attention forward pass and of its gradient.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into a separate shared
 * library that only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg load.  The CUDA library never links, includes or calls it,
 * and it shares no code, header or constant table with the CUDA library.
 *
 * Source: the page "深入解析 Transformers 中的 MRA 模型：多分辨率近似自注意力
 * 机制的架构、配置与实战" (blog.gitcode.com), cited below as [MRA page]:
 *   - section "MraConfig：四个专属参数与完整默认值": the four knobs
 *     (block_per_row, approx_mode, initial_prior_first_n_blocks,
 *     initial_prior_diagonal_n_blocks) and the num_block formula;
 *   - section "源码级原理：MRA 两级注意力到底怎么算", steps one to four
 *     (第一步 .. 第四步), and the paragraph on engineering details that follows
 *     them (N must be a multiple of the 32-token block).
 *
 * Every floating-point step runs in double precision on inputs that the
 * caller has widened exactly from their fp32 or bf16 bytes.  Where the page
 * leaves a step open, the reading taken is stated at the step; the list of
 * readings lives in the design notes of the repository.
 *
 * Notation: BH = B*H meta-batch, nbr = N/32 blocks per sequence, block b holds
 * tokens 32b..32b+31, m_t in {0,1} is the key-padding mask of token t (shared
 * by all heads of a batch entry), cnt_b = sum of m_t over block b.
 *
 * Parity status of each function (what pins it) is listed in the header of
 * oracle/__init__.py; nothing here is pinned by this file itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define MRA_ORACLE_BLOCK 32

/* Penalty for empty blocks and bias for prior blocks, as printed on the page
 * (step one: empty blocks pushed to a very small value; step two: a 5e3 bias
 * on prior blocks).  The empty-block penalty of 1e4 is the reading taken for
 * "压到极小值" (pushed to a tiny value). */
static const double ORACLE_EMPTY_PENALTY = 1.0e4;
static const double ORACLE_PRIOR_BIAS = 5.0e3;

/* [MRA page, "MraConfig：四个专属参数与完整默认值", num_block formula]:
 * num_block = min((L/32) * block_per_row, (L/32)^2).  Here L is the sequence
 * length N of the call. */
long mra_oracle_num_block(long N, long block_per_row)
{
    long nbr = N / MRA_ORACLE_BLOCK;
    long budget = nbr * block_per_row;
    long all = nbr * nbr;
    return budget < all ? budget : all;
}

/* Valid-token count of every block, cnt[b][blk] = sum of m_t over the block.
 * mask is [B][N] with 0/1 entries, or NULL for "every token valid".
 * [MRA page, step one: the mean uses the count of valid tokens per block.] */
void mra_oracle_block_counts(const double *mask, int B, int N, double *cnt)
{
    int nbr = N / MRA_ORACLE_BLOCK;
    for (int b = 0; b < B; ++b)
        for (int blk = 0; blk < nbr; ++blk) {
            double s = 0.0;
            for (int t = 0; t < MRA_ORACLE_BLOCK; ++t)
                s += mask ? mask[(size_t)b * N + blk * MRA_ORACLE_BLOCK + t] : 1.0;
            cnt[(size_t)b * nbr + blk] = s;
        }
}

/* Masked block mean of one head's [N][D] rows into xhat [nbr][D]:
 * xhat_b = sum_{t in b} m_t x_t / cnt_b, and 0 when cnt_b = 0.
 * [MRA page, step one: reshape to (seq/32, 32, head_dim) and take the mean
 * over the block, counting only valid tokens when a mask is given.] */
static void pool_head(const double *x, const double *mask_row, int N, int D,
                      double *xhat)
{
    int nbr = N / MRA_ORACLE_BLOCK;
    for (int blk = 0; blk < nbr; ++blk) {
        double c = 0.0;
        for (int d = 0; d < D; ++d) xhat[(size_t)blk * D + d] = 0.0;
        for (int t = blk * MRA_ORACLE_BLOCK; t < (blk + 1) * MRA_ORACLE_BLOCK; ++t) {
            double m = mask_row ? mask_row[t] : 1.0;
            c += m;
            for (int d = 0; d < D; ++d) xhat[(size_t)blk * D + d] += m * x[(size_t)t * D + d];
        }
        for (int d = 0; d < D; ++d)
            xhat[(size_t)blk * D + d] = (c > 0.0) ? xhat[(size_t)blk * D + d] / c : 0.0;
    }
}

/* Pool every head: x is [B][H][N][D], xhat is [B*H][nbr][D]. */
void mra_oracle_pool(const double *x, const double *mask, int B, int H, int N, int D,
                     double *xhat)
{
    int nbr = N / MRA_ORACLE_BLOCK;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t bh = (size_t)b * H + h;
            pool_head(x + bh * N * D, mask ? mask + (size_t)b * N : NULL, N, D,
                      xhat + bh * nbr * D);
        }
}

/* Low-resolution logits of one head: logit[r][c] = qhat_r . khat_c / sqrt(D).
 * [MRA page, step one: a small full matmul query_hat @ key_hat^T on block
 * granularity.]  Reading: the same 1/sqrt(D) scale as the high-resolution
 * scores (the page prints no scale for this map). */
static void lowres_logits_head(const double *qhat, const double *khat, int nbr, int D,
                               double *logit)
{
    double scale = 1.0 / sqrt((double)D);
    for (int r = 0; r < nbr; ++r)
        for (int c = 0; c < nbr; ++c) {
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += qhat[(size_t)r * D + d] * khat[(size_t)c * D + d];
            logit[(size_t)r * nbr + c] = s * scale;
        }
}

void mra_oracle_lowres_logits(const double *qhat, const double *khat, int BH, int nbr,
                              int D, double *logit)
{
    for (int bh = 0; bh < BH; ++bh)
        lowres_logits_head(qhat + (size_t)bh * nbr * D, khat + (size_t)bh * nbr * D, nbr, D,
                           logit + (size_t)bh * nbr * nbr);
}

/* Row max of the low-resolution map over valid key blocks:
 * mlo[r] = max over c with cnt_c > 0 of logit[r][c]; 0 when no column is
 * valid.  [MRA page, step four: the low-resolution row maximum that
 * log_correction reconciles with the high-resolution one.]  Reading: taken
 * over valid columns, before any penalty. */
static void row_max_head(const double *logit, const double *cnt_row, int nbr, double *mlo)
{
    for (int r = 0; r < nbr; ++r) {
        int any = 0;
        double m = 0.0;
        for (int c = 0; c < nbr; ++c) {
            if (!(cnt_row[c] > 0.0)) continue;
            double v = logit[(size_t)r * nbr + c];
            if (!any || v > m) m = v;
            any = 1;
        }
        mlo[r] = any ? m : 0.0;
    }
}

void mra_oracle_row_max(const double *logit, const double *cnt, int B, int H, int nbr,
                        double *mlo)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t bh = (size_t)b * H + h;
            row_max_head(logit + bh * nbr * nbr, cnt + (size_t)b * nbr, nbr, mlo + bh * nbr);
        }
}

/* Is block (r, c) inside the diagonal prior band of width g?  The band is
 * centred on the main diagonal: offsets c - r in [-floor(g/2), ceil(g/2) - 1],
 * so g = 1 is the diagonal itself and g = 3 is |r - c| <= 1.
 * [MRA page, step two: a bias on the band of blocks centred on the main
 * diagonal when initial_prior_diagonal_n_blocks > 0.] */
static int in_diagonal_band(int r, int c, int g)
{
    if (g <= 0) return 0;
    int lo = -(g / 2);
    int hi = (g + 1) / 2 - 1;
    int off = c - r;
    return off >= lo && off <= hi;
}

/* Selection key of one head, in exact fp64 arithmetic:
 * key[r][c] = (logit[r][c] - mlo[r])
 *             - 1e4 * ([cnt_r == 0] + [cnt_c == 0])
 *             + 5e3 * ([f > 0 and (r < f or c < f)] + [(r, c) in the band]).
 * [MRA page, step one (empty-block rows and columns pushed down) and step two
 * (5e3 bias on the first-n row/column blocks and on the diagonal band).]
 * Readings: the map is ranked relative to each row's maximum; the two prior
 * biases add up when a block is in both priors. */
static void selection_keys_head(const double *logit, const double *mlo, const double *cnt_row,
                                int nbr, int first_n, int diag_n, double *key)
{
    for (int r = 0; r < nbr; ++r)
        for (int c = 0; c < nbr; ++c) {
            double v = logit[(size_t)r * nbr + c] - mlo[r];
            if (!(cnt_row[r] > 0.0)) v -= ORACLE_EMPTY_PENALTY;
            if (!(cnt_row[c] > 0.0)) v -= ORACLE_EMPTY_PENALTY;
            if (first_n > 0 && (r < first_n || c < first_n)) v += ORACLE_PRIOR_BIAS;
            if (in_diagonal_band(r, c, diag_n)) v += ORACLE_PRIOR_BIAS;
            key[(size_t)r * nbr + c] = v;
        }
}

void mra_oracle_selection_keys(const double *logit, const double *mlo, const double *cnt,
                               int B, int H, int nbr, int first_n, int diag_n, double *key)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t bh = (size_t)b * H + h;
            selection_keys_head(logit + bh * nbr * nbr, mlo + bh * nbr, cnt + (size_t)b * nbr,
                                nbr, first_n, diag_n, key + bh * nbr * nbr);
        }
}

typedef struct {
    double key;
    int32_t idx;
} keyed_t;

/* Larger key first; equal keys: smaller flat index first. */
static int keyed_cmp(const void *pa, const void *pb)
{
    const keyed_t *a = (const keyed_t *)pa, *b = (const keyed_t *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

static int idx_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Global top-k of one head's nbr*nbr keys: sort by key descending, equal keys
 * by smaller flat index r*nbr + c, keep the first k, and return them sorted
 * by flat index.  [MRA page, step two: a global top-k over the low-resolution
 * map with k = num_block.]  Reading: the tie rule (smaller index wins) is
 * this oracle's, the page names none. */
static void select_head(const double *key, int nbr, long k, int32_t *sel)
{
    long n = (long)nbr * nbr;
    keyed_t *tmp = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)n);
    for (long i = 0; i < n; ++i) {
        tmp[i].key = key[i];
        tmp[i].idx = (int32_t)i;
    }
    qsort(tmp, (size_t)n, sizeof(keyed_t), keyed_cmp);
    for (long i = 0; i < k; ++i) sel[i] = tmp[i].idx;
    qsort(sel, (size_t)k, sizeof(int32_t), idx_cmp);
    free(tmp);
}

void mra_oracle_select(const double *key, int BH, int nbr, long k, int32_t *sel)
{
    for (int bh = 0; bh < BH; ++bh)
        select_head(key + (size_t)bh * nbr * nbr, nbr, k, sel + (size_t)bh * k);
}

/* Attention of one head given its selected set.
 * For query i in block r with m_i = 1 the included terms are
 *   - for every selected (r, c) and every valid key j in block c:
 *     weight e^{s_ij}, value v_j, with s_ij = q_i . k_j / sqrt(D)
 *     [MRA page, step three: scores only on the selected blocks, row max,
 *     exp times V, and the sum of weights as normaliser];
 *   - in full mode, for every unselected c with cnt_c > 0:
 *     weight cnt_c * e^{logit[r][c]}, value vhat_c, the same for every query
 *     of block r [MRA page, step four: block-pooled V times the
 *     low-resolution weights, repeated over the 32 tokens of the block, with
 *     both parts brought to a shared maximum before the normalisers add].
 * out_i = sum(weight * value) / sum(weight), evaluated with the true maximum
 * over the included exponents.  A row with no term, and every padded query
 * (m_i = 0), gets 0 (reading: the page leaves both open). */
static void attend_head(const double *q, const double *k, const double *v,
                        const double *mask_row, const double *cnt_row,
                        const double *logit, const double *vhat, const unsigned char *selected,
                        int N, int D, int full_mode, double *out)
{
    int nbr = N / MRA_ORACLE_BLOCK;
    double scale = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    for (int i = 0; i < N; ++i) {
        int r = i / MRA_ORACLE_BLOCK;
        double *o = out + (size_t)i * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (mask_row && !(mask_row[i] > 0.0)) continue;

        /* exponents of every included term, and their maximum */
        int any = 0;
        double mx = 0.0;
        for (int c = 0; c < nbr; ++c) {
            if (selected[(size_t)r * nbr + c]) {
                for (int j = c * MRA_ORACLE_BLOCK; j < (c + 1) * MRA_ORACLE_BLOCK; ++j) {
                    if (mask_row && !(mask_row[j] > 0.0)) continue;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += q[(size_t)i * D + d] * k[(size_t)j * D + d];
                    s[j] = dot * scale;
                    if (!any || s[j] > mx) mx = s[j];
                    any = 1;
                }
            } else if (full_mode && cnt_row[c] > 0.0) {
                double l = logit[(size_t)r * nbr + c];
                if (!any || l > mx) mx = l;
                any = 1;
            }
        }
        if (!any) continue;

        double den = 0.0;
        for (int c = 0; c < nbr; ++c) {
            if (selected[(size_t)r * nbr + c]) {
                for (int j = c * MRA_ORACLE_BLOCK; j < (c + 1) * MRA_ORACLE_BLOCK; ++j) {
                    if (mask_row && !(mask_row[j] > 0.0)) continue;
                    double w = exp(s[j] - mx);
                    den += w;
                    for (int d = 0; d < D; ++d) o[d] += w * v[(size_t)j * D + d];
                }
            } else if (full_mode && cnt_row[c] > 0.0) {
                double w = cnt_row[c] * exp(logit[(size_t)r * nbr + c] - mx);
                den += w;
                for (int d = 0; d < D; ++d) o[d] += w * vhat[(size_t)c * D + d];
            }
        }
        for (int d = 0; d < D; ++d) o[d] /= den;
    }
    free(s);
}

/* The whole forward pass, step by step, one (batch, head) at a time.
 * q, k, v, out: [B][H][N][D]; mask: [B][N] of 0/1 or NULL.
 * mode 0 = "full" (high resolution plus low-resolution correction),
 * mode 1 = "sparse" (high resolution only)
 * [MRA page, table of MraConfig knobs, approx_mode].
 * Optional outputs (NULL to skip):
 *   sel    [B*H][k]        selected flat indices r*nbr + c, ascending
 *   key    [B*H][nbr][nbr] selection keys
 *   logit  [B*H][nbr][nbr] low-resolution logits
 *   pooled [3][B*H][nbr][D] qhat, khat, vhat
 *   cnt    [B][nbr]        valid tokens per block
 * nthreads <= 0 leaves the OpenMP default.
 * Returns 0, or -1 on invalid arguments (N not a multiple of 32
 * [MRA page, engineering-details paragraph], bad mode, block_per_row < 1,
 * priors outside [0, nbr]). */
int mra_oracle_forward(const double *q, const double *k, const double *v, const double *mask,
                       int B, int H, int N, int D, int block_per_row, int mode, int first_n,
                       int diag_n, double *out, int32_t *sel, double *key, double *logit,
                       double *pooled, double *cnt_out, int nthreads)
{
    if (B < 1 || H < 1 || N < MRA_ORACLE_BLOCK || N % MRA_ORACLE_BLOCK != 0 || D < 1) return -1;
    if (block_per_row < 1 || (mode != 0 && mode != 1)) return -1;
    int nbr = N / MRA_ORACLE_BLOCK;
    if (first_n < 0 || first_n > nbr || diag_n < 0 || diag_n > nbr) return -1;
    long kk = mra_oracle_num_block(N, block_per_row);
    int BH = B * H;

    double *cnt = (double *)malloc(sizeof(double) * (size_t)B * nbr);
    mra_oracle_block_counts(mask, B, N, cnt);
    if (cnt_out) memcpy(cnt_out, cnt, sizeof(double) * (size_t)B * nbr);

#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        int b = bh / H;
        size_t xoff = (size_t)bh * N * D;
        const double *mrow = mask ? mask + (size_t)b * N : NULL;
        const double *crow = cnt + (size_t)b * nbr;
        double *qh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *vh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *lg = (double *)malloc(sizeof(double) * (size_t)nbr * nbr);
        double *ml = (double *)malloc(sizeof(double) * (size_t)nbr);
        double *ky = (double *)malloc(sizeof(double) * (size_t)nbr * nbr);
        int32_t *sl = (int32_t *)malloc(sizeof(int32_t) * (size_t)kk);
        unsigned char *is_sel = (unsigned char *)calloc((size_t)nbr * nbr, 1);

        /* step one: pool, low-resolution logits, row max */
        pool_head(q + xoff, mrow, N, D, qh);
        pool_head(k + xoff, mrow, N, D, kh);
        pool_head(v + xoff, mrow, N, D, vh);
        lowres_logits_head(qh, kh, nbr, D, lg);
        row_max_head(lg, crow, nbr, ml);
        /* step two: keys with penalties and priors, global top-k */
        selection_keys_head(lg, ml, crow, nbr, first_n, diag_n, ky);
        select_head(ky, nbr, kk, sl);
        for (long i = 0; i < kk; ++i) is_sel[sl[i]] = 1;
        /* steps three and four: high resolution on the selected blocks,
         * low-resolution correction (full mode), shared normaliser */
        attend_head(q + xoff, k + xoff, v + xoff, mrow, crow, lg, vh, is_sel, N, D, mode == 0,
                    out + xoff);

        if (sel) memcpy(sel + (size_t)bh * kk, sl, sizeof(int32_t) * (size_t)kk);
        if (key) memcpy(key + (size_t)bh * nbr * nbr, ky, sizeof(double) * (size_t)nbr * nbr);
        if (logit) memcpy(logit + (size_t)bh * nbr * nbr, lg, sizeof(double) * (size_t)nbr * nbr);
        if (pooled) {
            size_t plane = (size_t)BH * nbr * D;
            memcpy(pooled + 0 * plane + (size_t)bh * nbr * D, qh, sizeof(double) * (size_t)nbr * D);
            memcpy(pooled + 1 * plane + (size_t)bh * nbr * D, kh, sizeof(double) * (size_t)nbr * D);
            memcpy(pooled + 2 * plane + (size_t)bh * nbr * D, vh, sizeof(double) * (size_t)nbr * D);
        }
        free(qh); free(kh); free(vh); free(lg); free(ml); free(ky); free(sl); free(is_sel);
    }
    free(cnt);
    return 0;
}

/* Attention given an externally chosen selected set (used by tests that fix
 * the selection, e.g. to evaluate the GPU's own index set when it differs
 * from the oracle's only at near-ties).  sel is [B*H][k] flat indices. */
int mra_oracle_attend_with_selection(const double *q, const double *k, const double *v,
                                     const double *mask, int B, int H, int N, int D, int mode,
                                     const int32_t *sel, long kk, double *out, int nthreads)
{
    if (B < 1 || H < 1 || N < MRA_ORACLE_BLOCK || N % MRA_ORACLE_BLOCK != 0 || D < 1) return -1;
    if (mode != 0 && mode != 1) return -1;
    int nbr = N / MRA_ORACLE_BLOCK;
    int BH = B * H;
    double *cnt = (double *)malloc(sizeof(double) * (size_t)B * nbr);
    mra_oracle_block_counts(mask, B, N, cnt);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int bh = 0; bh < BH; ++bh) {
        int b = bh / H;
        size_t xoff = (size_t)bh * N * D;
        const double *mrow = mask ? mask + (size_t)b * N : NULL;
        const double *crow = cnt + (size_t)b * nbr;
        double *qh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *vh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *lg = (double *)malloc(sizeof(double) * (size_t)nbr * nbr);
        unsigned char *is_sel = (unsigned char *)calloc((size_t)nbr * nbr, 1);
        pool_head(q + xoff, mrow, N, D, qh);
        pool_head(k + xoff, mrow, N, D, kh);
        pool_head(v + xoff, mrow, N, D, vh);
        lowres_logits_head(qh, kh, nbr, D, lg);
        for (long i = 0; i < kk; ++i) {
            int32_t s = sel[(size_t)bh * kk + i];
            if (s < 0 || s >= nbr * nbr) bad = 1;
            else is_sel[s] = 1;
        }
        attend_head(q + xoff, k + xoff, v + xoff, mrow, crow, lg, vh, is_sel, N, D, mode == 0,
                    out + xoff);
        free(qh); free(kh); free(vh); free(lg); free(is_sel);
    }
    free(cnt);
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ backward
 * Gradient of the forward output with respect to q, k and v, with the
 * selected set held fixed (the top-k indices are not differentiated).
 * [MRA page, step three: the sampled-dense products are autograd functions
 * whose backward passes reuse the same kernels through transposed indices, so
 * the model trains end to end; step four: in "sparse" mode the
 * low-resolution branch only chooses blocks, under no_grad, so no gradient
 * flows through it; in "full" mode the low-resolution output is part of the
 * result and its gradient flows through the pooled Q, K and V.]
 *
 * For query i (m_i = 1) with included terms t (as in attend_head), weights
 * p_t = w_t / sum(w), output out_i = sum_t p_t value_t and incoming dout_i,
 * with Dlt_i = dout_i . out_i:
 *   hi term (key j of a selected block):  ds_ij = p_ij (dout_i . v_j - Dlt_i)
 *       dv_j += p_ij dout_i,   dq_i += ds_ij k_j / sqrt(D),   dk_j += ds_ij q_i / sqrt(D)
 *   lo term (unselected block c, full mode):  dl_rc += p_ic (dout_i . vhat_c - Dlt_i)
 *       dvhat_c += p_ic dout_i
 * then dqhat_r += dl_rc khat_c / sqrt(D), dkhat_c += dl_rc qhat_r / sqrt(D), and
 * the block means hand their gradients to their valid tokens:
 *   dx_t += dxhat_b / cnt_b  for m_t = 1, t in block b.
 * A padded query and a row without terms output the constant 0: no gradient. */
static void backward_head(const double *q, const double *k, const double *v,
                          const double *mask_row, const double *cnt_row, const double *qh,
                          const double *kh, const double *vh, const double *logit,
                          const unsigned char *selected, const double *dout, int N, int D,
                          int full_mode, double *dq, double *dk, double *dv)
{
    int nbr = N / MRA_ORACLE_BLOCK;
    double scale = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    double *dl = (double *)calloc((size_t)nbr * nbr, sizeof(double));
    double *dqh = (double *)calloc((size_t)nbr * D, sizeof(double));
    double *dkh = (double *)calloc((size_t)nbr * D, sizeof(double));
    double *dvh = (double *)calloc((size_t)nbr * D, sizeof(double));
    for (size_t e = 0; e < (size_t)N * D; ++e) dq[e] = dk[e] = dv[e] = 0.0;

    for (int i = 0; i < N; ++i) {
        int r = i / MRA_ORACLE_BLOCK;
        if (mask_row && !(mask_row[i] > 0.0)) continue;
        const double *qi = q + (size_t)i * D;
        const double *gi = dout + (size_t)i * D;
        /* the forward terms of query i: exponents, maximum, normaliser, output */
        int any = 0;
        double mx = 0.0;
        for (int c = 0; c < nbr; ++c) {
            if (selected[(size_t)r * nbr + c]) {
                for (int j = c * MRA_ORACLE_BLOCK; j < (c + 1) * MRA_ORACLE_BLOCK; ++j) {
                    if (mask_row && !(mask_row[j] > 0.0)) continue;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += qi[d] * k[(size_t)j * D + d];
                    s[j] = dot * scale;
                    if (!any || s[j] > mx) mx = s[j];
                    any = 1;
                }
            } else if (full_mode && cnt_row[c] > 0.0) {
                double l = logit[(size_t)r * nbr + c];
                if (!any || l > mx) mx = l;
                any = 1;
            }
        }
        if (!any) continue;
        double den = 0.0;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int c = 0; c < nbr; ++c) {
            if (selected[(size_t)r * nbr + c]) {
                for (int j = c * MRA_ORACLE_BLOCK; j < (c + 1) * MRA_ORACLE_BLOCK; ++j) {
                    if (mask_row && !(mask_row[j] > 0.0)) continue;
                    double w = exp(s[j] - mx);
                    den += w;
                    for (int d = 0; d < D; ++d) o[d] += w * v[(size_t)j * D + d];
                }
            } else if (full_mode && cnt_row[c] > 0.0) {
                double w = cnt_row[c] * exp(logit[(size_t)r * nbr + c] - mx);
                den += w;
                for (int d = 0; d < D; ++d) o[d] += w * vh[(size_t)c * D + d];
            }
        }
        double delta = 0.0;
        for (int d = 0; d < D; ++d) {
            o[d] /= den;
            delta += gi[d] * o[d];
        }
        /* the gradients of every term */
        for (int c = 0; c < nbr; ++c) {
            if (selected[(size_t)r * nbr + c]) {
                for (int j = c * MRA_ORACLE_BLOCK; j < (c + 1) * MRA_ORACLE_BLOCK; ++j) {
                    if (mask_row && !(mask_row[j] > 0.0)) continue;
                    double p = exp(s[j] - mx) / den;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += gi[d] * v[(size_t)j * D + d];
                    double ds = p * (dot - delta);
                    for (int d = 0; d < D; ++d) {
                        dv[(size_t)j * D + d] += p * gi[d];
                        dq[(size_t)i * D + d] += ds * scale * k[(size_t)j * D + d];
                        dk[(size_t)j * D + d] += ds * scale * qi[d];
                    }
                }
            } else if (full_mode && cnt_row[c] > 0.0) {
                double p = cnt_row[c] * exp(logit[(size_t)r * nbr + c] - mx) / den;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += gi[d] * vh[(size_t)c * D + d];
                dl[(size_t)r * nbr + c] += p * (dot - delta);
                for (int d = 0; d < D; ++d) dvh[(size_t)c * D + d] += p * gi[d];
            }
        }
    }
    /* low-resolution logits -> block means -> tokens */
    for (int r = 0; r < nbr; ++r)
        for (int c = 0; c < nbr; ++c) {
            double g = dl[(size_t)r * nbr + c];
            if (g == 0.0) continue;
            for (int d = 0; d < D; ++d) {
                dqh[(size_t)r * D + d] += g * scale * kh[(size_t)c * D + d];
                dkh[(size_t)c * D + d] += g * scale * qh[(size_t)r * D + d];
            }
        }
    for (int t = 0; t < N; ++t) {
        int b = t / MRA_ORACLE_BLOCK;
        if (mask_row && !(mask_row[t] > 0.0)) continue;
        if (!(cnt_row[b] > 0.0)) continue;
        for (int d = 0; d < D; ++d) {
            dq[(size_t)t * D + d] += dqh[(size_t)b * D + d] / cnt_row[b];
            dk[(size_t)t * D + d] += dkh[(size_t)b * D + d] / cnt_row[b];
            dv[(size_t)t * D + d] += dvh[(size_t)b * D + d] / cnt_row[b];
        }
    }
    free(s); free(o); free(dl); free(dqh); free(dkh); free(dvh);
}

/* The backward pass: the forward's selection (recomputed exactly as in
 * mra_oracle_forward), then backward_head per (batch, head).
 * q, k, v, dout, dq, dk, dv: [B][H][N][D]; mask: [B][N] of 0/1 or NULL.
 * Returns 0, or -1 on the forward's invalid arguments. */
int mra_oracle_backward(const double *q, const double *k, const double *v, const double *mask,
                        const double *dout, int B, int H, int N, int D, int block_per_row, int mode,
                        int first_n, int diag_n, double *dq, double *dk, double *dv, int nthreads)
{
    if (B < 1 || H < 1 || N < MRA_ORACLE_BLOCK || N % MRA_ORACLE_BLOCK != 0 || D < 1) return -1;
    if (block_per_row < 1 || (mode != 0 && mode != 1)) return -1;
    int nbr = N / MRA_ORACLE_BLOCK;
    if (first_n < 0 || first_n > nbr || diag_n < 0 || diag_n > nbr) return -1;
    long kk = mra_oracle_num_block(N, block_per_row);
    int BH = B * H;
    double *cnt = (double *)malloc(sizeof(double) * (size_t)B * nbr);
    mra_oracle_block_counts(mask, B, N, cnt);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        int b = bh / H;
        size_t xoff = (size_t)bh * N * D;
        const double *mrow = mask ? mask + (size_t)b * N : NULL;
        const double *crow = cnt + (size_t)b * nbr;
        double *qh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *vh = (double *)malloc(sizeof(double) * (size_t)nbr * D);
        double *lg = (double *)malloc(sizeof(double) * (size_t)nbr * nbr);
        double *ml = (double *)malloc(sizeof(double) * (size_t)nbr);
        double *ky = (double *)malloc(sizeof(double) * (size_t)nbr * nbr);
        int32_t *sl = (int32_t *)malloc(sizeof(int32_t) * (size_t)kk);
        unsigned char *is_sel = (unsigned char *)calloc((size_t)nbr * nbr, 1);
        pool_head(q + xoff, mrow, N, D, qh);
        pool_head(k + xoff, mrow, N, D, kh);
        pool_head(v + xoff, mrow, N, D, vh);
        lowres_logits_head(qh, kh, nbr, D, lg);
        row_max_head(lg, crow, nbr, ml);
        selection_keys_head(lg, ml, crow, nbr, first_n, diag_n, ky);
        select_head(ky, nbr, kk, sl);
        for (long i = 0; i < kk; ++i) is_sel[sl[i]] = 1;
        backward_head(q + xoff, k + xoff, v + xoff, mrow, crow, qh, kh, vh, lg, is_sel, dout + xoff, N,
                      D, mode == 0, dq + xoff, dk + xoff, dv + xoff);
        free(qh); free(kh); free(vh); free(lg); free(ml); free(ky); free(sl); free(is_sel);
    }
    free(cnt);
    return 0;
}
