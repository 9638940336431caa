/*
 * BSA forward oracle: a plain, slow, fp64 CPU statement of mesh-aligned
 * block-sparse attention, written step by step from the MOSAIC note
 * ("(Sparse) Attention to the Details", papernotes.org ICML 2026 page,
 * section "Mesh-aligned Block-Sparse Attention (BSA)"):
 *
 *   partition the N NESTED tokens into m contiguous blocks, pool each block
 *   (phi = mean), (a) compressed branch softmax(q̄_i·k̄_j/sqrt(d)) block to
 *   block, broadcast to the tokens of block i, (b) selection branch: each
 *   query block keeps the top-n key blocks by compressed score and runs
 *   full-resolution attention over their tokens, (c) local branch: standard
 *   attention over a sliding window, and o = g_CG o_CG + g_FG o_FG + g_L o_L.
 * The note trains the model through BSA (its loss and training sections), so
 * the file also holds the backward pass of the same forward: the chain rule
 * through each step above in reverse, with the block selection held fixed.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file or its library; only the tests, the package's smoke check
 * and the benchmark's CPU-baseline leg use it. It shares no code with the
 * CUDA library.
 *
 * Readings where the note is silent (each also listed in the design notes):
 *  - phi is the arithmetic mean over the block's tokens.
 *  - o_CG of query block i is sum_j softmax_j(z_ij) * v̄_j (pooled values),
 *    identical for every token of block i.
 *  - one scale s = 1/sqrt(d) (or the caller's) in all three branches.
 *  - top-n ranks the logits z_ij (softmax is monotone); equal logits go to
 *    the lower block index; output order is (z descending, j ascending).
 *  - no causal mask; selected blocks may overlap the local window, the two
 *    branches keep separate softmaxes.
 *  - the local window is block aligned, blocks max(0,i-w) .. min(m-1,i+w),
 *    clamped at the ends of the NESTED sequence (no wrap-around).
 *  - gates are given per token, order (CG, FG, L), not normalised.
 *
 * All arrays are row-major and describe ONE (batch, head) slab:
 *   q, k, v [N][d], gates [N][3], pooled [m][d], idx [m][n] (int32).
 * Functions return 0 on success, -1 on bad arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- step 1-2: block partition and pooling phi (mean) ------------------ */

/* xbar[j][c] = (1/B) * sum over the B tokens of block j of x[t][c];
 * block j holds tokens j*B .. j*B+B-1 (one parent pixel in NESTED order). */
int oracle_pool(int64_t n_tokens, int64_t d, int64_t block,
                const double *x, double *xbar)
{
    if (n_tokens <= 0 || d <= 0 || block <= 0 || n_tokens % block != 0) return -1;
    int64_t m = n_tokens / block;
    for (int64_t j = 0; j < m; ++j) {
        for (int64_t c = 0; c < d; ++c) {
            double s = 0.0;
            for (int64_t t = j * block; t < (j + 1) * block; ++t) s += x[t * d + c];
            xbar[j * d + c] = s / (double)block;
        }
    }
    return 0;
}

/* ---- step 3-4: compressed branch and top-n selection ------------------- */

typedef struct { double z; int32_t j; } scored_block;

/* Sort key (-z, j): larger logit first, equal logits by lower block index. */
static int by_score_then_index(const void *pa, const void *pb)
{
    const scored_block *a = (const scored_block *)pa, *b = (const scored_block *)pb;
    if (a->z > b->z) return -1;
    if (a->z < b->z) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

/*
 * For query blocks i in [r0, r1):
 *   z_ij    = s * sum_c q̄_ic k̄_jc                     (j = 0 .. m-1)
 *   ā_ij    = exp(z_ij - max_j z_ij) / sum_j exp(...)
 *   o_cg_i  = sum_j ā_ij v̄_j
 *   idx_i   = the n blocks first in the order (z desc, j asc)
 *   gap_i   = z_(n) - z_(n+1) in that order, +inf when n == m
 * Output rows are relative to r0. z_out (nullable) receives the logits.
 */
int oracle_compressed_rows(int64_t m, int64_t d, int64_t n, double scale,
                           const double *qbar, const double *kbar, const double *vbar,
                           int64_t r0, int64_t r1,
                           double *o_cg, int32_t *idx, double *gap, double *z_out)
{
    if (m <= 0 || d <= 0 || n < 1 || n > m || r0 < 0 || r1 > m || r0 > r1) return -1;
    int64_t rows = r1 - r0;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t i = r0 + r;
        scored_block *sb = (scored_block *)malloc((size_t)m * sizeof(scored_block));
        double *w = (double *)malloc((size_t)m * sizeof(double));
        if (!sb || !w) { free(sb); free(w); bad = 1; continue; }
        double zmax = -INFINITY;
        for (int64_t j = 0; j < m; ++j) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qbar[i * d + c] * kbar[j * d + c];
            double z = scale * dot;
            sb[j].z = z;
            sb[j].j = (int32_t)j;
            if (z_out) z_out[r * m + j] = z;
            if (z > zmax) zmax = z;
        }
        double denom = 0.0;
        for (int64_t j = 0; j < m; ++j) { w[j] = exp(sb[j].z - zmax); denom += w[j]; }
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < m; ++j) acc += w[j] * vbar[j * d + c];
            o_cg[r * d + c] = acc / denom;
        }
        qsort(sb, (size_t)m, sizeof(scored_block), by_score_then_index);
        for (int64_t t = 0; t < n; ++t) idx[r * n + t] = sb[t].j;
        gap[r] = (n < m) ? sb[n - 1].z - sb[n].z : INFINITY;
        free(sb);
        free(w);
    }
    return bad ? -1 : 0;
}

/* ---- step 5-7: selection branch, local branch, gated combine ----------- */

/* Softmax attention of one query row over the tokens of the listed blocks:
 * out[c] = sum_u p_u v_uc, p_u = softmax_u(s * q·k_u). */
static void attend_blocks(int64_t d, int64_t block, double scale, const double *qt,
                          const double *k, const double *v,
                          const int64_t *blocks, int64_t nb, double *scores, double *out)
{
    int64_t nk = nb * block;
    double smax = -INFINITY;
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t t = 0; t < block; ++t) {
            int64_t u = blocks[b] * block + t;
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qt[c] * k[u * d + c];
            double s = scale * dot;
            scores[b * block + t] = s;
            if (s > smax) smax = s;
        }
    }
    double denom = 0.0;
    for (int64_t e = 0; e < nk; ++e) { scores[e] = exp(scores[e] - smax); denom += scores[e]; }
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t t = 0; t < block; ++t) {
            int64_t u = blocks[b] * block + t;
            double p = scores[b * block + t] / denom;
            for (int64_t c = 0; c < d; ++c) out[c] += p * v[u * d + c];
        }
    }
}

/*
 * For query blocks i in [qb0, qb1) and every token t of block i:
 *   o_fg_t = attention over the tokens of blocks idx[i][0..n-1]
 *   o_l_t  = attention over the tokens of blocks max(0,i-w) .. min(m-1,i+w)
 *   out_t  = g_t0 * o_cg[i] + g_t1 * o_fg_t + g_t2 * o_l_t
 * o_cg is the block-level compressed output [m][d]; idx is [m][n] with
 * entries in [0, m). Output rows are relative to token qb0*block.
 * o_fg_out / o_l_out are nullable.
 */
int oracle_fine_rows(int64_t n_tokens, int64_t d, int64_t block, int64_t n, int64_t w,
                     double scale, const double *q, const double *k, const double *v,
                     const double *gates, const double *o_cg, const int32_t *idx,
                     int64_t qb0, int64_t qb1,
                     double *out, double *o_fg_out, double *o_l_out)
{
    if (n_tokens <= 0 || d <= 0 || block <= 0 || n_tokens % block != 0) return -1;
    int64_t m = n_tokens / block;
    if (n < 1 || n > m || w < 0 || qb0 < 0 || qb1 > m || qb0 > qb1) return -1;
    for (int64_t i = qb0; i < qb1; ++i)
        for (int64_t t = 0; t < n; ++t)
            if (idx[i * n + t] < 0 || idx[i * n + t] >= m) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = qb0; i < qb1; ++i) {
        int64_t lo = (i - w < 0) ? 0 : i - w;
        int64_t hi = (i + w > m - 1) ? m - 1 : i + w;
        int64_t nl = hi - lo + 1;
        int64_t nmax = (n > nl) ? n : nl;
        int64_t *sel = (int64_t *)malloc((size_t)n * sizeof(int64_t));
        int64_t *loc = (int64_t *)malloc((size_t)nl * sizeof(int64_t));
        double *scores = (double *)malloc((size_t)(nmax * block) * sizeof(double));
        double *ofg = (double *)malloc((size_t)d * sizeof(double));
        double *ol = (double *)malloc((size_t)d * sizeof(double));
        if (!sel || !loc || !scores || !ofg || !ol) {
            free(sel); free(loc); free(scores); free(ofg); free(ol); bad = 1; continue;
        }
        for (int64_t t = 0; t < n; ++t) sel[t] = idx[i * n + t];
        for (int64_t b = 0; b < nl; ++b) loc[b] = lo + b;
        for (int64_t t = i * block; t < (i + 1) * block; ++t) {
            const double *qt = q + t * d;
            attend_blocks(d, block, scale, qt, k, v, sel, n, scores, ofg);
            attend_blocks(d, block, scale, qt, k, v, loc, nl, scores, ol);
            int64_t r = t - qb0 * block;
            const double *g = gates + t * 3;
            for (int64_t c = 0; c < d; ++c) {
                out[r * d + c] = g[0] * o_cg[i * d + c] + g[1] * ofg[c] + g[2] * ol[c];
                if (o_fg_out) o_fg_out[r * d + c] = ofg[c];
                if (o_l_out) o_l_out[r * d + c] = ol[c];
            }
        }
        free(sel); free(loc); free(scores); free(ofg); free(ol);
    }
    return bad ? -1 : 0;
}

/*
 * The whole forward pass of one slab, steps 1-7 in order. When forced_idx is
 * non-null the selection branch uses it instead of the computed top-n (the
 * computed indices and gaps are still returned), so that a caller can
 * re-evaluate outputs on another implementation's near-tie choices.
 * Outputs: out [N][d]; nullable extras: qbar/kbar/vbar [m][d], o_cg [m][d],
 * idx [m][n], gap [m].
 */
int oracle_forward_slab(int64_t n_tokens, int64_t d, int64_t block, int64_t n, int64_t w,
                        double scale, const double *q, const double *k, const double *v,
                        const double *gates, const int32_t *forced_idx,
                        double *out, double *qbar_out, double *kbar_out, double *vbar_out,
                        double *o_cg_out, int32_t *idx_out, double *gap_out)
{
    if (n_tokens <= 0 || d <= 0 || block <= 0 || n_tokens % block != 0) return -1;
    int64_t m = n_tokens / block;
    if (n < 1 || n > m) return -1;
    double *qb = (double *)malloc((size_t)(m * d) * sizeof(double));
    double *kb = (double *)malloc((size_t)(m * d) * sizeof(double));
    double *vb = (double *)malloc((size_t)(m * d) * sizeof(double));
    double *ocg = (double *)malloc((size_t)(m * d) * sizeof(double));
    int32_t *ix = (int32_t *)malloc((size_t)(m * n) * sizeof(int32_t));
    double *gp = (double *)malloc((size_t)m * sizeof(double));
    int rc = -1;
    if (qb && kb && vb && ocg && ix && gp &&
        oracle_pool(n_tokens, d, block, q, qb) == 0 &&
        oracle_pool(n_tokens, d, block, k, kb) == 0 &&
        oracle_pool(n_tokens, d, block, v, vb) == 0 &&
        oracle_compressed_rows(m, d, n, scale, qb, kb, vb, 0, m, ocg, ix, gp, NULL) == 0 &&
        oracle_fine_rows(n_tokens, d, block, n, w, scale, q, k, v, gates, ocg,
                         forced_idx ? forced_idx : ix, 0, m, out, NULL, NULL) == 0) {
        rc = 0;
        if (qbar_out) memcpy(qbar_out, qb, (size_t)(m * d) * sizeof(double));
        if (kbar_out) memcpy(kbar_out, kb, (size_t)(m * d) * sizeof(double));
        if (vbar_out) memcpy(vbar_out, vb, (size_t)(m * d) * sizeof(double));
        if (o_cg_out) memcpy(o_cg_out, ocg, (size_t)(m * d) * sizeof(double));
        if (idx_out) memcpy(idx_out, ix, (size_t)(m * n) * sizeof(int32_t));
        if (gap_out) memcpy(gap_out, gp, (size_t)m * sizeof(double));
    }
    free(qb); free(kb); free(vb); free(ocg); free(ix); free(gp);
    return rc;
}

/* ---- backward pass (training) -------------------------------------------- */

/* Gradient of one softmax-attention row over the listed blocks (the reverse
 * of attend_blocks): with p_u = softmax_u(s q·k_u) and the gradient dO that
 * reaches this row's output o = sum_u p_u v_u,
 *   dv_u += p_u dO,   dp_u = dO·v_u,   D = sum_u p_u dp_u,
 *   ds_u  = p_u (dp_u - D),
 *   dq_t += s sum_u ds_u k_u,   dk_u += s ds_u q_t.
 * p and dp are scratch arrays of nb*block doubles. */
static void attend_blocks_backward(int64_t d, int64_t block, double scale, const double *qt,
                                   const double *k, const double *v, const int64_t *blocks, int64_t nb,
                                   const double *dO, double *p, double *dp,
                                   double *dq_t, double *dk, double *dv)
{
    int64_t nk = nb * block;
    double smax = -INFINITY;
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t t = 0; t < block; ++t) {
            int64_t u = blocks[b] * block + t;
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qt[c] * k[u * d + c];
            p[b * block + t] = scale * dot;
            if (p[b * block + t] > smax) smax = p[b * block + t];
        }
    }
    double denom = 0.0;
    for (int64_t e = 0; e < nk; ++e) { p[e] = exp(p[e] - smax); denom += p[e]; }
    for (int64_t e = 0; e < nk; ++e) p[e] /= denom;
    double D = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t t = 0; t < block; ++t) {
            int64_t u = blocks[b] * block + t, e = b * block + t;
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += dO[c] * v[u * d + c];
            dp[e] = dot;
            D += p[e] * dot;
        }
    }
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t t = 0; t < block; ++t) {
            int64_t u = blocks[b] * block + t, e = b * block + t;
            double ds = p[e] * (dp[e] - D);
            for (int64_t c = 0; c < d; ++c) {
                dq_t[c] += scale * ds * k[u * d + c];
                dk[u * d + c] += scale * ds * qt[c];
                dv[u * d + c] += p[e] * dO[c];
            }
        }
    }
}

/*
 * Backward of one slab: given dout = dL/dout [N][d], the gradients dL/dq,
 * dL/dk, dL/dv [N][d] and dL/dgates [N][3] of the forward pass, with the block
 * selection idx [m][n] held fixed (the top-n choice is a discrete decision and
 * carries no gradient). The chain rule through the forward steps in reverse:
 *   (7) combine: dgates_t = (dout_t·o_CG_i, dout_t·o_FG_t, dout_t·o_L_t); the
 *       selection and local branches receive g_FG,t dout_t and g_L,t dout_t;
 *   (5, 6) the selection and local attention rows (attend_blocks_backward);
 *   (3) compressed branch: dO_CG_i = sum over the tokens t of block i of
 *       g_CG,t dout_t; with ā_ij = softmax_j(z_ij), dā_ij = dO_CG_i·v̄_j,
 *       D_i = sum_j ā_ij dā_ij and dz_ij = ā_ij (dā_ij - D_i):
 *       dq̄_i = s sum_j dz_ij k̄_j,  dk̄_j += s dz_ij q̄_i,  dv̄_j += ā_ij dO_CG_i;
 *   (2) pooling φ (mean): every token of block j receives 1/B of dq̄_j, dk̄_j, dv̄_j.
 * A query block whose dout rows are all zero contributes exact zeros to every
 * sum, so it is skipped. Query blocks run in parallel threads; their sums into
 * dk, dv, dk̄ and dv̄ go to per-thread copies that are added up at the end.
 */
int oracle_backward_slab(int64_t n_tokens, int64_t d, int64_t block, int64_t n, int64_t w,
                         double scale, const double *q, const double *k, const double *v,
                         const double *gates, const int32_t *idx, const double *dout,
                         double *dq, double *dk, double *dv, double *dgates)
{
    if (n_tokens <= 0 || d <= 0 || block <= 0 || n_tokens % block != 0) return -1;
    int64_t m = n_tokens / block;
    if (n < 1 || n > m || w < 0) return -1;
    for (int64_t i = 0; i < m * n; ++i)
        if (idx[i] < 0 || idx[i] >= m) return -1;
    int64_t nl_max = 2 * w + 1 < m ? 2 * w + 1 : m;
    int64_t nmax = (n > nl_max) ? n : nl_max;
    double *qb = (double *)calloc((size_t)(m * d), sizeof(double));
    double *kb = (double *)calloc((size_t)(m * d), sizeof(double));
    double *vb = (double *)calloc((size_t)(m * d), sizeof(double));
    double *dqb = (double *)calloc((size_t)(m * d), sizeof(double));
    double *dkb = (double *)calloc((size_t)(m * d), sizeof(double));
    double *dvb = (double *)calloc((size_t)(m * d), sizeof(double));
    int bad = 0;
    if (!qb || !kb || !vb || !dqb || !dkb || !dvb ||
        oracle_pool(n_tokens, d, block, q, qb) != 0 || oracle_pool(n_tokens, d, block, k, kb) != 0 ||
        oracle_pool(n_tokens, d, block, v, vb) != 0) {
        bad = 1;
        goto done;
    }
    memset(dq, 0, (size_t)(n_tokens * d) * sizeof(double));
    memset(dk, 0, (size_t)(n_tokens * d) * sizeof(double));
    memset(dv, 0, (size_t)(n_tokens * d) * sizeof(double));
    memset(dgates, 0, (size_t)(n_tokens * 3) * sizeof(double));
    /* Query blocks are independent except for their sums into dk, dv, dk̄, dv̄:
     * each thread sums into private copies, added together at the end. The
     * private copies are capped at about 2 GB in all (fewer threads if needed). */
    int nt = 1;
#ifdef _OPENMP
    nt = omp_get_max_threads();
#endif
    {
        double per = (double)(2 * n_tokens * d + 2 * m * d) * sizeof(double);
        int cap = (int)(2e9 / per);
        if (cap < 1) cap = 1;
        if (nt > cap) nt = cap;
    }
#pragma omp parallel num_threads(nt)
    {
        double *dk_p = (double *)calloc((size_t)(n_tokens * d), sizeof(double));
        double *dv_p = (double *)calloc((size_t)(n_tokens * d), sizeof(double));
        double *dkb_p = (double *)calloc((size_t)(m * d), sizeof(double));
        double *dvb_p = (double *)calloc((size_t)(m * d), sizeof(double));
        double *a = (double *)malloc((size_t)m * sizeof(double));
        double *da = (double *)malloc((size_t)m * sizeof(double));
        double *ocg = (double *)malloc((size_t)d * sizeof(double));
        double *docg = (double *)malloc((size_t)d * sizeof(double));
        double *ofg = (double *)malloc((size_t)d * sizeof(double));
        double *ol = (double *)malloc((size_t)d * sizeof(double));
        double *dO = (double *)malloc((size_t)d * sizeof(double));
        double *p = (double *)malloc((size_t)(nmax * block) * sizeof(double));
        double *dp = (double *)malloc((size_t)(nmax * block) * sizeof(double));
        int64_t *sel = (int64_t *)malloc((size_t)n * sizeof(int64_t));
        int64_t *loc = (int64_t *)malloc((size_t)nl_max * sizeof(int64_t));
        int mine_ok = dk_p && dv_p && dkb_p && dvb_p && a && da && ocg && docg && ofg && ol && dO && p && dp &&
                      sel && loc;
        if (!mine_ok) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < m; ++i) {
            if (!mine_ok) continue;
            int any = 0;
            for (int64_t e = i * block * d; e < (i + 1) * block * d; ++e)
                if (dout[e] != 0.0) { any = 1; break; }
            if (!any) continue;
            /* (3) compressed branch, row i: forward probabilities, then its gradients */
            double zmax = -INFINITY;
            for (int64_t j = 0; j < m; ++j) {
                double dot = 0.0;
                for (int64_t c = 0; c < d; ++c) dot += qb[i * d + c] * kb[j * d + c];
                a[j] = scale * dot;
                if (a[j] > zmax) zmax = a[j];
            }
            double denom = 0.0;
            for (int64_t j = 0; j < m; ++j) { a[j] = exp(a[j] - zmax); denom += a[j]; }
            for (int64_t j = 0; j < m; ++j) a[j] /= denom;
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < m; ++j) acc += a[j] * vb[j * d + c];
                ocg[c] = acc;
                double g = 0.0;
                for (int64_t t = i * block; t < (i + 1) * block; ++t) g += gates[t * 3] * dout[t * d + c];
                docg[c] = g;
            }
            double D = 0.0;
            for (int64_t j = 0; j < m; ++j) {
                double dot = 0.0;
                for (int64_t c = 0; c < d; ++c) dot += docg[c] * vb[j * d + c];
                da[j] = dot;
                D += a[j] * dot;
            }
            for (int64_t j = 0; j < m; ++j) {
                double dz = a[j] * (da[j] - D);
                for (int64_t c = 0; c < d; ++c) {
                    dqb[i * d + c] += scale * dz * kb[j * d + c];
                    dkb_p[j * d + c] += scale * dz * qb[i * d + c];
                    dvb_p[j * d + c] += a[j] * docg[c];
                }
            }
            /* (5)-(7) the tokens of block i: combine, selection and local branches
             * (local window: blocks max(0, i-w) .. min(m-1, i+w)) */
            int64_t lo = i - w, hi = i + w;
            if (lo < 0) lo = 0;
            if (hi > m - 1) hi = m - 1;
            int64_t nl = hi - lo + 1;
            for (int64_t t = 0; t < n; ++t) sel[t] = (int64_t)idx[i * n + t];
            for (int64_t b = 0; b < nl; ++b) loc[b] = lo + b;
            for (int64_t t = i * block; t < (i + 1) * block; ++t) {
                const double *qt = q + t * d, *g = gates + t * 3, *dy = dout + t * d;
                attend_blocks(d, block, scale, qt, k, v, sel, n, p, ofg);
                attend_blocks(d, block, scale, qt, k, v, loc, nl, p, ol);
                double s0 = 0.0, s1 = 0.0, s2 = 0.0;
                for (int64_t c = 0; c < d; ++c) { s0 += dy[c] * ocg[c]; s1 += dy[c] * ofg[c]; s2 += dy[c] * ol[c]; }
                dgates[t * 3] = s0;
                dgates[t * 3 + 1] = s1;
                dgates[t * 3 + 2] = s2;
                for (int64_t c = 0; c < d; ++c) dO[c] = g[1] * dy[c];
                attend_blocks_backward(d, block, scale, qt, k, v, sel, n, dO, p, dp, dq + t * d, dk_p, dv_p);
                for (int64_t c = 0; c < d; ++c) dO[c] = g[2] * dy[c];
                attend_blocks_backward(d, block, scale, qt, k, v, loc, nl, dO, p, dp, dq + t * d, dk_p, dv_p);
            }
        }
#pragma omp critical
        {
            if (mine_ok) {
                for (int64_t e = 0; e < n_tokens * d; ++e) { dk[e] += dk_p[e]; dv[e] += dv_p[e]; }
                for (int64_t e = 0; e < m * d; ++e) { dkb[e] += dkb_p[e]; dvb[e] += dvb_p[e]; }
            }
        }
        free(dk_p); free(dv_p); free(dkb_p); free(dvb_p); free(a); free(da); free(ocg); free(docg);
        free(ofg); free(ol); free(dO); free(p); free(dp); free(sel); free(loc);
    }
    if (bad) goto done;
    /* (2) pooling: the mean hands 1/B of each pooled gradient to every token of its block */
    for (int64_t t = 0; t < n_tokens; ++t) {
        int64_t j = t / block;
        for (int64_t c = 0; c < d; ++c) {
            dq[t * d + c] += dqb[j * d + c] / (double)block;
            dk[t * d + c] += dkb[j * d + c] / (double)block;
            dv[t * d + c] += dvb[j * d + c] / (double)block;
        }
    }
done:
    free(qb); free(kb); free(vb); free(dqb); free(dkb); free(dvb);
    return bad ? -1 : 0;
}

/* ---- lat-lon -> HEALPix cross-attention interpolation ------------------ */
/*
 * The step before BSA in the note's pipeline ("overall framework" (1) and the
 * HEALPix paragraph): every HEALPix target pixel i attends to its neighbouring
 * source points j of a latitude-longitude grid, with the relative position
 * p_ij as the query and the source features as keys and values:
 *   o_i = sum_{j in N_i} softmax_j(q_ij . k_j / sqrt(d)) v_j.
 * Readings where the note is silent (also listed in the design notes):
 *  - HEALPix pixel centres follow the published HEALPix definition (Gorski et
 *    al. 2005): 4*Nside-1 iso-latitude rings; ring i (from the north) has
 *    4i pixels at z = 1 - i^2/(3 Nside^2), phi = (j - 1/2) pi/(2i) in the
 *    polar caps (i < Nside, mirrored in the south), and 4 Nside pixels at
 *    z = 4/3 - 2i/(3 Nside), phi = (j - s/2) pi/(2 Nside), s = (i - Nside + 1)
 *    mod 2, in the equatorial belt. In NESTED order pixel p lies in base face
 *    f = p / Nside^2, and the bits of p mod Nside^2 interleave the face
 *    coordinates (x in the even bits, y in the odd ones), which makes the
 *    children of p the pixels 4p .. 4p+3.
 *  - the source grid has nlat rows from +90 to -90 degrees (poles included)
 *    and nlon columns from 0 degrees eastwards; N_i is the 4 x 4 block of grid
 *    points around the target: rows r0 .. r0+3 with r0 = floor(u) - 1 clamped
 *    to [0, nlat-4], u = (90 - lat)/dlat, and columns c0-1 .. c0+2 (wrapping
 *    in longitude), c0 = floor(lon/dlon);
 *  - p_ij = (x_j - x_i) / h, the difference of the unit vectors divided by
 *    the grid's angular step h = dlat in radians, and q_ij = W_q p_ij with a
 *    given matrix W_q [d][3]; k_j, v_j are the given source features.
 */

static const double kPi = 3.14159265358979323846;

/* Centre of NESTED pixel p at resolution nside: z = cos(colatitude), phi in [0, 2 pi).
 * Face f spans rings face_row[f]*nside - 2 nside + 1 .. face_row[f]*nside - 1;
 * its pixel (x, y) sits on ring face_row[f]*nside - x - y - 1, and (x - y)
 * counts half pixel steps of azimuth (pi / (4 nr), nr = the ring's pixels / 4)
 * from the face's central meridian at face_col[f] * pi/4. */
void oracle_healpix_center(int64_t nside, int64_t p, double *z, double *phi)
{
    static const int face_row[12] = {2, 2, 2, 2, 3, 3, 3, 3, 4, 4, 4, 4};
    static const int face_col[12] = {1, 3, 5, 7, 0, 2, 4, 6, 1, 3, 5, 7};
    int64_t per_face = nside * nside;
    int64_t f = p / per_face, ipf = p % per_face;
    int64_t x = 0, y = 0;
    for (int b = 0; ((int64_t)1 << (2 * b)) < per_face; ++b) {     /* de-interleave the Morton bits */
        x |= ((ipf >> (2 * b)) & 1) << b;
        y |= ((ipf >> (2 * b + 1)) & 1) << b;
    }
    int64_t ring = face_row[f] * nside - x - y - 1;                 /* 1 .. 4 nside - 1 from the north */
    int64_t nr;
    if (ring < nside) {                                              /* north polar cap */
        nr = ring;
        *z = 1.0 - (double)(nr * nr) / (3.0 * (double)per_face);
    } else if (ring > 3 * nside) {                                   /* south polar cap */
        nr = 4 * nside - ring;
        *z = -1.0 + (double)(nr * nr) / (3.0 * (double)per_face);
    } else {                                                         /* equatorial belt */
        nr = nside;
        *z = 4.0 / 3.0 - 2.0 * (double)ring / (3.0 * (double)nside);
    }
    double ph = (double)(face_col[f] * nr + (x - y)) * (kPi / 4.0) / (double)nr;
    if (ph < 0.0) ph += 2.0 * kPi;
    if (ph >= 2.0 * kPi) ph -= 2.0 * kPi;
    *phi = ph;
}

/* Neighbourhoods and relative positions of every pixel of a HEALPix grid over
 * an nlat x nlon lat-lon grid: nbr [npix][16] (source index r*nlon + c), rel
 * [npix][16][3]. Returns -1 on bad sizes. */
int oracle_latlon_plan(int64_t nside, int64_t nlat, int64_t nlon, int32_t *nbr, double *rel)
{
    if (nside < 1 || nlat < 4 || nlon < 4) return -1;
    int64_t npix = 12 * nside * nside;
    double dlat = 180.0 / (double)(nlat - 1), dlon = 360.0 / (double)nlon;
    double h = dlat * kPi / 180.0;
    for (int64_t i = 0; i < npix; ++i) {
        double z, phi;
        oracle_healpix_center(nside, i, &z, &phi);
        double lat = asin(z) * 180.0 / kPi, lon = phi * 180.0 / kPi;
        double st = sqrt(1.0 - z * z);
        double xi[3] = {st * cos(phi), st * sin(phi), z};
        int64_t r0 = (int64_t)floor((90.0 - lat) / dlat) - 1;
        if (r0 < 0) r0 = 0;
        if (r0 > nlat - 4) r0 = nlat - 4;
        int64_t c0 = (int64_t)floor(lon / dlon);
        for (int64_t a = 0; a < 4; ++a) {
            for (int64_t b = 0; b < 4; ++b) {
                int64_t r = r0 + a, c = ((c0 - 1 + b) % nlon + nlon) % nlon;
                int64_t e = i * 16 + a * 4 + b;
                nbr[e] = (int32_t)(r * nlon + c);
                double la = (90.0 - (double)r * dlat) * kPi / 180.0, lo = (double)c * dlon * kPi / 180.0;
                double xj[3] = {cos(la) * cos(lo), cos(la) * sin(lo), sin(la)};
                for (int t = 0; t < 3; ++t) rel[e * 3 + t] = (xj[t] - xi[t]) / h;
            }
        }
    }
    return 0;
}

/* o_i = sum_j softmax_j(scale * (W_q p_ij) . k_{nbr_ij}) v_{nbr_ij} for i < n_tgt,
 * with K neighbours each: nbr [n_tgt][K], rel [n_tgt][K][3], wq [d][3],
 * ksrc, vsrc [n_src][d], out [n_tgt][d]. */
int oracle_interp(int64_t n_tgt, int64_t K, int64_t d, int64_t n_src, double scale, const int32_t *nbr,
                  const double *rel, const double *wq, const double *ksrc, const double *vsrc, double *out)
{
    if (n_tgt < 0 || K < 1 || d < 1 || n_src < 1) return -1;
    for (int64_t e = 0; e < n_tgt * K; ++e)
        if (nbr[e] < 0 || nbr[e] >= n_src) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_tgt; ++i) {
        double *s = (double *)malloc((size_t)K * sizeof(double));
        if (!s) { bad = 1; continue; }
        double smax = -INFINITY;
        for (int64_t j = 0; j < K; ++j) {
            const double *p = rel + (i * K + j) * 3, *kj = ksrc + (int64_t)nbr[i * K + j] * d;
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) {
                double qc = wq[c * 3] * p[0] + wq[c * 3 + 1] * p[1] + wq[c * 3 + 2] * p[2];
                dot += qc * kj[c];
            }
            s[j] = scale * dot;
            if (s[j] > smax) smax = s[j];
        }
        double denom = 0.0;
        for (int64_t j = 0; j < K; ++j) { s[j] = exp(s[j] - smax); denom += s[j]; }
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j) acc += s[j] * vsrc[(int64_t)nbr[i * K + j] * d + c];
            out[i * d + c] = acc / denom;
        }
        free(s);
    }
    return bad ? -1 : 0;
}
