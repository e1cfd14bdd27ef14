/*
 * Float64 CPU oracle for fused softmax cross-entropy.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. The CUDA product
 * path never calls it and shares no code, header, helper or constant with it.
 *
 * It is a plain, slow, obviously correct restatement of what the method
 * computes, written from the pages:
 *   - "Shift by the max in cross_entropy" (MLX PR #4188, Proposed changes):
 *     the loss only depends on the gaps between logits, so it is assembled
 *     from values shifted by the row max m; the label-smoothing term
 *     subtracts the mean logit and is invariant to the shift.
 *   - "A fused linear cross-entropy forward kernel for Apple GPUs" (Ineshin),
 *     section 1 "Streaming the loss without full logits": Z = H W^T,
 *     loss_i = logsumexp(Z_i) - Z_{i,y_i}, logsumexp = m + log(s).
 *   - MLX issue #4686 (the fast.cross_entropy VJP): the gradient of the summed
 *     loss with respect to the logits, softmax minus one-hot, scaled by g_i.
 *
 * Everything is computed in double from inputs upcast exactly to double.
 * Sums run left to right over the vocabulary in index order. OpenMP only
 * splits independent rows (or independent output entries) across threads;
 * nothing inside a row is reordered or blocked.
 *
 * Readings taken where the pages are silent (each repeated at its function):
 *   - ignore_index: a row whose target equals ignore_index has loss 0 and a
 *     zero gradient row; its lse is still computed.
 *   - a target outside [0, V) that is not ignore_index: loss NaN, gradient
 *     row NaN.
 *   - label smoothing eps spreads eps/V over all V classes, the target
 *     included: loss = (1-eps)(lse - z_y) + eps(lse - mean_j z_j).
 *   - a NaN anywhere in the row: m, lse and loss are NaN; argmax is the index
 *     of the first NaN.
 *   - a row whose entries are all -inf: lse = -inf (the log of an empty sum),
 *     loss NaN, gradient row NaN.
 *   - a -inf entry in a row with a finite max contributes exp(-inf) = 0 to
 *     the sum; as the target it makes the loss +inf; with eps > 0 it makes the
 *     mean -inf and the loss +inf. At eps = 0 the smoothing term is absent.
 *   - argmax is the lowest index attaining the row max.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One row of the forward. Returns through the pointers; m_out and s_out give
 * the row max and the sum of exp(z_j - m) for callers that need them. */
static void row_forward(const double* z, int64_t V, int64_t y, double eps,
                        int64_t ignore_index, double* loss, double* lse,
                        int64_t* argmax, double* m_out, double* s_out)
{
    /* Step 1: row max m, first index attaining it; a NaN wins at its first
     * occurrence. */
    double m = -INFINITY;
    int64_t am = 0;
    int has_nan = 0;
    for (int64_t j = 0; j < V; ++j) {
        double v = z[j];
        if (isnan(v)) { m = NAN; am = j; has_nan = 1; break; }
        if (v > m) { m = v; am = j; }
    }
    if (argmax) *argmax = am;

    if (has_nan) {
        *lse = NAN;
        *loss = (y == ignore_index) ? 0.0 : NAN;
        *m_out = NAN; *s_out = NAN;
        return;
    }
    if (m == -INFINITY) {
        /* every entry is -inf: the sum of exponentials is empty */
        *lse = -INFINITY;
        *loss = (y == ignore_index) ? 0.0 : NAN;
        *m_out = m; *s_out = 0.0;
        return;
    }

    /* Step 2: s = sum_j exp(z_j - m); lse = m + log s (Ineshin section 1). */
    double s = 0.0;
    for (int64_t j = 0; j < V; ++j) s += exp(z[j] - m);
    *lse = m + log(s);
    *m_out = m; *s_out = s;

    /* Step 3: loss assembled from shifted values (MLX PR #4188):
     *   loss = log s - (1-eps)(z_y - m) - eps (mean_j z_j - m). */
    if (y == ignore_index) { *loss = 0.0; return; }
    if (y < 0 || y >= V) { *loss = NAN; return; }
    double l = log(s) - (1.0 - eps) * (z[y] - m);
    if (eps != 0.0) {
        double shifted_sum = 0.0;
        for (int64_t j = 0; j < V; ++j) shifted_sum += (z[j] - m);
        l -= eps * (shifted_sum / (double)V);
    }
    *loss = l;
}

/* Row cross-entropy forward over a contiguous (N, V) matrix of doubles.
 * loss, lse: N doubles. argmax: N int64 or NULL. */
void orc_ce_forward(const double* z, int64_t N, int64_t V, const int64_t* y,
                    double eps, int64_t ignore_index,
                    double* loss, double* lse, int64_t* argmax)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        double m, s;
        row_forward(z + i * V, V, y[i], eps, ignore_index, &loss[i], &lse[i],
                    argmax ? &argmax[i] : NULL, &m, &s);
    }
}

/* Gradient of sum_i g_i loss_i with respect to one row of logits:
 *   dz_j = g (exp(z_j - m)/s - (1-eps)[j = y] - eps/V). */
static void row_backward(const double* z, int64_t V, int64_t y, double g,
                         double eps, int64_t ignore_index, double* dz)
{
    if (y == ignore_index) {
        for (int64_t j = 0; j < V; ++j) dz[j] = 0.0;
        return;
    }
    double loss, lse, m, s;
    int64_t am;
    row_forward(z, V, y, eps, ignore_index, &loss, &lse, &am, &m, &s);
    if (y < 0 || y >= V || isnan(m) || m == -INFINITY) {
        for (int64_t j = 0; j < V; ++j) dz[j] = NAN;
        return;
    }
    for (int64_t j = 0; j < V; ++j) {
        double p = exp(z[j] - m) / s;
        double onehot = (j == y) ? 1.0 : 0.0;
        dz[j] = g * (p - (1.0 - eps) * onehot - eps / (double)V);
    }
}

/* Row cross-entropy VJP. g: N per-row upstream gradients. dz: N*V doubles. */
void orc_ce_backward(const double* z, int64_t N, int64_t V, const int64_t* y,
                     const double* g, double eps, int64_t ignore_index,
                     double* dz)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        row_backward(z + i * V, V, y[i], g[i], eps, ignore_index, dz + i * V);
}

/* One row of logits of the linear head: Z_ij = sum_d H_id W_jd, in double,
 * d in order (Ineshin section 1, Z = H W^T). H, W hold bf16 values widened
 * exactly to float. */
static void linear_row(const float* h, const float* W, int64_t V, int64_t D,
                       double* zrow)
{
    for (int64_t j = 0; j < V; ++j) {
        const float* w = W + j * D;
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += (double)h[d] * (double)w[d];
        zrow[j] = acc;
    }
}

/* Fused-linear forward, computed the unfused way: each row of Z = H W^T in
 * double, then the row definition above. Works on any subset of rows: rows
 * lists the row indices to compute (nrows of them); loss/lse are indexed by
 * position in that list. */
void orc_linear_ce_forward_rows(const float* H, const float* W, int64_t V,
                                int64_t D, const int64_t* rows, int64_t nrows,
                                const int64_t* y, double eps,
                                int64_t ignore_index, double* loss, double* lse)
{
    #pragma omp parallel
    {
        double* zrow = (double*)malloc((size_t)V * sizeof(double));
        #pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < nrows; ++k) {
            int64_t i = rows[k];
            double m, s;
            int64_t am;
            linear_row(H + i * D, W, V, D, zrow);
            row_forward(zrow, V, y[i], eps, ignore_index, &loss[k], &lse[k],
                        &am, &m, &s);
        }
        free(zrow);
    }
}

/* Fused-linear backward for selected rows: G_i = dloss/dZ_i (row_backward on
 * the double row of Z), then dH_i = sum_j G_ij W_j (the chain rule through
 * Z = H W^T). dH: nrows*D doubles, indexed by position in rows. */
void orc_linear_ce_dh_rows(const float* H, const float* W, int64_t V,
                           int64_t D, const int64_t* rows, int64_t nrows,
                           const int64_t* y, const double* g, double eps,
                           int64_t ignore_index, double* dH)
{
    #pragma omp parallel
    {
        double* zrow = (double*)malloc((size_t)V * sizeof(double));
        double* grow = (double*)malloc((size_t)V * sizeof(double));
        #pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < nrows; ++k) {
            int64_t i = rows[k];
            linear_row(H + i * D, W, V, D, zrow);
            row_backward(zrow, V, y[i], g[i], eps, ignore_index, grow);
            double* out = dH + k * D;
            for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
            for (int64_t j = 0; j < V; ++j) {
                const float* w = W + j * D;
                double gij = grow[j];
                for (int64_t d = 0; d < D; ++d) out[d] += gij * (double)w[d];
            }
        }
        free(zrow);
        free(grow);
    }
}

/* Fused-linear backward for selected vocabulary entries: the rows of
 * dW = G^T H (the chain rule through Z = H W^T, Ineshin section 1) for the
 * listed vocabulary indices. Column v of the logit gradient needs only
 * column v of Z, z_iv = H_i . W_v (double, d in order), and the log-sum-exp
 * lse_i of every row (an input: the forward over the full rows), so
 *   G_iv = g_i (exp(z_iv - lse_i) - (1-eps)[v = y_i] - eps/V)
 * (zero for ignore_index rows, NaN for a target outside [0, V)), and
 *   dW_v = sum_i G_iv H_i, i in order.
 * dW: ncols*D doubles, indexed by position in cols. */
void orc_linear_ce_dw_rows(const float* H, const float* W, int64_t N, int64_t V,
                           int64_t D, const int64_t* cols, int64_t ncols,
                           const int64_t* y, const double* g, const double* lse,
                           double eps, int64_t ignore_index, double* dW)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < ncols; ++k) {
        const int64_t v = cols[k];
        const float* w = W + v * D;
        double* out = dW + k * D;
        for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
        for (int64_t i = 0; i < N; ++i) {
            double giv;
            if (y[i] == ignore_index) {
                giv = 0.0;
            } else if (y[i] < 0 || y[i] >= V) {
                giv = NAN;
            } else {
                const float* h = H + i * D;
                double z = 0.0;
                for (int64_t d = 0; d < D; ++d) z += (double)h[d] * (double)w[d];
                const double onehot = (v == y[i]) ? 1.0 : 0.0;
                giv = g[i] * (exp(z - lse[i]) - (1.0 - eps) * onehot - eps / (double)V);
            }
            if (giv == 0.0) continue;
            const float* h = H + i * D;
            for (int64_t d = 0; d < D; ++d) out[d] += giv * (double)h[d];
        }
    }
}

/* Full fused-linear backward for small problems: G = dloss/dZ (N x V double,
 * caller-provided scratch), dH = G W (N x D), dW = G^T H (V x D). Sums over
 * the contracted index run in order. */
void orc_linear_ce_backward(const float* H, const float* W, int64_t N,
                            int64_t V, int64_t D, const int64_t* y,
                            const double* g, double eps, int64_t ignore_index,
                            double* G, double* dH, double* dW)
{
    #pragma omp parallel
    {
        double* zrow = (double*)malloc((size_t)V * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t i = 0; i < N; ++i) {
            linear_row(H + i * D, W, V, D, zrow);
            row_backward(zrow, V, y[i], g[i], eps, ignore_index, G + i * V);
        }
        free(zrow);
    }
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < V; ++j)
                acc += G[i * V + j] * (double)W[j * D + d];
            dH[i * D + d] = acc;
        }
    }
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < V; ++j) {
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t i = 0; i < N; ++i)
                acc += G[i * V + j] * (double)H[i * D + d];
            dW[j * D + d] = acc;
        }
    }
}

/* ---- Probability (soft) targets --------------------------------------------
 * The cross-entropy of the softmax of a row z against a target distribution
 * t over the same V classes (MLX PR #4188, "Shift by the max in
 * cross_entropy": the loss is lse minus the target-weighted logits, assembled
 * from shifted values):
 *     loss = sum_j t'_j (lse - z_j),   t'_j = (1-eps) t_j + eps/V,
 * which is lse - sum_j t_j z_j when t sums to 1 and eps = 0. Its gradient
 * with respect to z_k, scaled by g, is
 *     dz_k = g (p_k T' - t'_k),   p_k = exp(z_k - lse),   T' = sum_j t'_j.
 * Readings where the pages are silent:
 *   - t is used as given (not renormalised; negative entries allowed).
 *   - label smoothing mixes t with the uniform distribution, as for hard
 *     targets: eps/V on every class.
 *   - a class whose t'_j is exactly 0 contributes nothing, even where z_j is
 *     -inf (the 0 log 0 = 0 convention of cross-entropy).
 *   - NaN anywhere in z, or a row of z that is all -inf: lse as for hard
 *     targets (NaN, -inf), loss NaN, gradient row NaN.
 *   - there is no ignore_index. */
static void soft_row_forward(const double* z, const double* t, int64_t V, double eps,
                             double* loss, double* lse, double* m_out, double* s_out)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < V; ++j) {
        if (isnan(z[j])) { m = NAN; break; }
        if (z[j] > m) m = z[j];
    }
    *m_out = m;
    if (isnan(m) || m == -INFINITY) {
        *lse = isnan(m) ? NAN : -INFINITY;
        *loss = NAN;
        *s_out = isnan(m) ? NAN : 0.0;
        return;
    }
    double s = 0.0;
    for (int64_t j = 0; j < V; ++j) s += exp(z[j] - m);
    const double L = log(s);
    *lse = m + L;
    *s_out = s;
    double l = 0.0;
    for (int64_t j = 0; j < V; ++j) {
        const double tj = (1.0 - eps) * t[j] + eps / (double)V;
        if (tj != 0.0) l += tj * (L - (z[j] - m));
    }
    *loss = l;
}

/* Soft-target forward over contiguous (N, V) logits and targets. */
void orc_ce_soft_forward(const double* z, const double* t, int64_t N, int64_t V, double eps,
                         double* loss, double* lse)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        double m, s;
        soft_row_forward(z + i * V, t + i * V, V, eps, &loss[i], &lse[i], &m, &s);
    }
}

/* Soft-target VJP: dz_k = g_i (p_k T' - t'_k). g: N doubles; dz: N*V. */
void orc_ce_soft_backward(const double* z, const double* t, int64_t N, int64_t V,
                          const double* g, double eps, double* dz)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double* zr = z + i * V;
        const double* tr = t + i * V;
        double* d = dz + i * V;
        double loss, lse, m, s;
        soft_row_forward(zr, tr, V, eps, &loss, &lse, &m, &s);
        if (isnan(m) || m == -INFINITY) {
            for (int64_t j = 0; j < V; ++j) d[j] = NAN;
            continue;
        }
        double T = 0.0;
        for (int64_t j = 0; j < V; ++j) T += (1.0 - eps) * tr[j] + eps / (double)V;
        for (int64_t j = 0; j < V; ++j) {
            const double p = exp(zr[j] - m) / s;
            const double tj = (1.0 - eps) * tr[j] + eps / (double)V;
            d[j] = g[i] * (p * T - tj);
        }
    }
}

/* ---- KL divergence of a student distribution from a teacher's ------------
 * "One barrier short" (Suryavanshi), the fused KL loss of mlx-lm: per row,
 * with teacher logits zp and student logits zq over the same V classes,
 *     p = softmax(zp), q = softmax(zq),
 *     loss = sum_j p_j (log p_j - log q_j),
 * and the gradient of sum_i g_i loss_i with respect to the student logits,
 *     dzq_j = g (q_j - p_j).
 * Readings where the pages are silent:
 *   - a class with p_j = 0 (teacher logit -inf) adds nothing, even where
 *     the student's is -inf too (0 log 0 = 0); a student -inf under teacher
 *     mass makes the loss +inf.
 *   - NaN in either row, or a row of either that is all -inf: loss NaN and
 *     a NaN gradient row; each lse as for the cross-entropy (NaN, -inf). */
static double row_lse(const double* z, int64_t V, double* m_out, double* s_out)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < V; ++j) {
        if (isnan(z[j])) { *m_out = NAN; *s_out = NAN; return NAN; }
        if (z[j] > m) m = z[j];
    }
    *m_out = m;
    if (m == -INFINITY) { *s_out = 0.0; return -INFINITY; }
    double s = 0.0;
    for (int64_t j = 0; j < V; ++j) s += exp(z[j] - m);
    *s_out = s;
    return m + log(s);
}

void orc_kl_forward(const double* zq, const double* zp, int64_t N, int64_t V,
                    double* loss, double* lse_q, double* lse_p)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double* q = zq + i * V;
        const double* p = zp + i * V;
        double mq, sq, mp, sp;
        lse_q[i] = row_lse(q, V, &mq, &sq);
        lse_p[i] = row_lse(p, V, &mp, &sp);
        if (!isfinite(lse_q[i]) || !isfinite(lse_p[i])) { loss[i] = NAN; continue; }
        double l = 0.0;
        for (int64_t j = 0; j < V; ++j) {
            const double lp = p[j] - lse_p[i];
            const double pj = exp(lp);
            if (pj != 0.0) l += pj * (lp - (q[j] - lse_q[i]));
        }
        loss[i] = l;
    }
}

void orc_kl_backward(const double* zq, const double* zp, int64_t N, int64_t V,
                     const double* g, double* dzq)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double* q = zq + i * V;
        const double* p = zp + i * V;
        double* d = dzq + i * V;
        double mq, sq, mp, sp;
        const double lq = row_lse(q, V, &mq, &sq);
        const double lp = row_lse(p, V, &mp, &sp);
        if (!isfinite(lq) || !isfinite(lp)) {
            for (int64_t j = 0; j < V; ++j) d[j] = NAN;
            continue;
        }
        for (int64_t j = 0; j < V; ++j) d[j] = g[i] * (exp(q[j] - lq) - exp(p[j] - lp));
    }
}

/* Threads OpenMP will use, for reporting the CPU baseline's core count. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
