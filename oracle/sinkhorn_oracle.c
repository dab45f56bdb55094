/*
 * sinkhorn_oracle.c -- TEST INFRASTRUCTURE, not part of the product path.
 *
 * A plain, slow, float64 CPU statement of what the GPU library computes:
 * online log-domain Sinkhorn between two point clouds under squared-Euclidean
 * cost, the transport-plan row formula, the marginal residuals and the exact
 * min_row threshold. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code,
 * header, table or constant with the CUDA sources.
 *
 * Sources (the pages this follows):
 *  - moscot PR #846, "materialize transport-matrix rows instead of pushing
 *    indicator columns", section "Fix": the entropic plan entry
 *    T_ij = exp((f_i + g_j - C_ij) / eps) with C from the point-cloud cost, and
 *    the rule that the parent's resolved inv_scale_cost / eps are captured
 *    (never re-derived from a subset).
 *  - same page, section "Behavioural changes": min_row keeps the largest
 *    threshold that leaves every row non-empty, min_i max_j T_ij; rows that
 *    carry no mass keep nothing and do not take part in the threshold.
 *  - "FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section 2.1:
 *    log-domain Sinkhorn alternates source and target dual-potential updates,
 *    each a log-sum-exp reduction; the cost is computed on the fly.
 *  - same paper, section D.3: accurate evaluation builds the cost from
 *    coordinate differences in FP64 (this file always does).
 *  - POT PR #868, test list: a log-sum-exp over an all -inf row is -inf.
 *
 * Readings where the pages are silent (each one is listed with the design):
 *  - No a(x)b factor in the plan (plan = exp((f+g-C)/eps)), so the updates are
 *      f_i = eps*ln(a_i) - eps*LSE_j((g_j - C_ij)/eps)
 *      g_j = eps*ln(b_j) - eps*LSE_i((f_i - C_ij)/eps),
 *    f first, from f = g = 0 unless a warm start is given.
 *  - The stopping residual is ||T 1 - a||_1 of the state after a full
 *    iteration, checked after every iteration when tol > 0.
 *  - scale "mean"/"max" are the unweighted mean / max over all n*m pairs of
 *    the squared distance; eps is absolute, on the scaled cost.
 *  - A massless row (a_i == 0) has f_i = -inf.
 *
 * Parallelism: OpenMP over rows (or columns), each row reduced serially in
 * index order, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* squared Euclidean distance from coordinate differences, in float64 */
static double sqdist(const float *p, const float *q, int d) {
    double s = 0.0;
    for (int k = 0; k < d; ++k) {
        double t = (double)p[k] - (double)q[k];
        s += t * t;
    }
    return s;
}

/* C_ij as used by the method: inv_scale_cost * ||x_i - y_j||^2 */
static double cost(const float *x, const float *y, int64_t i, int64_t j, int d, double c) {
    return c * sqdist(x + i * (int64_t)d, y + j * (int64_t)d, d);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- scale --
 * mode 0: no scaling (c = 1); 1: c = 1/mean_ij ||x_i-y_j||^2 (brute force over
 * all pairs); 2: c = 1/max_ij ||x_i-y_j||^2; 3: c = 1/value.               */
double orc_inv_scale_cost(const float *x, const float *y, int64_t n, int64_t m, int d,
                          int mode, double value) {
    if (mode == 0) return 1.0;
    if (mode == 3) return 1.0 / value;
    double *acc = (double *)calloc((size_t)n, sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0, mx = 0.0;
        for (int64_t j = 0; j < m; ++j) {
            double cij = cost(x, y, i, j, d, 1.0);
            s += cij;
            if (cij > mx) mx = cij;
        }
        acc[i] = (mode == 1) ? s : mx;
    }
    double r = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (mode == 1) r += acc[i];
        else if (acc[i] > r) r = acc[i];
    }
    free(acc);
    if (mode == 1) r /= ((double)n * (double)m);
    return 1.0 / r;
}

/* ------------------------------------------------------------------ LSE --
 * log(sum_k exp(v_k)) with the max shift; all -inf gives -inf.             */
static double lse(const double *v, int64_t len) {
    double mx = -INFINITY;
    for (int64_t k = 0; k < len; ++k)
        if (v[k] > mx) mx = v[k];
    if (mx == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int64_t k = 0; k < len; ++k) s += exp(v[k] - mx);
    return mx + log(s);
}

/* ----------------------------------------------------------- half-steps --
 * f-update (FlashSinkhorn 2, section 2.1; source potential first):
 *   f_i = eps*ln a_i - eps*LSE_j((g_j - C_ij)/eps),   f_i = -inf if a_i == 0.
 * rows: only the listed rows are updated when rows != NULL (used to check a
 * sample of a large problem one row at a time).                            */
void orc_f_step(const float *x, const float *y, const double *a, const double *g,
                int64_t n, int64_t m, int d, double c, double eps,
                const int64_t *rows, int64_t nrows, double *f_out) {
    int64_t cnt = rows ? nrows : n;
    #pragma omp parallel
    {
        double *v = (double *)malloc((size_t)(m > 0 ? m : 1) * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < cnt; ++r) {
            int64_t i = rows ? rows[r] : r;
            double out;
            if (a[i] == 0.0) {
                out = -INFINITY;
            } else {
                for (int64_t j = 0; j < m; ++j) v[j] = (g[j] - cost(x, y, i, j, d, c)) / eps;
                out = eps * log(a[i]) - eps * lse(v, m);
            }
            f_out[rows ? r : i] = out;
        }
        free(v);
    }
}

/* g-update, the same reduction over the other index:
 *   g_j = eps*ln b_j - eps*LSE_i((f_i - C_ij)/eps),   g_j = -inf if b_j == 0. */
void orc_g_step(const float *x, const float *y, const double *b, const double *f,
                int64_t n, int64_t m, int d, double c, double eps,
                const int64_t *cols, int64_t ncols, double *g_out) {
    int64_t cnt = cols ? ncols : m;
    #pragma omp parallel
    {
        double *v = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < cnt; ++r) {
            int64_t j = cols ? cols[r] : r;
            double out;
            if (b[j] == 0.0) {
                out = -INFINITY;
            } else {
                for (int64_t i = 0; i < n; ++i) v[i] = (f[i] - cost(x, y, i, j, d, c)) / eps;
                out = eps * log(b[j]) - eps * lse(v, n);
            }
            g_out[cols ? r : j] = out;
        }
        free(v);
    }
}

/* ----------------------------------------------------------- plan entry --
 * T_ij = exp((f_i + g_j - C_ij)/eps)  (moscot PR #846, "Fix", entropic rows). */
static double plan_entry(const float *x, const float *y, const double *f, const double *g,
                         int64_t i, int64_t j, int d, double c, double eps) {
    if (f[i] == -INFINITY || g[j] == -INFINITY) return 0.0;
    return exp((f[i] + g[j] - cost(x, y, i, j, d, c)) / eps);
}

/* ------------------------------------------------------------- residual --
 * row_l1 = sum_i |sum_j T_ij - a_i|, col_l1 = sum_j |sum_i T_ij - b_j|;
 * row_sums/col_sums (optional) receive the marginals of T.                  */
void orc_marginal_residual(const float *x, const float *y, const double *a, const double *b,
                           const double *f, const double *g, int64_t n, int64_t m, int d,
                           double c, double eps, double *row_l1, double *col_l1,
                           double *row_sums, double *col_sums) {
    double *rs = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double *cs = (double *)malloc((size_t)(m > 0 ? m : 1) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int64_t j = 0; j < m; ++j) s += plan_entry(x, y, f, g, i, j, d, c, eps);
        rs[i] = s;
    }
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < m; ++j) {
        double s = 0.0;
        for (int64_t i = 0; i < n; ++i) s += plan_entry(x, y, f, g, i, j, d, c, eps);
        cs[j] = s;
    }
    double r = 0.0, q = 0.0;
    for (int64_t i = 0; i < n; ++i) r += fabs(rs[i] - a[i]);
    for (int64_t j = 0; j < m; ++j) q += fabs(cs[j] - b[j]);
    if (row_l1) *row_l1 = r;
    if (col_l1) *col_l1 = q;
    if (row_sums) memcpy(row_sums, rs, (size_t)n * sizeof(double));
    if (col_sums) memcpy(col_sums, cs, (size_t)m * sizeof(double));
    free(rs);
    free(cs);
}

/* row residual only (the stopping test), ||T 1 - a||_1 */
static double row_residual(const float *x, const float *y, const double *a, const double *f,
                           const double *g, int64_t n, int64_t m, int d, double c, double eps) {
    double *rs = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int64_t j = 0; j < m; ++j) s += plan_entry(x, y, f, g, i, j, d, c, eps);
        rs[i] = fabs(s - a[i]);
    }
    double r = 0.0;
    for (int64_t i = 0; i < n; ++i) r += rs[i];
    free(rs);
    return r;
}

/* ------------------------------------------------------------ iterations --
 * One iteration = f-update then g-update (FlashSinkhorn 2, section 2.1).
 * f, g: in (warm start; zeros for a cold start) and out.
 * n_iters is the cap; tol > 0 stops after the first iteration whose state has
 * ||T 1 - a||_1 <= tol. Returns the number of iterations done; *resid gets the
 * row residual of the returned state (always computed).                    */
int orc_sinkhorn(const float *x, const float *y, const double *a, const double *b,
                 int64_t n, int64_t m, int d, double c, double eps, int n_iters, double tol,
                 double *f, double *g, double *resid) {
    int it = 0;
    double r = NAN;
    for (it = 1; it <= n_iters; ++it) {
        orc_f_step(x, y, a, g, n, m, d, c, eps, NULL, 0, f);
        orc_g_step(x, y, b, f, n, m, d, c, eps, NULL, 0, g);
        if (tol > 0.0) {
            r = row_residual(x, y, a, f, g, n, m, d, c, eps);
            if (r <= tol) break;
        }
    }
    if (it > n_iters) it = n_iters;
    if (tol <= 0.0 || isnan(r)) r = row_residual(x, y, a, f, g, n, m, d, c, eps);
    if (resid) *resid = r;
    return it;
}

/* eps-annealing driver (FlashSinkhorn 2, sections 3.1 and C.3 anneal eps and
 * continue at the target eps; the schedule itself is this build's reading):
 * stage k runs iters_per_stage iterations at eps_k = max(eps_target,
 * eps_init * decay^k), potentials carried over unchanged; the last stage is
 * the first one whose eps_k equals eps_target. Returns the number of stages;
 * *resid is the row residual at the end.                                   */
int orc_sinkhorn_anneal(const float *x, const float *y, const double *a, const double *b,
                        int64_t n, int64_t m, int d, double c, double eps_target,
                        double eps_init, double decay, int iters_per_stage,
                        double *f, double *g, double *resid) {
    int k = 0;
    for (;; ++k) {
        double ek = eps_init * pow(decay, (double)k);
        if (ek < eps_target) ek = eps_target;
        double r = 0.0;
        orc_sinkhorn(x, y, a, b, n, m, d, c, ek, iters_per_stage, 0.0, f, g, &r);
        if (ek == eps_target) {
            if (resid) *resid = r;
            break;
        }
    }
    return k + 1;
}

/* --------------------------------------------------------- materializer --
 * out[r*m + j] = T_{row_idx[r], j}  (moscot PR #846, "Fix": rows built from
 * the potentials and the captured inv_scale_cost/eps, O(k*m) memory).      */
void orc_materialize_rows(const float *x, const float *y, const double *f, const double *g,
                          int64_t n, int64_t m, int d, double c, double eps,
                          const int64_t *row_idx, int64_t k, double *out) {
    (void)n;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < k; ++r) {
        int64_t i = row_idx[r];
        for (int64_t j = 0; j < m; ++j)
            out[r * m + j] = plan_entry(x, y, f, g, i, j, d, c, eps);
    }
}

/* the full n x m plan, entry by entry (used only on small inputs) */
void orc_dense_plan(const float *x, const float *y, const double *f, const double *g,
                    int64_t n, int64_t m, int d, double c, double eps, double *T) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < m; ++j)
            T[i * m + j] = plan_entry(x, y, f, g, i, j, d, c, eps);
}

/* --------------------------------------------------------------- min_row --
 * moscot PR #846, "Behavioural changes": thr = min over rows carrying mass of
 * max_j T_ij; entries with T_ij >= thr are kept; massless rows (a_i == 0) keep
 * nothing and are excluded from the min. The rows are visited in blocks of
 * block_rows, which must not change any result. counts (optional, [n]) gets
 * the kept entries per row. Returns the number of massless rows; *thr_out is
 * +inf when every row is massless; *argmin_out is the row attaining thr
 * (smallest index on ties).                                                 */
int64_t orc_min_row(const float *x, const float *y, const double *a, const double *f,
                    const double *g, int64_t n, int64_t m, int d, double c, double eps,
                    int64_t block_rows, double *thr_out, int64_t *argmin_out,
                    int64_t *counts, int64_t *nnz_out) {
    double *rowmax = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    if (block_rows <= 0) block_rows = n > 0 ? n : 1;
    for (int64_t r0 = 0; r0 < n; r0 += block_rows) {
        int64_t r1 = r0 + block_rows < n ? r0 + block_rows : n;
        #pragma omp parallel for schedule(static)
        for (int64_t i = r0; i < r1; ++i) {
            double mx = -INFINITY;
            for (int64_t j = 0; j < m; ++j) {
                double t = plan_entry(x, y, f, g, i, j, d, c, eps);
                if (t > mx) mx = t;
            }
            rowmax[i] = mx;
        }
    }
    double thr = INFINITY;
    int64_t arg = -1, massless = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (a[i] == 0.0) { ++massless; continue; }
        if (rowmax[i] < thr) { thr = rowmax[i]; arg = i; }
    }
    int64_t nnz = 0;
    for (int64_t r0 = 0; r0 < n; r0 += block_rows) {
        int64_t r1 = r0 + block_rows < n ? r0 + block_rows : n;
        #pragma omp parallel for schedule(static) reduction(+ : nnz)
        for (int64_t i = r0; i < r1; ++i) {
            int64_t cnt = 0;
            if (a[i] != 0.0)
                for (int64_t j = 0; j < m; ++j)
                    if (plan_entry(x, y, f, g, i, j, d, c, eps) >= thr) ++cnt;
            if (counts) counts[i] = cnt;
            nnz += cnt;
        }
    }
    free(rowmax);
    if (thr_out) *thr_out = thr;
    if (argmin_out) *argmin_out = arg;
    if (nnz_out) *nnz_out = nnz;
    return massless;
}

/* ------------------------------------------------------------ low rank --
 * Rows of a low-rank coupling (moscot PR #846, "Fix": for low-rank outputs
 * T[rows] = (Q diag(1/g) R^T)[rows], a matrix product, no geometry):
 *     out[t*m + j] = sum_k Q[i,k] R[j,k] / g[k],   i = rows[t].
 * Q [n,r], R [m,r], g [r] as given (float32, promoted to double).          */
void orc_lr_rows(const float *Q, const float *R, const float *g, int64_t n, int64_t m, int r,
                 const int64_t *rows, int64_t k, double *out) {
    (void)n;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < k; ++t) {
        const int64_t i = rows[t];
        for (int64_t j = 0; j < m; ++j) {
            double s = 0.0;
            for (int q = 0; q < r; ++q)
                s += (double)Q[i * r + q] * (double)R[j * r + q] / (double)g[q];
            out[t * m + j] = s;
        }
    }
}

/* Entropic rows on a low-rank cost geometry (same page: cost rows
 * cost_1[rows] @ cost_2^T + bias), with the captured scale c and eps:
 *     C_ij = c * (sum_k cost1[i,k] cost2[j,k] + bias),
 *     out[t*m + j] = exp((f_i + g_j - C_ij) / eps),   i = rows[t].         */
void orc_lrc_rows(const float *c1, const float *c2, const double *f, const double *g, int64_t n,
                  int64_t m, int r, double bias, double c, double eps, const int64_t *rows,
                  int64_t k, double *out) {
    (void)n;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < k; ++t) {
        const int64_t i = rows[t];
        for (int64_t j = 0; j < m; ++j) {
            double dot = 0.0;
            for (int q = 0; q < r; ++q) dot += (double)c1[i * r + q] * (double)c2[j * r + q];
            const double C = c * (dot + bias);
            out[t * m + j] = exp((f[i] + g[j] - C) / eps);
        }
    }
}

/* ------------------------------------------------------------- sparsify --
 * The sparse plan that thresholding produces (moscot PR #846, "Behavioural
 * changes": entries with T_ij >= thr are kept, rows without mass keep nothing),
 * in compressed-row form: row_ptr [n+1], and for row i the kept columns in
 * increasing order in col_idx[row_ptr[i] .. row_ptr[i+1]) with their values in
 * vals. A first pass counts every row, a second writes them. Returns nnz, or
 * -1 (writing no entry) when nnz exceeds cap.                               */
int64_t orc_sparsify_csr(const float *x, const float *y, const double *a, const double *f,
                         const double *g, int64_t n, int64_t m, int d, double c, double eps,
                         double thr, int64_t *row_ptr, int64_t *col_idx, double *vals,
                         int64_t cap) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t cnt = 0;
        if (a[i] != 0.0)
            for (int64_t j = 0; j < m; ++j)
                if (plan_entry(x, y, f, g, i, j, d, c, eps) >= thr) ++cnt;
        row_ptr[i + 1] = cnt;
    }
    row_ptr[0] = 0;
    for (int64_t i = 0; i < n; ++i) row_ptr[i + 1] += row_ptr[i];
    if (row_ptr[n] > cap) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        if (a[i] == 0.0) continue;
        int64_t k = row_ptr[i];
        for (int64_t j = 0; j < m; ++j) {
            const double t = plan_entry(x, y, f, g, i, j, d, c, eps);
            if (t >= thr) {
                col_idx[k] = j;
                vals[k] = t;
                ++k;
            }
        }
    }
    return row_ptr[n];
}

/* ------------------------------------------------- block-sparse updates --
 * "FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", sections 3,
 * 3.2, A.3, B.1 and B.3: points in Morton order, blocks of B consecutive
 * points, a block-pair screen from block potential maxima and bounding boxes,
 * verification of the surviving pairs by their exact mass over the B x B
 * point pairs, and half-steps that reduce only over the admitted tiles (a
 * block with no admitted tile reduces over everything).
 *
 * Readings (the pages state the rules in words, not formulas):
 *  - Morton code: every coordinate is quantised over the joint bounding box
 *    of both clouds (lo_k = min, hi_k = max over all points) into 2^bits
 *    cells, bits = 30/d (d = 1, 2, 3: 30, 15, 10):
 *        q_k = floor((v_k - lo_k) * (2^bits / (hi_k - lo_k))), clamped to
 *        [0, 2^bits - 1] (q_k = 0 when hi_k == lo_k);
 *    bit t of q_k is bit t*d + (d-1-k) of the code (coordinate 0 the most
 *    significant of each group); points are ordered by (code, index).
 *  - Tile mass M_pq = sum over i in I_p, j in J_q of exp((f_i + g_j - C_ij)/eps).
 *    Screen bound: C_ij >= c D_pq with D_pq the squared distance between the
 *    two blocks' bounding boxes, f_i <= F_p = max over I_p, g_j <= G_q, so
 *        M_pq <= U_pq = |I_p| |J_q| exp((F_p + G_q - c D_pq)/eps).
 *  - Threshold (the mass-dependent rule of A.3): rho_pq = delta * min(amin_p,
 *    bmin_q), amin_p the smallest nonzero a_i of block p. A tile is a
 *    candidate when U_pq > rho_pq and admitted when it is a candidate and
 *    (with verification) M_pq > rho_pq, so an omitted tile adds at most
 *    delta a_i to row i and delta b_j to column j. delta defaults to
 *    tol / (4 max(NB, MB)) (section 3.2): at most tol/4 of the mass is
 *    omitted over all rows when the weights sum to one.
 *  - A fine iteration builds the mask at the current (f, g) and runs the f-
 *    and the g-update on it (the g-update reads it transposed). The stop test
 *    takes the admitted plan's row residual at the state the mask was built
 *    at and compares it with tol - MB delta sum(a), so that the full residual
 *    (admitted plus omitted) is at most tol.
 *  - An iteration whose candidate count exceeds dense_frac * NB * MB runs the
 *    dense updates instead (sparse updates pay only when the admitted tiles
 *    are well below all block pairs); its residual is then the full one.
 */
void orc_morton_codes(const float *x, int64_t n, int d, const double *lo, const double *hi,
                      uint64_t *code) {
    const int bits = 30 / d;
    const double cells = (double)((int64_t)1 << bits);
    for (int64_t i = 0; i < n; ++i) {
        uint64_t cd = 0;
        for (int k = 0; k < d; ++k) {
            int64_t q = 0;
            if (hi[k] > lo[k]) {
                const double s = cells / (hi[k] - lo[k]);
                const double t = floor(((double)x[i * d + k] - lo[k]) * s);
                q = t < 0.0 ? 0 : t > cells - 1.0 ? (int64_t)cells - 1 : (int64_t)t;
            }
            for (int t = 0; t < bits; ++t)
                if ((q >> t) & 1) cd |= (uint64_t)1 << (t * d + (d - 1 - k));
        }
        code[i] = cd;
    }
}

typedef struct {
    uint64_t code;
    int64_t idx;
} morton_key;

static int morton_cmp(const void *p, const void *q) {
    const morton_key *u = (const morton_key *)p, *v = (const morton_key *)q;
    if (u->code != v->code) return u->code < v->code ? -1 : 1;
    return u->idx < v->idx ? -1 : u->idx > v->idx ? 1 : 0;
}

/* perm[r] = index of the r-th point in Morton order */
void orc_morton_order(const float *x, int64_t n, int d, const double *lo, const double *hi,
                      int64_t *perm) {
    uint64_t *code = (uint64_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(uint64_t));
    morton_key *key = (morton_key *)malloc((size_t)(n > 0 ? n : 1) * sizeof(morton_key));
    orc_morton_codes(x, n, d, lo, hi, code);
    for (int64_t i = 0; i < n; ++i) {
        key[i].code = code[i];
        key[i].idx = i;
    }
    qsort(key, (size_t)n, sizeof(morton_key), morton_cmp);
    for (int64_t r = 0; r < n; ++r) perm[r] = key[r].idx;
    free(code);
    free(key);
}

/* per block: potential maximum, smallest nonzero weight, bounding box */
static void block_summary(const float *x, const double *w, const double *pot, int64_t cnt,
                          int d, int64_t B, int64_t p, double *pmax, double *wmin, double *lo,
                          double *hi) {
    const int64_t i0 = p * B, i1 = (p + 1) * B < cnt ? (p + 1) * B : cnt;
    *pmax = -INFINITY;
    *wmin = INFINITY;
    for (int k = 0; k < d; ++k) {
        lo[k] = INFINITY;
        hi[k] = -INFINITY;
    }
    for (int64_t i = i0; i < i1; ++i) {
        if (pot[i] > *pmax) *pmax = pot[i];
        if (w[i] > 0.0 && w[i] < *wmin) *wmin = w[i];
        for (int k = 0; k < d; ++k) {
            const double v = (double)x[i * d + k];
            if (v < lo[k]) lo[k] = v;
            if (v > hi[k]) hi[k] = v;
        }
    }
}

/* The block-pair mask at (f, g). x, y, a, b, f, g in Morton order. cand and
 * adm: [NB * MB] bytes, 1 for a candidate / admitted tile. Optional outputs:
 * screen_margin[pq] = ln U_pq - ln rho_pq and mass_margin[pq] = ln M_pq -
 * ln rho_pq (NAN where not evaluated), n_cand. Returns the admitted count. */
int64_t orc_block_mask(const float *x, const float *y, const double *a, const double *b,
                       const double *f, const double *g, int64_t n, int64_t m, int d,
                       double c, double eps, int64_t B, double delta, int verify,
                       uint8_t *cand, uint8_t *adm, double *screen_margin, double *mass_margin,
                       int64_t *n_cand) {
    const int64_t NB = (n + B - 1) / B, MB = (m + B - 1) / B;
    double *rs = (double *)malloc((size_t)NB * (2 + 2 * d) * sizeof(double));
    double *cs = (double *)malloc((size_t)MB * (2 + 2 * d) * sizeof(double));
    for (int64_t p = 0; p < NB; ++p) {
        double *s = rs + p * (2 + 2 * d);
        block_summary(x, a, f, n, d, B, p, s, s + 1, s + 2, s + 2 + d);
    }
    for (int64_t q = 0; q < MB; ++q) {
        double *s = cs + q * (2 + 2 * d);
        block_summary(y, b, g, m, d, B, q, s, s + 1, s + 2, s + 2 + d);
    }
    int64_t nc = 0, na = 0;
    #pragma omp parallel for schedule(dynamic, 1) reduction(+ : nc, na)
    for (int64_t p = 0; p < NB; ++p) {
        const double *sp = rs + p * (2 + 2 * d);
        const int64_t ni = ((p + 1) * B < n ? (p + 1) * B : n) - p * B;
        double *v = (double *)malloc((size_t)(B * B) * sizeof(double));
        for (int64_t q = 0; q < MB; ++q) {
            const double *sq = cs + q * (2 + 2 * d);
            const int64_t mj = ((q + 1) * B < m ? (q + 1) * B : m) - q * B;
            const int64_t pq = p * MB + q;
            cand[pq] = adm[pq] = 0;
            if (screen_margin) screen_margin[pq] = -INFINITY;
            if (mass_margin) mass_margin[pq] = NAN;
            if (sp[0] == -INFINITY || sq[0] == -INFINITY) continue;  /* U_pq = 0 */
            double D = 0.0;
            for (int k = 0; k < d; ++k) {
                double gap = 0.0;
                if (sp[2 + k] - sq[2 + d + k] > gap) gap = sp[2 + k] - sq[2 + d + k];
                if (sq[2 + k] - sp[2 + d + k] > gap) gap = sq[2 + k] - sp[2 + d + k];
                D += gap * gap;
            }
            const double log_rho = log(delta) + log(sp[1] < sq[1] ? sp[1] : sq[1]);
            const double log_u = log((double)ni * (double)mj) + (sp[0] + sq[0] - c * D) / eps;
            if (screen_margin) screen_margin[pq] = log_u - log_rho;
            if (!(log_u > log_rho)) continue;
            cand[pq] = 1;
            ++nc;
            if (!verify) {
                adm[pq] = 1;
                ++na;
                continue;
            }
            int64_t len = 0;
            for (int64_t i = p * B; i < p * B + ni; ++i)
                for (int64_t j = q * B; j < q * B + mj; ++j)
                    v[len++] = (f[i] == -INFINITY || g[j] == -INFINITY)
                                   ? -INFINITY
                                   : (f[i] + g[j] - cost(x, y, i, j, d, c)) / eps;
            const double log_m = lse(v, len);
            if (mass_margin) mass_margin[pq] = log_m - log_rho;
            if (log_m > log_rho) {
                adm[pq] = 1;
                ++na;
            }
        }
        free(v);
    }
    free(rs);
    free(cs);
    if (n_cand) *n_cand = nc;
    return na;
}

/* does block p (of the updated side) have an admitted tile? */
static int block_has_tile(const uint8_t *adm, int64_t NB, int64_t MB, int64_t p, int rows_side) {
    if (rows_side) {
        for (int64_t q = 0; q < MB; ++q)
            if (adm[p * MB + q]) return 1;
    } else {
        for (int64_t r = 0; r < NB; ++r)
            if (adm[r * MB + p]) return 1;
    }
    return 0;
}

/* f-update on the mask (section 3.2): row i of block p reduces over the
 * columns of the tiles q with adm[p][q]; over every column when block p has
 * no admitted tile. x, y, a, g in Morton order.                            */
void orc_sparse_f_step(const float *x, const float *y, const double *a, const double *g,
                       int64_t n, int64_t m, int d, double c, double eps, int64_t B,
                       const uint8_t *adm, double *f_out) {
    const int64_t NB = (n + B - 1) / B, MB = (m + B - 1) / B;
    #pragma omp parallel
    {
        double *v = (double *)malloc((size_t)(m > 0 ? m : 1) * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t i = 0; i < n; ++i) {
            const int64_t p = i / B;
            const int all = !block_has_tile(adm, NB, MB, p, 1);
            if (a[i] == 0.0) {
                f_out[i] = -INFINITY;
                continue;
            }
            int64_t len = 0;
            for (int64_t j = 0; j < m; ++j)
                if (all || adm[p * MB + j / B]) v[len++] = (g[j] - cost(x, y, i, j, d, c)) / eps;
            f_out[i] = eps * log(a[i]) - eps * lse(v, len);
        }
        free(v);
    }
}

/* g-update on the same mask, read by columns. */
void orc_sparse_g_step(const float *x, const float *y, const double *b, const double *f,
                       int64_t n, int64_t m, int d, double c, double eps, int64_t B,
                       const uint8_t *adm, double *g_out) {
    const int64_t NB = (n + B - 1) / B, MB = (m + B - 1) / B;
    #pragma omp parallel
    {
        double *v = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t j = 0; j < m; ++j) {
            const int64_t q = j / B;
            const int all = !block_has_tile(adm, NB, MB, q, 0);
            if (b[j] == 0.0) {
                g_out[j] = -INFINITY;
                continue;
            }
            int64_t len = 0;
            for (int64_t i = 0; i < n; ++i)
                if (all || adm[(i / B) * MB + q]) v[len++] = (f[i] - cost(x, y, i, j, d, c)) / eps;
            g_out[j] = eps * log(b[j]) - eps * lse(v, len);
        }
        free(v);
    }
}

/* row residual of the admitted plan, sum_i |sum_{admitted j} T_ij - a_i|
 * (every column for a row block without an admitted tile).               */
double orc_sparse_row_residual(const float *x, const float *y, const double *a, const double *f,
                               const double *g, int64_t n, int64_t m, int d, double c,
                               double eps, int64_t B, const uint8_t *adm) {
    const int64_t NB = (n + B - 1) / B, MB = (m + B - 1) / B;
    double *rs = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t p = i / B;
        const int all = !block_has_tile(adm, NB, MB, p, 1);
        double s = 0.0;
        for (int64_t j = 0; j < m; ++j)
            if (all || adm[p * MB + j / B]) s += plan_entry(x, y, f, g, i, j, d, c, eps);
        rs[i] = fabs(s - a[i]);
    }
    double r = 0.0;
    for (int64_t i = 0; i < n; ++i) r += rs[i];
    free(rs);
    return r;
}

/* Block-sparse solve (fine updates only; the readings above). Inputs and
 * f, g (warm start in, result out) in the caller's order; the iterations run
 * in Morton order. delta <= 0 takes tol / (4 max(NB, MB)) (then tol must be
 * > 0). stats (optional, 4 entries): sparse iterations, dense iterations,
 * candidates and admitted tiles of the last mask. Returns the iterations
 * done, or -1 for bad arguments; *resid gets the stop test's residual of the
 * returned state.                                                          */
int orc_sinkhorn_sparse(const float *x, const float *y, const double *a, const double *b,
                        int64_t n, int64_t m, int d, double c, double eps, int n_iters,
                        double tol, int64_t B, double delta, int verify, double dense_frac,
                        double *f, double *g, double *resid, int64_t *stats) {
    if (B < 1 || n < 1 || m < 1) return -1;
    const int64_t NB = (n + B - 1) / B, MB = (m + B - 1) / B;
    if (delta <= 0.0) {
        if (!(tol > 0.0)) return -1;
        delta = tol / (4.0 * (double)(NB > MB ? NB : MB));
    }
    double lo[3], hi[3];
    for (int k = 0; k < d; ++k) {
        lo[k] = INFINITY;
        hi[k] = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            const double v = (double)x[i * d + k];
            if (v < lo[k]) lo[k] = v;
            if (v > hi[k]) hi[k] = v;
        }
        for (int64_t j = 0; j < m; ++j) {
            const double v = (double)y[j * d + k];
            if (v < lo[k]) lo[k] = v;
            if (v > hi[k]) hi[k] = v;
        }
    }
    int64_t *px = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    int64_t *py = (int64_t *)malloc((size_t)m * sizeof(int64_t));
    orc_morton_order(x, n, d, lo, hi, px);
    orc_morton_order(y, m, d, lo, hi, py);
    float *xs = (float *)malloc((size_t)n * d * sizeof(float));
    float *ys = (float *)malloc((size_t)m * d * sizeof(float));
    double *as = (double *)malloc((size_t)n * sizeof(double));
    double *bs = (double *)malloc((size_t)m * sizeof(double));
    double *fs = (double *)malloc((size_t)n * sizeof(double));
    double *gs = (double *)malloc((size_t)m * sizeof(double));
    double asum = 0.0;
    for (int64_t r = 0; r < n; ++r) {
        for (int k = 0; k < d; ++k) xs[r * d + k] = x[px[r] * d + k];
        as[r] = a[px[r]];
        fs[r] = f[px[r]];
        asum += as[r];
    }
    for (int64_t r = 0; r < m; ++r) {
        for (int k = 0; k < d; ++k) ys[r * d + k] = y[py[r] * d + k];
        bs[r] = b[py[r]];
        gs[r] = g[py[r]];
    }
    const double tol_eff = tol - (double)MB * delta * asum;
    uint8_t *cand = (uint8_t *)malloc((size_t)(NB * MB));
    uint8_t *adm = (uint8_t *)malloc((size_t)(NB * MB));
    int64_t n_sparse = 0, n_dense = 0, nc = 0, na = 0;
    double r = NAN;
    int it = 0;
    for (;; ++it) {
        na = orc_block_mask(xs, ys, as, bs, fs, gs, n, m, d, c, eps, B, delta, verify, cand, adm,
                            NULL, NULL, &nc);
        const int dense = (double)nc > dense_frac * (double)NB * (double)MB;
        const int test = tol > 0.0 && it >= 1;
        if (test || it == n_iters) {
            r = dense ? row_residual(xs, ys, as, fs, gs, n, m, d, c, eps)
                      : orc_sparse_row_residual(xs, ys, as, fs, gs, n, m, d, c, eps, B, adm);
            if (test && r <= tol_eff) break;
        }
        if (it == n_iters) break;
        if (dense) {
            orc_f_step(xs, ys, as, gs, n, m, d, c, eps, NULL, 0, fs);
            orc_g_step(xs, ys, bs, fs, n, m, d, c, eps, NULL, 0, gs);
            ++n_dense;
        } else {
            orc_sparse_f_step(xs, ys, as, gs, n, m, d, c, eps, B, adm, fs);
            orc_sparse_g_step(xs, ys, bs, fs, n, m, d, c, eps, B, adm, gs);
            ++n_sparse;
        }
    }
    for (int64_t r2 = 0; r2 < n; ++r2) f[px[r2]] = fs[r2];
    for (int64_t r2 = 0; r2 < m; ++r2) g[py[r2]] = gs[r2];
    if (resid) *resid = r;
    if (stats) {
        stats[0] = n_sparse;
        stats[1] = n_dense;
        stats[2] = nc;
        stats[3] = na;
    }
    free(px); free(py); free(xs); free(ys); free(as); free(bs); free(fs); free(gs);
    free(cand); free(adm);
    return it;
}
