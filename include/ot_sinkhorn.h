/*
 * ot_sinkhorn.h -- C ABI of the B200 (sm_100a) online log-domain Sinkhorn library.
 *
 * Entropic optimal transport between two point clouds x[n,d], y[m,d] with
 * weights a[n], b[m] under the squared-Euclidean cost
 *     C_ij = inv_scale_cost * ||x_i - y_j||^2,
 * solved by alternating log-domain updates of the dual potentials f[n], g[m]
 * ("FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section 2.1:
 * source and target potentials are updated in turn, each update a streaming
 * log-sum-exp over on-the-fly costs, O((n+m)d) working memory, the n x m
 * matrix never stored):
 *     f_i <- eps*ln a_i - eps*LSE_j((g_j - C_ij)/eps)
 *     g_j <- eps*ln b_j - eps*LSE_i((f_i - C_ij)/eps)
 * and the transport plan they define (moscot PR #846, "materialize
 * transport-matrix rows instead of pushing indicator columns", section Fix):
 *     T_ij = exp((f_i + g_j - C_ij)/eps).
 *
 * Conventions for every entry point:
 *  - Arrays named as device arrays are CUDA device pointers on the current
 *    device, owned by the caller; the library never frees them and keeps no
 *    reference to them beyond the lifetime of a plan that was given them.
 *  - Floating-point inputs are float32, contiguous, row-major ([n,d]: point i
 *    at x + i*d). Indices and counts are int64.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Work is ordered after everything already queued on it, and the
 *    results are complete on it when the call returns, unless stated otherwise.
 *  - Every call returns an int status (OT_OK = 0, warnings > 0, errors < 0),
 *    never aborts and never prints. ot_last_error_string() describes the last
 *    non-OK status of the calling thread.
 *  - No CPU fallback exists: without a usable sm_100 device every call that
 *    computes returns OT_ERR_CUDA.
 *  - Each call is wrapped in an NVTX range named after it (visible to Nsight
 *    tools; a no-op without one).
 *  - A plan keeps scratch and state between calls (workspaces, the Morton
 *    orders of the row passes, the last row call's statistics): calls on one
 *    plan must not overlap; different plans may be used from different threads.
 */
#ifndef OT_SINKHORN_H
#define OT_SINKHORN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OT_ABI_VERSION 4

#if defined(__GNUC__)
#define OT_API __attribute__((visibility("default")))
#else
#define OT_API
#endif

/* ----------------------------------------------------------- status codes */
#define OT_OK 0
#define OT_WARN_MASSLESS_ROWS 1   /* results valid; some a_i == 0 (moscot PR #846,
                                     "Behavioural changes": such rows keep no
                                     entries and do not take part in min_row) */
#define OT_ERR_INVALID_ARG (-1)   /* bad pointer/size/eps/weights/row index */
#define OT_ERR_OVERFLOW (-2)      /* a size product exceeds what the kernels index */
#define OT_ERR_CUDA (-3)          /* a CUDA runtime call failed (no device, bad stream) */
#define OT_ERR_OOM (-4)           /* workspace allocation failed */
#define OT_ERR_NONFINITE (-5)     /* a NaN/inf input, or a potential left the finite range */
#define OT_ERR_UNSUPPORTED (-6)   /* a valid request this build does not implement */

/* ------------------------------------------------------------ cost scale
 * The cost is scaled once, on the whole problem, and that resolved factor is
 * captured by the plan and reused by every later call on any row subset
 * (moscot PR #846, section Fix: re-deriving it from a subset gave 15% value
 * error). eps is absolute and applies to the scaled cost.                 */
typedef enum ot_scale {
    OT_SCALE_NONE = 0,      /* inv_scale_cost = 1 */
    OT_SCALE_MEAN = 1,      /* 1 / (mean over all n*m pairs of ||x_i - y_j||^2) */
    OT_SCALE_MAX_COST = 2,  /* 1 / (max over all n*m pairs of ||x_i - y_j||^2) */
    OT_SCALE_VALUE = 3      /* 1 / opt->scale_value */
} ot_scale;

/* ---------------------------------------------------------------- options
 * Fill with ot_options_default() and change fields; NULL means defaults.   */
typedef struct ot_options {
    int32_t warm_start;       /* 0: start from f = g = 0; 1: f, g hold the start */
    int32_t check_every;      /* iterations between host reads of the stop flag
                                 (also the CUDA-graph chunk length); default 16 */
    int32_t use_graphs;       /* 1 (default): replay the iteration loop as CUDA
                                 graphs; 0: plain launches */
    int32_t iters_per_stage;  /* annealing: iterations per eps stage (default 20) */
    double scale_value;       /* divisor for OT_SCALE_VALUE */
    double eps_init;          /* > 0 enables eps-annealing: stage k runs at
                                 max(eps, eps_init * eps_decay^k); the last stage
                                 is the first at eps (FlashSinkhorn 2, sections
                                 3.1 and C.3 anneal eps and continue at the
                                 target). 0 (default): no annealing */
    double eps_decay;         /* in (0, 1); default 0.7 */
    int32_t timing;           /* 1: time the iteration loop with CUDA events on the
                                 internal stream (ot_info.loop_ms); default 0 */
    int32_t col_splits;       /* tuning: column splits of the half-steps (0 = chosen
                                 from the problem size and the SM count) */
    int32_t rows_per_thread;  /* tuning, d <= 3: 1, 2, 4 or 8 rows per thread (0 =
                                 auto); the device-resident loop runs 1 or 2 and
                                 is not used when 4 or 8 is asked for */
    int32_t tensor_cores;     /* 16 <= d <= 64: 1 (default) computes x.y on the tcgen05
                                 tensor cores (bf16 splits, fp32 accumulation); 0 uses
                                 the CUDA-core FMA kernel */
    int32_t device_loop;      /* d <= 3: run the iterations inside one cooperative
                                 kernel per chunk (no per-half-step launches): -1
                                 (default) for problems up to 2^28 pairs, 0 never,
                                 1 always */
    int32_t reserved1;
    int32_t block_sparse;     /* d <= 3: 1 runs block-sparse fine iterations ("FlashSinkhorn 2:
                                 Block-Sparse Entropic Optimal Transport", sections 3, 3.2,
                                 A.3, B.3): the points are put in Morton order once; every
                                 iteration screens all block pairs with the bound
                                 |I||J| exp((F_I + G_J - c D_IJ)/eps) (block potential maxima,
                                 squared bounding-box distance) against rho_IJ = delta *
                                 min(smallest nonzero a_i of I, b_j of J), verifies the
                                 candidates by their exact mass, and runs both half-steps over
                                 the admitted tiles only (every tile for a block with none).
                                 The stop test compares the admitted plan's row residual with
                                 tol - MB delta sum(a), so that the full residual is <= tol.
                                 f and g are returned in the caller's order. The choice of
                                 dense or sparse updates is made on the device each iteration;
                                 the host reads the stop flag every check_every iterations;
                                 use_graphs and device_loop do not apply. 0 (default): dense
                                 iterations */
    int32_t sparse_block;     /* block size B: 128 or 256 (0 = 128 when NB * MB <= 2^27,
                                 else 256) */
    int32_t sparse_verify;    /* 1 (default): candidate tiles are verified by their exact mass;
                                 0: the box screen alone decides */
    int32_t reserved2;
    double sparse_delta;      /* delta of the tile threshold; 0 (default): tol / (4 max(NB,
                                 MB)) (section 3.2), which needs tol > 0 */
    double sparse_dense_frac; /* an iteration whose candidate tiles exceed this fraction of
                                 all NB * MB block pairs runs the dense half-steps instead
                                 (default 0.5) */
    double *resid_history;    /* optional device float64 array [resid_history_len]: entry
                                 k - 1 receives ||T 1 - a||_1 of the state after iteration k
                                 (all stages counted), as measured in the loop by the next
                                 f-update (FlashSinkhorn 2, section 3.1: the marginal residual
                                 is the convergence measure). Entries no f-update measured
                                 (the last iteration of each annealing stage but the final
                                 one; iterations beyond the run) are NaN. NULL: none */
    int64_t resid_history_len;/* entries of resid_history (0 = none) */
    uint8_t *sparse_mask_out; /* block-sparse mode, optional device array [NB * MB] (NB, MB: the
                                 blocks of x and y in Morton order; NB * MB <= sparse_mask_len,
                                 else OT_ERR_INVALID_ARG): receives the block mask of the first
                                 fine update of the solve, the one built at the starting
                                 potentials -- 1 for an admitted tile (a candidate, in an
                                 iteration that ran dense), row-major by x block. NULL: none */
    int64_t sparse_mask_len;  /* bytes available at sparse_mask_out */
} ot_options;

/* -------------------------------------------------------- solve report   */
typedef struct ot_info {
    int32_t iterations;        /* iterations of the returned state (all stages) */
    int32_t converged;         /* 1 if the tol test stopped the loop */
    int32_t stages;            /* eps stages run (1 without annealing) */
    int32_t col_splits;        /* launch shape of the f half-step: column splits */
    double residual;           /* ||T 1 - a||_1 of the returned state, measured in
                                  the loop from the next f-update (float32 LSE) */
    double inv_scale_cost;     /* resolved scale factor, captured by the plan */
    double eps;                /* resolved (final) eps, captured by the plan */
    int64_t n_massless_rows;   /* number of a_i == 0 */
    int64_t n_massless_cols;   /* number of b_j == 0 */
    int64_t half_steps;        /* half-step launches that did work (2 per iteration,
                                  plus the f-update that measures the final residual) */
    int64_t kernel_launches;   /* kernels this call launched (graph nodes included) */
    double loop_ms;            /* device time of the iteration loop, from CUDA events
                                  around each chunk (opt->timing), else 0 */
    /* block-sparse mode only (zero otherwise) */
    int64_t sparse_iterations; /* iterations run on a block mask */
    int64_t dense_iterations;  /* iterations run dense (too many candidate tiles) */
    int64_t tiles_candidate;   /* last mask: tiles that passed the box screen */
    int64_t tiles_admitted;    /* last mask: tiles admitted after verification */
    int64_t tiles_exact;       /* last mask: candidates whose exact mass was evaluated (the
                                  others fell below the threshold on a point-level bound) */
    int64_t tiles_total;       /* NB * MB block pairs */
    double omitted_bound;      /* bound on the row mass one mask omits: MB delta sum(a) */
    double verify_ms;          /* with opt->timing: device time of the tile verifications */
    double sparse_hs_ms;       /* with opt->timing: device time of the block-sparse half-steps */
    int64_t sparse_hs_launches;/* with opt->timing: block-sparse half-step launches timed */
} ot_info;

/* Opaque plan: the pages' "row materializer built once", which captures the
 * resolved eps and inv_scale_cost (moscot PR #846, section Fix). It borrows
 * x, y, a, b, f, g (read again by every later call, so they must stay alive
 * and unchanged) and owns its device workspace.                            */
typedef struct ot_plan ot_plan;

/* ABI version (OT_ABI_VERSION of the build). */
OT_API int ot_version(void);

/* Human-readable description of the calling thread's last non-OK status. */
OT_API const char *ot_last_error_string(void);

/* Default options (warm_start 0, check_every 16, use_graphs 1,
 * iters_per_stage 20, scale_value 1, eps_init 0, eps_decay 0.7, timing 0,
 * col_splits 0, rows_per_thread 0, tensor_cores 1, device_loop -1,
 * block_sparse 0, sparse_block 0, sparse_verify 1, sparse_delta 0,
 * sparse_dense_frac 0.5, resid_history NULL, resid_history_len 0,
 * sparse_mask_out NULL, sparse_mask_len 0). */
OT_API void ot_options_default(ot_options *opt);

/* ------------------------------------------------- ot_sinkhorn_pointcloud
 * Solves the problem above on one GPU.
 *  x [n,d], y [m,d], a [n], b [m]: device, float32. Weights must be finite and
 *      >= 0 with positive sums; they are not renormalised. 1 <= d <= 64.
 *  eps > 0: entropic regularisation on the scaled cost (the final eps when
 *      annealing). Held in float64 throughout, so the plan is the one of
 *      exactly this eps.
 *  scale_cost: see ot_scale.
 *  n_iters >= 0: iteration cap (one iteration = f-update then g-update; the
 *      f-update comes first, from f = g = 0 unless opt->warm_start).
 *      n_iters == 0 runs nothing and builds a plan at the given f, g (which
 *      must then be a warm start), e.g. to materialise rows of a known plan.
 *  tol: if > 0, stop after the first iteration whose ||T 1 - a||_1 <= tol;
 *      if <= 0, run exactly n_iters iterations. Missing tol is not an error.
 *      With opt->block_sparse the test is on the admitted plan's residual
 *      against tol - (the omitted-mass bound), so the full residual is <= tol.
 *  Block-sparse mode (opt->block_sparse) needs d <= 3 (else OT_ERR_UNSUPPORTED),
 *      sparse_block 0/128/256, sparse_delta >= 0 (0 needs tol > 0) and
 *      sparse_dense_frac in [0, 1] (else OT_ERR_INVALID_ARG), and block counts
 *      whose mask fits (NB * MB <= 2^32, NB <= 2^21; else OT_ERR_UNSUPPORTED).
 *  f [n], g [m]: device float32 outputs (and inputs for a warm start). A
 *      massless row/column gets -inf.
 *  plan_out: if non-NULL, receives a plan to pass to the calls below; free it
 *      with ot_plan_destroy. If NULL, the workspace is freed before returning.
 *  info: if non-NULL, receives the report.
 * Returns OT_OK, OT_WARN_MASSLESS_ROWS, or an error (then *plan_out = NULL and
 * f, g are unspecified). Synchronises `stream` (it reads scalars back). */
OT_API int ot_sinkhorn_pointcloud(const float *x, const float *y, const float *a, const float *b,
                           int64_t n, int64_t m, int32_t d, double eps, ot_scale scale_cost,
                           int32_t n_iters, double tol, float *f, float *g, void *stream,
                           const ot_options *opt, ot_plan **plan_out, ot_info *info);

/* ------------------------------------------------ ot_sinkhorn_pointcloud_host
 * ot_sinkhorn_pointcloud for a caller that holds its arrays in HOST memory:
 * x, y, a, b (and f, g with opt->warm_start) are copied to the device on
 * `stream`, the problem is solved as above, and f, g are copied back into the
 * caller's host arrays before the call returns. Host arrays may be pageable or
 * pinned (pinned ones copy asynchronously and faster). The device copies come
 * from the library's workspace cache; if plan_out is non-NULL the plan owns
 * them (its row calls then take DEVICE row_idx / out arrays as usual) and
 * ot_plan_destroy returns them, otherwise they are released before the call
 * returns. Arguments, statuses and info are those of ot_sinkhorn_pointcloud.
 * Synchronises `stream`. */
OT_API int ot_sinkhorn_pointcloud_host(const float *x, const float *y, const float *a,
                                       const float *b, int64_t n, int64_t m, int32_t d, double eps,
                                       ot_scale scale_cost, int32_t n_iters, double tol, float *f,
                                       float *g, void *stream, const ot_options *opt,
                                       ot_plan **plan_out, ot_info *info);

/* ---------------------------------------------------- ot_marginal_residual
 * row_l1 = sum_i |sum_j T_ij - a_i|, col_l1 = sum_j |sum_i T_ij - b_j| at the
 * plan's current f, g (FlashSinkhorn 2, sections 3.1 and C.4: the residual is
 * evaluated at the returned potentials; section D.3: the exponent is built in
 * float64 from the coordinates). Each T_ij: float64 exponent, float32 exp.
 * Deterministic (fixed reduction order). row_l1/col_l1: host pointers, either
 * may be NULL. Synchronises `stream`.
 * Tile screen (d <= 3; also in the min_row and count passes): rows and columns
 * are visited in Morton order, and a tile of 32 rows x 256 columns whose bound
 * kappa (max f + max g) - kappa c dist(boxes)^2 on the base-2 exponent is below
 * -127 is skipped -- each of its entries is below 2^-126, where the entry is
 * exactly 0 -- so the results are those of visiting every entry (sums up to
 * summation order); ot_row_pass_stats reports how much was evaluated. */
OT_API int ot_marginal_residual(const ot_plan *plan, double *row_l1, double *col_l1, void *stream);

/* ------------------------------------------------------ ot_materialize_rows
 * out[r*m + j] = T_{row_idx[r], j} for r < k, j < m (moscot PR #846, section
 * Fix: entropic rows exp((f_i + g_j - C_ij)/eps) with the captured scale and
 * eps; O(k*m) memory). row_idx [k]: device int64, each in [0, n) (repeats
 * allowed); out [k,m]: device float32, row-major. The exponent is assembled
 * in float64; the value is rounded to float32, with entries of 2^128 or more
 * returned as +inf and entries below 2^-126 (1.2e-38, the smallest normal
 * float) as 0 (the same holds for every row call). A row index out of range makes
 * the call return OT_ERR_INVALID_ARG (checked on the device, no fault); the
 * rows with valid indices are still written. Synchronises `stream`. */
OT_API int ot_materialize_rows(const ot_plan *plan, const int64_t *row_idx, int64_t k, float *out,
                        void *stream);

/* ------------------------------------------------ ot_materialize_rows_lowrank
 * Rows of a low-rank coupling (moscot PR #846, section Fix: for low-rank
 * outputs the rows are (Q diag(1/g) R^T)[rows], a matrix product that never
 * touches a geometry):
 *     out[t*m + j] = sum_k Q[i*r + k] * R[j*r + k] / g[k],   i = row_idx[t].
 *  Q [n,r], R [m,r], g [r]: device float32, row-major (g > 0); 1 <= r <= 128.
 *  row_idx [k]: device int64 in [0, n); out [k,m]: device float32, row-major.
 * Accumulated in float32 in k order: relative error <= r * 2^-24 for the
 * nonnegative factors of a low-rank coupling. No plan, no allocation beyond a
 * cached flag. A row index out of range returns OT_ERR_INVALID_ARG (checked on
 * the device; that row is not written). Synchronises `stream`. */
OT_API int ot_materialize_rows_lowrank(const float *Q, const float *R, const float *g, int64_t n,
                                       int64_t m, int32_t r, const int64_t *row_idx, int64_t k,
                                       float *out, void *stream);

/* ------------------------------------------------- ot_materialize_rows_lrcost
 * Entropic rows on a low-rank cost geometry (moscot PR #846, section Fix: the
 * cost rows of an LRCGeometry are cost_1[rows] @ cost_2^T + bias):
 *     C_ij = inv_scale_cost * (sum_k cost1[i*r + k] * cost2[j*r + k] + bias),
 *     out[t*m + j] = exp((f_i + g_j - C_ij) / eps),   i = row_idx[t],
 * with the caller's resolved inv_scale_cost and eps (a subset never
 * re-derives them). cost1 [n,r], cost2 [m,r], f [n], g [m]: device float32;
 * 1 <= r <= 128. The dot products and the exponent are assembled in float64
 * (as ot_materialize_rows), the value rounded to float32; f_i or g_j = -inf
 * gives 0. row_idx / out and errors as ot_materialize_rows_lowrank.
 * Synchronises `stream`. */
OT_API int ot_materialize_rows_lrcost(const float *cost1, const float *cost2, const float *f,
                                      const float *g, int64_t n, int64_t m, int32_t r, double bias,
                                      double inv_scale_cost, double eps, const int64_t *row_idx,
                                      int64_t k, float *out, void *stream);

/* ------------------------------------------------------ ot_sparsify_min_row
 * The exact min_row threshold (moscot PR #846, "Behavioural changes"):
 *     thr = min over rows with a_i > 0 of max_j T_ij,
 * with every T_ij computed by the same float path as ot_materialize_rows, so
 * that keeping T_ij >= thr leaves every massful row non-empty. Massless rows
 * (a_i == 0) keep nothing and take no part. block_rows (> 0, or 0 = all rows)
 * only sets how many rows one launch covers (raised to sixteen waves of the
 * GPU when smaller); it never changes a result.
 *  thr_out: host float (+inf if every row is massless).
 *  row_counts: device int64 [n] or NULL: kept entries per row.
 *  nnz_out, n_massless_out, argmin_out: host int64 or NULL (argmin_out: the
 *      row attaining thr, smallest index on ties; -1 if none).
 * Returns OT_WARN_MASSLESS_ROWS if any row is massless. Synchronises `stream`. */
OT_API int ot_sparsify_min_row(const ot_plan *plan, int64_t block_rows, float *thr_out,
                        int64_t *row_counts, int64_t *nnz_out, int64_t *n_massless_out,
                        int64_t *argmin_out, void *stream);

/* ---------------------------------------------------------- ot_sparsify_csr
 * The plan thresholded at thr (moscot PR #846, "Behavioural changes": the
 * entries T_ij >= thr are kept, rows with a_i == 0 keep nothing), written in
 * compressed-row form for an [n, m] matrix: row i's kept columns, increasing,
 * in col_idx[row_ptr[i] .. row_ptr[i+1]) and their values in vals. Values and
 * comparisons come from the same float path as ot_materialize_rows and
 * ot_sparsify_min_row: with thr = its thr_out, row_ptr differences are its
 * row_counts and the total its nnz_out (use that to size col_idx / vals).
 * The pages describe the threshold and the kept set; the compressed-row layout
 * is this library's (the common sparse format; no page fixes one).
 *  block_rows: rows per pass (> 0, or 0 = all); never changes a result.
 *  row_ptr [n+1] int64, col_idx [capacity] int64, vals [capacity] float32:
 *      device, caller-owned outputs.
 *  nnz_out: host int64 or NULL: the number of kept entries (set also when it
 *      exceeds capacity).
 * Returns OT_ERR_OVERFLOW, with row_ptr written and col_idx / vals untouched,
 * when the kept entries exceed capacity; OT_ERR_CUDA if the count and write
 * passes ever disagreed (not expected: both call one entry function).
 * Synchronises `stream`. */
OT_API int ot_sparsify_csr(const ot_plan *plan, int64_t block_rows, float thr, int64_t *row_ptr,
                           int64_t *col_idx, float *vals, int64_t capacity, int64_t *nnz_out,
                           void *stream);

/* ------------------------------------------- ot_marginal_residual_noalloc
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory when they need a residual -- a process
 * whose device memory is wholly owned by another allocator (a framework's
 * caching pool, or a budget fixed at start-up), or a tight loop in which a
 * cudaMalloc/cudaFree would stall every stream on the device. It returns the
 * same two sums as ot_marginal_residual, at the given f, g, without a plan and
 * without allocating anything: its scratch is a fixed array of
 * OT_NOALLOC_MAX_POINTS/8 + 2 doubles (1 MiB) in the library's device image,
 * which every device that loads the library keeps until the process exits.
 *  x [n,d], y [m,d], a [n], b [m], f [n], g [m]: device float32, caller-owned.
 *  eps > 0 and inv_scale_cost > 0: the resolved values (e.g. ot_info.eps and
 *      ot_info.inv_scale_cost of the solve), so that C = inv_scale_cost*|x-y|^2.
 *  row_l1, col_l1: host doubles (either may be NULL).
 * n or m above OT_NOALLOC_MAX_POINTS returns OT_ERR_UNSUPPORTED with a message.
 * The first call on a device looks up the scratch's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. The address is kept for the life of the process, so the device must
 * not be reset (cudaDeviceReset) after that first call. All calls on a device share the scratch and each call overwrites
 * every slot it reads, so nothing carries over from the previous call; but
 * calls whose GPU work overlaps (e.g. from two host threads on two streams)
 * race on it. Synchronises `stream`. Calls no allocating routine.           */
#define OT_NOALLOC_MAX_POINTS (1 << 20)
OT_API int ot_marginal_residual_noalloc(const float *x, const float *y, const float *a,
                                        const float *b, const float *f, const float *g,
                                        int64_t n, int64_t m, int32_t d, double eps,
                                        double inv_scale_cost, double *row_l1, double *col_l1,
                                        void *stream);

/* ------------------------------------------------------------ sharded solve
 * The solve split by rows across several GPUs ("FlashSinkhorn 2: Block-Sparse
 * Entropic Optimal Transport", section 5: at 10^10 points one measure exceeds a
 * single GPU, so the work is spread over several). Every rank holds x, y, a, b
 * in full and updates one contiguous range of x's rows in the f-update and of
 * y's rows in the g-update; between the half-steps the caller exchanges the
 * updated ranges (an all-gather of the potential, e.g. NCCL over NVLink) and,
 * for a stopping test, sums the ranks' residual partials (an all-reduce). The
 * kernels are those of ot_sinkhorn_pointcloud; the half-step of a row tile
 * depends only on that tile's rows and the other side's whole potential, so a
 * tile-aligned split with the same opt->col_splits and opt->rows_per_thread
 * gives the unsplit solve's potentials bit for bit. */

/* ot_max_sqdist: *out = max over i in [x_lo, x_hi), j < m of ||x_i - y_j||^2,
 * evaluated exactly as the OT_SCALE_MAX_COST pass does (float32 on coordinates
 * shifted by the midpoint of the clouds' means), so the max over ranks of their
 * ranges' values is the unsplit max_cost, and OT_SCALE_VALUE with that value
 * resolves the same inv_scale_cost. x [n,d], y [m,d]: device float32; out:
 * host float (0 for an empty range). Synchronises `stream`. */
OT_API int ot_max_sqdist(const float *x, const float *y, int64_t n, int64_t m, int32_t d,
                         int64_t x_lo, int64_t x_hi, float *out, void *stream);

/* ot_shard_plan_create: a plan for the rows [x_lo, x_hi) of x and [y_lo, y_hi)
 * of y (0 <= lo <= hi <= n or m; lo a multiple of 8; empty ranges allowed),
 * with eps and the scale resolved as in ot_sinkhorn_pointcloud (pass the
 * max_cost of all ranks as OT_SCALE_VALUE, see ot_max_sqdist). x, y, a, b are
 * borrowed as by a solve. Honoured options: scale_value, col_splits,
 * rows_per_thread, tensor_cores; block_sparse is OT_ERR_UNSUPPORTED. info (may
 * be NULL) receives inv_scale_cost, eps, the massless counts and col_splits.
 * The plan serves ot_shard_half_step only (row calls refuse it); free it with
 * ot_plan_destroy. Synchronises `stream`. */
OT_API int ot_shard_plan_create(const float *x, const float *y, const float *a, const float *b,
                                int64_t n, int64_t m, int32_t d, double eps, ot_scale scale_cost,
                                int64_t x_lo, int64_t x_hi, int64_t y_lo, int64_t y_hi, void *stream,
                                const ot_options *opt, ot_plan **plan_out, ot_info *info);

/* ot_shard_half_step: one half-step over the plan's rows of one side.
 *  side 0 (f-update): other = g [m] (all of it), cur = f [n] before the update
 *      (the rows of the range are read), out = f [n]: the range's rows are
 *      written; out may equal cur.
 *  side 1 (g-update): other = f [n], cur / out = g [m] likewise.
 *  resid: host double or NULL: the range's part of ||T1 - a||_1 (side 0) or of
 *      ||T^T 1 - b||_1 (side 1) at the state BEFORE the update (cur and other),
 *      the terms the single-GPU solve sums for its stopping test; the sum over
 *      ranks is the whole residual.
 * Work is queued on `stream` after what is already there; the call returns at
 * once unless resid is non-NULL or the range is non-empty (then it reads the
 * plan's status back and synchronises). A potential that leaves the finite
 * range returns OT_ERR_NONFINITE. */
OT_API int ot_shard_half_step(ot_plan *plan, int32_t side, const float *other, const float *cur,
                              float *out, double *resid, void *stream);

/* Row calls over a range of rows, for the same split (section 5 of FlashSinkhorn
 * 2 again): the rows of the plan are independent, so each rank reduces its own
 * and one all-reduce combines them. They take a plan of ot_sinkhorn_pointcloud
 * (on every rank, with the gathered potentials: n_iters = 0 with warm_start),
 * use the same kernels and float path as the whole-plan calls, and with the
 * full range give exactly their values. A range outside the plan returns
 * OT_ERR_INVALID_ARG; block_rows as in ot_sparsify_min_row. All synchronise
 * `stream`.
 *
 * ot_marginal_residual_range: *row_part = sum over i in [row_lo, row_hi) of
 *     |sum_j T_ij - a_i|, *col_part = sum over j in [col_lo, col_hi) of
 *     |sum_i T_ij - b_j| (host doubles, NULL ok); the sums over ranks of the
 *     parts are ot_marginal_residual's two values, in another summation order.
 * ot_min_row_range: pass A of ot_sparsify_min_row over rows [row_lo, row_hi)
 *     (moscot PR #846, "Behavioural changes"): *thr_out = min over the range's
 *     rows with a_i > 0 of max_j T_ij (+inf if none), *argmin_out = the global
 *     index of the row attaining it (smallest on ties, -1 if none),
 *     *n_massless_out = massless rows in the range. The min over ranks of
 *     thr_out is ot_sparsify_min_row's thr (and the smallest argmin among the
 *     ranks attaining it its argmin).
 * ot_kept_counts_range: pass B at a given thr (not NaN): row_counts (device
 *     int64 [row_hi - row_lo], NULL ok) = #{j : T_ij >= thr} per row of the
 *     range, 0 for a massless row; *nnz_out = their sum. */
/* ot_row_pass_stats: the tile screen's work in the plan's last row call
 * (ot_marginal_residual[_range], ot_sparsify_min_row, ot_min_row_range,
 * ot_kept_counts_range, the count pass of ot_sparsify_csr): tiles of 32 rows x
 * 256 columns evaluated, and those a visit of every entry evaluates (their
 * ratio is the share of the plan's entries the call computed). 0 and 0 for
 * d > 3 (no screen). Host outputs, NULL ok; no device work. */
OT_API int ot_row_pass_stats(const ot_plan *plan, int64_t *chunks_visited, int64_t *chunks_total);
OT_API int ot_marginal_residual_range(const ot_plan *plan, int64_t row_lo, int64_t row_hi,
                                      int64_t col_lo, int64_t col_hi, double *row_part,
                                      double *col_part, void *stream);
OT_API int ot_min_row_range(const ot_plan *plan, int64_t row_lo, int64_t row_hi, int64_t block_rows,
                            float *thr_out, int64_t *argmin_out, int64_t *n_massless_out,
                            void *stream);
OT_API int ot_kept_counts_range(const ot_plan *plan, int64_t row_lo, int64_t row_hi,
                                int64_t block_rows, float thr, int64_t *row_counts, int64_t *nnz_out,
                                void *stream);

/* Plans take their device workspace, pinned read-back buffer and internal
 * stream from a per-device cache and return them there when destroyed, so
 * repeated solves do not pay cudaMalloc/cudaFree (which synchronises the
 * device) each time; the cache keeps at most 4 GiB of device memory per device.
 * ot_trim_cache releases everything it holds (live plans are unaffected). */
OT_API void ot_trim_cache(void);

/* Returns the plan's workspace to the cache (NULL is a no-op). Does not touch
 * borrowed arrays. Waits for the plan's internal stream. */
OT_API void ot_plan_destroy(ot_plan *plan);

#ifdef __cplusplus
}
#endif
#endif /* OT_SINKHORN_H */
