// runtime.h -- host-side declarations of the kernel launchers (internal).
#pragma once
#include <cuda.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace ot {

// An NVTX range around one C-ABI call, so profilers show each call of the
// library by name (NVTX v3 is header-only: without a tool attached the push
// and pop cost a branch).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// api.cu: sets the thread's last-error text and returns code
int set_error(int code, const char *fmt, ...);

// pool.cu: cached device workspaces, pinned host buffers and streams (an
// allocation is made on the current device; a release names the device the
// resource belongs to)
cudaError_t pool_device_alloc(void **ptr, size_t bytes, size_t *got);
void pool_device_free(void *ptr, size_t bytes, int device);
cudaError_t pool_host_alloc(void **ptr, size_t bytes);
void pool_host_free(void *ptr, size_t bytes);
cudaError_t pool_stream(cudaStream_t *s);
void pool_stream_release(cudaStream_t s, int device);

// halfstep.cu
int halfstep_blocks_per_sm(int kind, int dim, int rpt);
cudaError_t launch_halfstep(int kind, int dim, int rpt, const HalfStep &A, int grid,
                            cudaStream_t s);

// loop.cu (device-resident iterations, d <= 3, 2 rows per thread)
struct LoopArgs {
    HalfStep f[2];          // f-update with the f buffers at parity 0 / 1
    HalfStep g[2];          // g-update (same buffers; indexed like f)
    int iters;              // iterations this launch may run
    int parity0;            // parity of the f buffer holding the current state
    unsigned *bar_count;    // grid barrier: arrivals
    unsigned *bar_gen;      // grid barrier: generation
    double *blk_resid;      // [grid] residual partial of each block
    unsigned long long wait_ns;  // grid-barrier time limit
    int withhold_block;     // failure tests only: this block returns before its first
                            // barrier arrival (-1: none)
};
int loop_blocks_per_sm(int d, int rpt);
cudaError_t launch_loop(int d, int rpt, const LoopArgs &L, int grid, cudaStream_t s);

// halfstep_tc.cu (16 <= d <= 64: tensor-core path)
int tc_ksteps(int d);
int tc_slabs(int d);
cudaError_t tc_setup(int d);
cudaError_t launch_halfstep_tc(int d, const HalfStep &A, const CUtensorMap *tmA,
                               const CUtensorMap *tmB, int grid, cudaStream_t s);
cudaError_t launch_tc_tables(const float *p, const float *pot, int64_t cnt, int64_t pad, int d,
                             int dpf, int kp, const double *o, const Params *prm, float *rowtab,
                             void *arow, void *bcol, cudaStream_t s);
int make_operand_map(CUtensorMap *map, void *base, int64_t rows, int kp);

// prep.cu
cudaError_t launch_coord_stats(const float *v, int64_t cnt, int d, double *part, double *part2,
                               double *out, double *out2, int *flags,
                               unsigned long long *zero_count, cudaStream_t s);
cudaError_t launch_max_cost(const float *x, const float *y, int64_t n, int64_t m, int d,
                            const double *o, unsigned *out_bits, cudaStream_t s);
cudaError_t launch_set_params(Params *prm, double eps, double c, double tol, double *hist,
                              int64_t hist_off, int64_t hist_len, cudaStream_t s);
cudaError_t launch_reset_state(State *st, cudaStream_t s);
cudaError_t launch_tables(const float *p, const float *pot, int64_t cnt, int64_t cnt_pad, int d,
                          int dp, const double *o, const Params *prm, float *rowtab,
                          float *coltab, int layout, cudaStream_t s);

// rows.cu
struct MatArgs {
    const float *x, *f;
    const double *dcol, *o;
    const Params *prm;
    const int64_t *row_idx;
    int64_t k, n, m;
    int d, vec;
    float *out;
    int *bad;
};
struct RowPassArgs {
    const float *pts, *pot, *w;
    const double *dcol, *o;
    const Params *prm;
    int64_t row_begin, row_end, cols;  // positions [row_begin, row_end) of the pass
    int d;
    float thr;
    float *rowmax;
    int64_t *counts;
    double *part;
    const int64_t *rperm;  // position -> row (NULL: the identity)
    const double *csum;    // chunk summaries of the column table for the tile screen (NULL: none)
    unsigned long long *visited;  // += chunks the pass evaluated (NULL: not counted)
};
struct LrArgs {
    const float *fa, *fb;       // row factors [n, r] and column factors [m, r]
    const float *g;             // coupling: the middle diagonal [r]
    const float *f, *gp;        // cost: potentials [n], [m]
    int64_t n, m, k;
    int r;
    const int64_t *row_idx;
    double bias, kc, kappa;     // cost: bias, kappa * inv_scale_cost, kappa = log2(e) / eps
    float *out;
    int vec;
    int *bad;
};
constexpr int kLrMaxRank = 128;
size_t lowrank_smem_bytes(int mode, int r);
cudaError_t launch_lowrank_rows(int mode, const LrArgs &L, cudaStream_t s);
struct CsrArgs {
    const float *pts, *pot, *w;
    const double *dcol, *o;
    const Params *prm;
    int64_t row_begin, row_end, cols;
    int d;
    float thr;
    const int64_t *row_ptr;   // [n+1], exclusive prefix sum of the kept counts
    int64_t *col_idx;
    float *vals;
    int *bad;                 // set if a row keeps a different number of entries
};
cudaError_t launch_csr_write(const CsrArgs &C, cudaStream_t s);
// row_ptr[0] = 0, row_ptr[i+1] = counts[0] + ... + counts[i]; tmp holds
// scan_tmp_count(n) int64
int64_t scan_tmp_count(int64_t n);
cudaError_t launch_row_ptr_scan(const int64_t *counts, int64_t n, int64_t *row_ptr, int64_t *tmp,
                                cudaStream_t s);
// sparse.cu (block-sparse fine updates, d <= 3)
struct MortonArgs {
    double lo[3];   // joint bounding box, lower corner
    double s[3];    // 2^bits / (hi - lo), 0 for a flat coordinate
    int bits;       // 30 / d
    int d;
};
struct BlockSum {     // one block of B consecutive points (Morton order)
    double lo[3], hi[3];  // bounding box (0 past d)
    double pmax;          // largest potential (refreshed every iteration)
    double l2gsum;        // log2 sum_j 2^(kappa pot_j) over the block (refreshed every iteration)
    double lnw, l2w;      // ln and log2 of the smallest nonzero weight (+inf: none)
    double lncnt;         // ln of the block's point count
};
constexpr int kModeSparse = 0, kModeDense = 1, kModeStopped = 2;
struct ScreenArgs {
    const State *st;           // nothing is screened once the solve has stopped
    const BlockSum *rs, *cs;   // row (x) and column (y) blocks
    int64_t nb, mb;
    int d;
    double c, eps, ln_delta;
    uint8_t *mask;             // [nb][mb]: 1 for a candidate
    int64_t *cnt, *cnt_t;      // candidates per row block / per column block (zeroed before)
    unsigned long long *total; // candidates (zeroed before)
};
struct VerifyArgs {
    const float4 *coltab;      // the column side's half-step table
    const float *rowtab;       // x' rows, 4 floats each
    const float *pot;          // f
    const float *pts;          // the row side's points (Morton order), [rows][d]
    const Params *prm;
    const BlockSum *rs, *cs;
    int64_t rows, cols_pad, nb, mb;
    double l2_delta;
    uint8_t *mask;             // candidates in, admitted tiles out
    const int64_t *cptr;       // candidates of row block p: clist[cptr[p] .. cptr[p+1])
    const int *clist;
    int segs;                  // work items per row block
    int64_t *cnt, *cnt_t;      // out: admitted per row block (zeroed before); in/out: per
                               // column block
    unsigned long long *total; // admitted tiles (zeroed before)
    unsigned long long *exact; // tiles whose exact mass was evaluated (zeroed before)
};
int sparse_blocks_per_sm(int which, int d, int rpt);  // which: 0 half-step, 1 verification
cudaError_t launch_box(const float *p, int64_t cnt, int d, unsigned *lohi, cudaStream_t s);
cudaError_t launch_morton_sort(const float *p, int64_t cnt, int64_t n2, const MortonArgs &M,
                               unsigned long long *keys, cudaStream_t s);
cudaError_t launch_gather(const unsigned long long *keys, int64_t cnt, int d, const float *p,
                          const float *w, const float *pot, int64_t *perm, float *ps, float *ws,
                          float *pots, cudaStream_t s);
cudaError_t launch_scatter(const float *in, const int64_t *perm, int64_t cnt, float *out,
                           cudaStream_t s);
cudaError_t launch_block_static(const float *ps, const float *ws, int64_t cnt, int d, int B,
                                BlockSum *bs, cudaStream_t s);
cudaError_t launch_block_max(const float *pot, int64_t cnt, int B, double kappa, BlockSum *bs,
                             cudaStream_t s);
cudaError_t launch_screen(const ScreenArgs &S, cudaStream_t s);
cudaError_t launch_sparse_prep(int64_t *cnt, int64_t nb, int64_t *cnt_t, int64_t mb,
                               unsigned long long *ctr, int nctr, const State *st, cudaStream_t s);
// mode[0]: this iteration's kind, mode[1]: the last counted one; n_mode[kind] += count
cudaError_t launch_decide(const unsigned long long *cand, double limit, const State *st, int *mode,
                          unsigned long long *n_mode, int count, cudaStream_t s);
// the verification fused with the f-update (A: the f half-step, V.segs splits)
cudaError_t launch_verify(int d, int rpt, const HalfStep &A, const VerifyArgs &V, int grid,
                          cudaStream_t s);
cudaError_t launch_mask_list(const uint8_t *mask, int64_t rows, int64_t cols, const int64_t *ptr,
                             int *list, cudaStream_t s);
cudaError_t launch_transpose_bytes(const uint8_t *in, int64_t rows, int64_t cols, uint8_t *out,
                                   cudaStream_t s);
cudaError_t launch_halfstep_sparse(int d, int rpt, const HalfStep &A, int grid, cudaStream_t s);

cudaError_t launch_dcol(const float *p, const float *pot, int64_t cnt, int d, const double *o,
                        const Params *prm, double *dcol, cudaStream_t s, const int64_t *perm = nullptr);
// chunks of the row passes' column table (256 columns each) and their summaries
int64_t chunk_count(int64_t cols);
cudaError_t launch_chunk_summary(const double *dcol, int64_t cnt, int d, const Params *prm,
                                 double *csum, cudaStream_t s);
cudaError_t launch_perm_from_keys(const unsigned long long *keys, int64_t cnt, int64_t off,
                                  int64_t *perm, cudaStream_t s);
cudaError_t launch_materialize(const MatArgs &M, cudaStream_t s);
cudaError_t launch_rowpass(int op, const RowPassArgs &R, cudaStream_t s);
// residual partials one pass over `rows` rows writes (blocks of the pass)
int64_t rowpass_blocks(int64_t rows, int d);
int64_t rowpass_rows_per_block(int d);
cudaError_t launch_min_row_reduce(const float *rowmax, const float *w, int64_t n, float *thr,
                                  int64_t *argmin, int64_t *n_massless, cudaStream_t s);
cudaError_t launch_sum_i64(const int64_t *v, int64_t cnt, int64_t *out, cudaStream_t s);
cudaError_t launch_sum_f64(const double *v, int64_t cnt, double *out, cudaStream_t s);

}  // namespace ot
