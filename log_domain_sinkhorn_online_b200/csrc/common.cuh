// common.cuh -- device-side helpers and the structs shared by the kernels and
// the host runtime of the B200 Sinkhorn library (internal; not installed).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace ot {

// ------------------------------------------------------------ constants --
constexpr int kMaxD = 64;            // largest point dimension this build supports
constexpr double kLog2e = 1.4426950408889634073599246810019;
constexpr double kLn2 = 0.69314718055994530941723212145818;

// Low-d half-step tiling: 128 threads x R rows each (R = 2, 4 or 8, chosen per
// problem); the column table is streamed through shared memory 256 columns at
// a time.
constexpr int kHsThreads = 128;
constexpr int kHsChunk = 256;

// Generic-d half-step tiling: 128 threads x 2 rows, 64-column chunks.
constexpr int kGnThreads = 128;
constexpr int kGnRows = 2;
constexpr int kGnTile = kGnThreads * kGnRows;
constexpr int kGnChunk = 64;

// every column table is padded (G = -inf) to a multiple of this many columns;
// column splits are multiples of it too, so no inner loop has a tail
constexpr int kColPad = 8;

// A lazily refreshed running maximum may lag the true one by this much (base-2
// units): every summed term is then at most 2^8, far from float overflow. The
// refresh is decided by a warp vote: a per-lane branch in the inner loop costs
// one more instruction on the ex2 pipe per test (measured: ~12% of the pipe's
// work at d <= 3); after the vote every lane moves its maximum to max(m, cm),
// which rescales by exactly 1 where nothing changed.
constexpr float kLazyMax = 8.0f;
constexpr float kNegBig = -1.0e30f;  // finite "no column seen yet" maximum

// -------------------------------------------------------- device structs --
// Per-stage scalars, resident on the device so one captured graph serves all
// annealing stages.
struct Params {
    double eps;       // entropic regularisation (scaled cost units)
    double kappa;     // log2(e) / eps
    double c;         // inv_scale_cost
    double tol;       // stopping tolerance on ||T1 - a||_1 (<= 0: none)
    double *hist;     // optional residual history: hist[hist_off + k - 1] = ||T1 - a||_1
                      // after iteration k of this stage (k < hist_len - hist_off)
    int64_t hist_off; // iterations of the earlier stages
    int64_t hist_len;
};

// Records the in-loop row residual `v` of the state after iteration `k` of the
// current stage in the optional history (one thread calls it).
__device__ __forceinline__ void record_residual(const Params *prm, int k, double v) {
    double *h = prm->hist;
    if (h && k >= 1) {
        const int64_t idx = prm->hist_off + (int64_t)k - 1;
        if (idx < prm->hist_len) h[idx] = v;
    }
}

// Solver state written by the kernels' last-finishing blocks.
struct State {
    int stop;           // set when the tol test passed: later half-steps return at once
    int nonfinite;      // a massful row produced a non-finite potential
    int bad_index;      // a row index outside [0, n) was given to a row kernel
    int iter_done;      // completed iterations in the current stage
    int conv_iter;      // iteration count at which tol was met (-1: not yet)
    int wait_timeout;   // a bounded device wait (grid barrier, mbarrier) gave up (error)
    double resid[2];    // last in-loop marginal residual of each side (0: rows, 1: cols)
    unsigned tiles_done[2];
    unsigned work[2];   // work-item counters of the per-launch CUDA-core half-steps (f, g side)
};

// Arguments of one half-step launch (the same kernel serves f and g: rows are
// the side being updated, columns the other side).
struct HalfStep {
    const float4 *coltab;      // column table (layout depends on the kernel)
    const float *rowtab;       // row coordinates minus the shift, [rows_pad][dp]
    int64_t rows;              // rows updated (n for the f side, m for g; a shard's count)
    int64_t row_off;           // index of the first updated row in its cloud (shards; 0 otherwise)
    int64_t cols_pad;          // padded column count (multiple of kColPad)
    int64_t cols_per_split;    // multiple of kColPad (the last chunk of a split may be partial)
    int splits;                // column splits S
    int tiles;                 // row tiles
    int tile_rows;             // rows per tile (partials are [splits][tiles*tile_rows])
    int dp;                    // row-table stride in floats
    int side;                  // 0: f-update (runs the stop test), 1: g-update
    float2 *part;              // [splits][tiles*tile] (running max, sum) partials
    unsigned *tile_cnt;        // [tiles] splits finished, reset by the last one
    double *tile_resid;        // [tiles] residual partial of each tile
    const float *w;            // weights of the updated side (a or b)
    const float *pot_old;      // potential before the update
    float *pot_new;            // potential after the update
    float *next_col;           // column table of the other half-step (float view)
    int64_t nxt_a, nxt_l, nxt_b;  // column i's G' sits at (i>>1)*nxt_a + (i&1)*nxt_l + nxt_b
    int nxt_bf16;              // 1: the other table is bf16 and G is stored as three bf16
                               //    terms at element i*nxt_a + nxt_b (tensor-core path)
    const Params *prm;
    State *st;
    // block-sparse half-step only: the updated side's blocks list their column
    // tiles in sp_idx[sp_ptr[t] .. sp_ptr[t+1]); an empty list means all
    // sp_coltiles tiles
    const int64_t *sp_ptr;
    const int *sp_idx;
    int sp_coltiles;
    const int64_t *sp_fallback;  // non-null: only blocks t with sp_fallback[t] == 0 are updated
    const int *gate;             // non-null: the launch does nothing unless *gate == gate_val
    int gate_val;                //   (block-sparse iterations choose dense or sparse on the device)
    // tensor-core half-step only: polls of one mbarrier wait before it gives up,
    // and (failure tests only) block 0's producer skipping its first column-chunk load
    unsigned wait_polls;
    int withhold;
};

// ------------------------------------------------------ device helpers --
__device__ __forceinline__ float ex2_approx(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// max of three floats in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ int ld_volatile(const int *p) {
    return *reinterpret_cast<const volatile int *>(p);
}

}  // namespace ot
