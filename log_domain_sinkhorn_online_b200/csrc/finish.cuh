// finish.cuh -- the tile finalizer shared by every fused half-step kernel.
//
// After the column splits of a row tile have written their (running max, sum)
// per row, the block that finishes last (atomic ticket, no waiting) merges
// them in split order, writes the new potential, the other half-step's column
// term, and the rows' terms of the marginal residual at the previous state;
// the last tile sums the tile residuals in tile order (deterministic) and runs
// the stop test.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace ot {

// New potential of one row from its merged (max M, sum S) over all columns:
// writes pot_new[row] and the other half-step's column term, returns the
// row's residual term |sum_j T_ij(old) - w_row|; *bad is set for a massful row
// whose potential is not finite.
__device__ __forceinline__ double finish_row(const HalfStep &A, int64_t row, float M, double S,
                                             double eps, double kappa, double c, bool *bad) {
    const float *xr = A.rowtab + row * (int64_t)A.dp;
    double nrm = 0.0;
    for (int q = 0; q < A.dp; ++q) nrm += (double)xr[q] * (double)xr[q];
    const double wi = (double)A.w[row];
    double pot = 0.0, term = 0.0;
    if (wi == 0.0) {
        pot = -INFINITY;  // massless row: empty row of the plan
    } else if (!(S > 0.0)) {
        pot = INFINITY;   // every column is massless: no finite potential
        *bad = true;
    } else {
        const double L = (double)M + log2(S) - kappa * c * nrm;
        pot = eps * log(wi) - L / kappa;
        const double old = (double)__ldcg(A.pot_old + row);
        term = fabs(exp2(kappa * old + L) - wi);
    }
    const float pf = (float)pot;
    if (wi != 0.0 && !isfinite(pf)) *bad = true;
    A.pot_new[row] = pf;
    const double Gn = (wi == 0.0) ? -INFINITY : kappa * ((double)pf - c * nrm);
    if (A.nxt_bf16) {
        // three bf16 terms whose sum carries G to ~24 bits (-inf: first term only)
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(A.next_col) + row * A.nxt_a + A.nxt_b;
        const __nv_bfloat16 g1 = __double2bfloat16(Gn);
        const double r1 = isfinite(Gn) ? Gn - (double)__bfloat162float(g1) : 0.0;
        const __nv_bfloat16 g2 = __double2bfloat16(r1);
        const __nv_bfloat16 g3 = __double2bfloat16(r1 - (double)__bfloat162float(g2));
        dst[0] = g1;
        dst[1] = g2;
        dst[2] = g3;
    } else {
        A.next_col[(row >> 1) * A.nxt_a + (row & 1) * A.nxt_l + A.nxt_b] = (float)Gn;
    }
    return term;
}

// Barrier among the THREADS threads that run finish_tile: the whole block
// (BAR == 0) or a named barrier BAR (warp-specialised kernels).
template <int THREADS, int BAR>
__device__ __forceinline__ void tile_sync() {
    if (BAR == 0)
        __syncthreads();
    else
        asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(THREADS) : "memory");
}

// Merge the column splits of one row tile; run by the block that finishes a
// tile last. Every one of the THREADS participating threads (tid < THREADS)
// must call it.
// skip_if_zero (block-sparse verification): when skip_if_zero[tile] == 0 the
// tile is left to a later launch (its ticket is reset, nothing is written).
template <int THREADS, int TILE, int BAR>
__device__ void finish_tile(const HalfStep &A, int tile, int tid, double *s_red, int *s_flag,
                            const int64_t *skip_if_zero = nullptr) {
    __threadfence();
    tile_sync<THREADS, BAR>();
    if (tid == 0) {
        unsigned prev = atomicAdd(&A.tile_cnt[tile], 1u);
        *s_flag = (prev == (unsigned)(A.splits - 1));
    }
    tile_sync<THREADS, BAR>();
    if (!*s_flag) return;
    __threadfence();
    if (skip_if_zero && __ldcg(skip_if_zero + tile) == 0) {
        tile_sync<THREADS, BAR>();  // every thread has read the count
        if (tid == 0) A.tile_cnt[tile] = 0;
        return;
    }

    const double eps = A.prm->eps, kappa = A.prm->kappa, c = A.prm->c, tol = A.prm->tol;
    const int64_t stride = (int64_t)A.tiles * TILE;
    constexpr int RPT = (TILE + THREADS - 1) / THREADS;  // rows of this thread
    constexpr int BU = RPT >= 8 ? 2 : 16 / RPT;  // splits per batch: 16 loads in flight
    // merge the splits' (max, sum) pairs: every load of a batch, for all of this
    // thread's rows, is independent, so one L2 round trip serves 16 partials
    float M[RPT];
    double S[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        M[k] = kNegBig;
        S[k] = 0.0;
    }
    for (int s0 = 0; s0 < A.splits; s0 += BU) {
        float2 pp[RPT][BU];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int64_t row = (int64_t)tile * TILE + k * THREADS + tid;
            const bool live = k * THREADS + tid < TILE && row < A.rows;
#pragma unroll
            for (int u = 0; u < BU; ++u)
                pp[k][u] = (s0 + u < A.splits && live)
                               ? __ldcg(&A.part[(s0 + u) * stride + row])
                               : make_float2(kNegBig, 0.0f);
        }
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            float bm = pp[k][0].x;
#pragma unroll
            for (int u = 1; u < BU; ++u) bm = fmaxf(bm, pp[k][u].x);
            if (bm > M[k]) {
                S[k] *= (double)ex2_approx(M[k] - bm);
                M[k] = bm;
            }
#pragma unroll
            for (int u = 0; u < BU; ++u)
                if (pp[k][u].y > 0.0f) S[k] += (double)pp[k][u].y * (double)ex2_approx(pp[k][u].x - M[k]);
        }
    }
    double rsum = 0.0;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int64_t row = (int64_t)tile * TILE + k * THREADS + tid;
        if (k * THREADS + tid >= TILE || row >= A.rows) continue;
        rsum += finish_row(A, row, M[k], S[k], eps, kappa, c, &bad);
    }
    if (bad) atomicExch(&A.st->nonfinite, 1);
    if (tid == 0) A.tile_cnt[tile] = 0;

    // deterministic block sum of the residual terms
    for (int off = 16; off > 0; off >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, off);
    if ((tid & 31) == 0) s_red[tid >> 5] = rsum;
    tile_sync<THREADS, BAR>();
    if (tid == 0) {
        double t = 0.0;
        for (int w = 0; w < THREADS / 32; ++w) t += s_red[w];
        A.tile_resid[tile] = t;
        __threadfence();
        unsigned prev = atomicAdd(&A.st->tiles_done[A.side], 1u);
        *s_flag = (prev == (unsigned)(A.tiles - 1));
    }
    tile_sync<THREADS, BAR>();
    if (!*s_flag) return;
    __threadfence();
    if (tid < 32) {
        double v = 0.0;
        for (int t = tid; t < A.tiles; t += 32) v += __ldcg(&A.tile_resid[t]);
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (tid == 0) {
            State *st = A.st;
            st->resid[A.side] = v;
            st->tiles_done[A.side] = 0;
            if (A.side == 0) {
                record_residual(A.prm, st->iter_done, v);
                if (tol > 0.0 && st->iter_done >= 1 && v <= tol) {
                    st->stop = 1;
                    st->conv_iter = st->iter_done;
                }
            } else {
                st->iter_done += 1;
            }
            __threadfence();
        }
    }
}

}  // namespace ot
