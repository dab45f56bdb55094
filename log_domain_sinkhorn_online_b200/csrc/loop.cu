// loop.cu -- device-resident Sinkhorn iterations for small d <= 3 problems.
//
// On small problems (n*m up to a few 10^8 pairs) each half-step takes tens of
// microseconds, so launch latency, the serialized merge of the column splits
// by one block per tile, and host round trips for the stop test cost as much
// as the arithmetic. This kernel runs many iterations of the alternating
// updates ("FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section
// 2.1) in one cooperative launch; per half-step:
//   compute  every block runs its (row tile, column split) items -> partials
//   barrier
//   merge    every thread of the grid merges whole rows (new potential, the
//            other side's column term, the row's residual term); each block
//            writes one residual partial
//   barrier
// After an f-update every block sums the block partials in the same fixed
// order, so all blocks take the same stop decision (tol on ||T1 - a||_1 of the
// state before the update) without another barrier.
//
// All co-resident by construction (cooperative launch). The grid barrier waits
// on an arrival counter with a time limit (globaltimer; 10 s, set by the
// host): past it the kernel records State::wait_timeout and every block leaves
// the loop. Data rewritten
// inside the kernel (column tables, potentials, partials) is read with L1
// bypassed.
#include "finish.cuh"
#include "lowd.cuh"
#include "runtime.h"

namespace ot {

namespace {

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier for a cooperative launch: a counter that only grows (the
// host zeroes it before each launch). Barrier k of the launch is passed when
// the counter reaches (k + 1) * gridDim.x; one release-add per block, acquire
// polling by thread 0. Returns false (uniformly per block) if the wait gave up,
// after setting *err.
__device__ bool grid_barrier(unsigned *count, unsigned &k, int *err, volatile int *s_ok,
                             uint64_t limit_ns) {
    __syncthreads();
    const unsigned target = (++k) * gridDim.x;
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
        int ok = 1;
        if (ld_acquire_u32(count) < target) {
            const uint64_t t0 = globaltimer();
            while (ld_acquire_u32(count) < target) {
                __nanosleep(20);
                if (globaltimer() - t0 > limit_ns) {
                    ok = 0;
                    atomicExch(err, 1);
                    break;
                }
            }
        }
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Every thread of the grid merges whole rows of one half-step; returns this
// block's residual partial (thread 0 only, others 0).
template <int THREADS>
__device__ double merge_phase(const HalfStep &A, double *s_red, bool *any_bad) {
    const double eps = A.prm->eps, kappa = A.prm->kappa, c = A.prm->c;
    const int64_t stride = (int64_t)A.tiles * A.tile_rows;
    double rsum = 0.0;
    bool bad = false;
    for (int64_t row = (int64_t)blockIdx.x * THREADS + threadIdx.x; row < A.rows;
         row += (int64_t)gridDim.x * THREADS) {
        float M = kNegBig;
        double S = 0.0;
        for (int s0 = 0; s0 < A.splits; s0 += 16) {
            float2 pp[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                pp[u] = s0 + u < A.splits ? __ldcg(&A.part[(s0 + u) * stride + row])
                                          : make_float2(kNegBig, 0.0f);
            float bm = pp[0].x;
#pragma unroll
            for (int u = 1; u < 16; ++u) bm = fmaxf(bm, pp[u].x);
            if (bm > M) {
                S *= (double)ex2_approx(M - bm);
                M = bm;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (pp[u].y > 0.0f) S += (double)pp[u].y * (double)ex2_approx(pp[u].x - M);
        }
        rsum += finish_row(A, row, M, S, eps, kappa, c, &bad);
    }
    if (bad) *any_bad = true;
    for (int off = 16; off > 0; off >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, off);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = rsum;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < THREADS / 32; ++w) t += s_red[w];
    __syncthreads();
    return t;
}

// Sum of the per-block residual partials in block order (same in every block).
template <int THREADS>
__device__ double grid_residual(const double *blk, double *s_red) {
    double v = 0.0;
    for (int b = threadIdx.x; b < (int)gridDim.x; b += THREADS) v += __ldcg(blk + b);
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < THREADS / 32; ++w) t += s_red[w];
    __syncthreads();
    return t;
}

}  // namespace

// The loop kernel runs R = 1 or 2 rows per thread in both half-steps (the cost
// model picks: 128-row tiles balance better across 148 SMs on some sizes, e.g.
// 63 x 7 = 441 items at n = 8000, 2-row tiles on others). At most 4 blocks per
// SM: the problems it runs have a few hundred work items, and the registers
// left free let the exponentials run ahead of the refresh vote.
template <int D, int R>
__global__ void __launch_bounds__(kHsThreads, 4) hs_loop_kernel(LoopArgs L) {
    __shared__ __align__(16) float4 sm[2][kHsChunk];
    __shared__ double s_red[kHsThreads / 32];
    __shared__ int s_ok;
    State *st = L.f[0].st;
    if (ld_volatile(&st->stop)) return;
    int par = L.parity0 & 1;
    int iter_done = ld_volatile(&st->iter_done);
    const double tol = L.f[0].prm->tol;
    bool bad = false;
    unsigned nbar = 0;  // grid barriers passed in this launch
    for (int it = 0; it < L.iters; ++it) {
        // ------------------------------------------------------- f-update
        const HalfStep &F = L.f[par];
        const int64_t nf = (int64_t)F.tiles * F.splits;
        for (int64_t item = blockIdx.x; item < nf; item += gridDim.x) {
            __syncthreads();
            lowd_item<D, R, true, true>(F, (int)(item / F.splits), (int)(item % F.splits), sm);
        }
        if (nbar == 0 && (int)blockIdx.x == L.withhold_block) return;  // failure tests only
        if (!grid_barrier(L.bar_count, nbar, &st->wait_timeout, &s_ok, L.wait_ns)) break;
        const double br = merge_phase<kHsThreads>(F, s_red, &bad);
        if (threadIdx.x == 0) L.blk_resid[blockIdx.x] = br;
        if (!grid_barrier(L.bar_count, nbar, &st->wait_timeout, &s_ok, L.wait_ns)) break;
        const double resid = grid_residual<kHsThreads>(L.blk_resid, s_red);
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            st->resid[0] = resid;
            record_residual(F.prm, iter_done, resid);
        }
        if (tol > 0.0 && iter_done >= 1 && resid <= tol) {  // the same decision in every block
            if (blockIdx.x == 0 && threadIdx.x == 0) {
                st->stop = 1;
                st->conv_iter = iter_done;
            }
            break;
        }
        // ------------------------------------------------------- g-update
        const HalfStep &G = L.g[par];
        const int64_t ng = (int64_t)G.tiles * G.splits;
        for (int64_t item = blockIdx.x; item < ng; item += gridDim.x) {
            __syncthreads();
            lowd_item<D, R, true, true>(G, (int)(item / G.splits), (int)(item % G.splits), sm);
        }
        if (!grid_barrier(L.bar_count, nbar, &st->wait_timeout, &s_ok, L.wait_ns)) break;
        merge_phase<kHsThreads>(G, s_red, &bad);
        if (!grid_barrier(L.bar_count, nbar, &st->wait_timeout, &s_ok, L.wait_ns)) break;
        ++iter_done;
        par ^= 1;
        if (blockIdx.x == 0 && threadIdx.x == 0) st->iter_done = iter_done;
    }
    if (bad) atomicExch(&st->nonfinite, 1);
}

template <int R>
static const void *loop_fn_r(int d) {
    if (d == 1) return (const void *)hs_loop_kernel<1, R>;
    if (d == 2) return (const void *)hs_loop_kernel<2, R>;
    return (const void *)hs_loop_kernel<3, R>;
}

static const void *loop_fn(int d, int rpt) {
    if (rpt == 1) return loop_fn_r<1>(d);
    if (rpt == 2) return loop_fn_r<2>(d);
    return nullptr;
}

int loop_blocks_per_sm(int d, int rpt) {
    const void *fn = loop_fn(d, rpt);
    int nb = 0;
    if (!fn || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kHsThreads, 0) != cudaSuccess)
        return 0;
    return nb;
}

cudaError_t launch_loop(int d, int rpt, const LoopArgs &L, int grid, cudaStream_t s) {
    const void *fn = loop_fn(d, rpt);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {(void *)&L};
    return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kHsThreads), args, 0, s);
}

}  // namespace ot
