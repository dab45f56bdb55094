// halfstep.cu -- fused log-domain Sinkhorn half-step for sm_100a.
//
// One launch performs f_i <- eps ln a_i - eps LSE_j((g_j - C_ij)/eps) for every
// row i (or the g-update with the roles of the clouds swapped), following
// "FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section 2.1: the
// update is a streaming log-sum-exp over column tiles whose costs are generated
// on the fly, so the n x m matrix never exists.
//
// Cost tile generator. In base-2 units, with kappa = log2(e)/eps, the shift o
// (midpoint of the two clouds' means) and x' = x - o, y' = y - o:
//   kappa (g_j - C_ij) = G_j + 2 c kappa x'_i . y'_j + R_i,
//   G_j = kappa (g_j - c |y'_j|^2)   (column table, refreshed by the other half-step),
//   R_i = -c kappa |x'_i|^2           (row constant, added once per row in float64).
// For d <= 3 the per-pair work is d packed-f32x2 FMAs (two columns per
// instruction), one subtraction of the running maximum, one MUFU ex2 and one
// add: the kernel is bound by the ex2 rate, not by memory.
//
// Split-column combine. Each work item is (row tile, column split). It writes
// (running max, sum) per row; the last split of a tile to finish (atomic
// ticket, no waiting) merges them in float64 in split order, writes the new
// potential, the other half-step's column-table entry, and this row's term of
// the marginal residual ||T 1 - a||_1 at the state before the update:
//   sum_j T_ij(old) = 2^(kappa f_old_i + L_i),  L_i = log2 sum_j 2^(kappa (g_j - C_ij)).
// The last tile to finish sums the residual partials in tile order (no float
// atomics, so the result is deterministic) and runs the stop test.
#include "finish.cuh"
#include "lowd.cuh"

namespace ot {

// ------------------------------------------------------------ d <= 3 path
// Column table: for the column pair (2p, 2p+1), two float4
//   [Y0_2p, Y0_2p+1, Y1_2p, Y1_2p+1]  [Y2_2p, Y2_2p+1, G_2p, G_2p+1]
// with Y = 2 c kappa y' (zero past d) and G as above; padding columns have
// Y = 0, G = -inf and add nothing. So column c's data starts at float4 c (c
// even) and a chunk of 256 columns is 256 float4 (4 KB of shared memory).
// Rows: thread t of a tile owns rows t + 128 k, k < R (R = 1, 2, 4 or 8; the
// tile is 128 R rows: fewer rows per thread give more tiles, hence fewer column
// splits to merge, on small problems; R = 1 serves the f-update that follows a
// 1-row device-resident loop, or a caller who asks for it).
//
// Work items are handed out dynamically: block b starts with item b, and each
// item's first thread claims the next one (grid + a per-side atomic counter)
// while the item runs. Blocks are not placed on SMs round-robin, so a static
// stride left whole SMs idle at the end of a launch (ncu: SMs active 85 % of
// the elapsed cycles at n = m = 1e5). The counter of one side is reset by
// every launch of the other side before anything else (f- and g-launches
// alternate, so its previous user has finished and its next user has not
// started); reset_state clears both at the start of a stage.
template <int D, int R>
__global__ void __launch_bounds__(kHsThreads, R == 8 ? 3 : R == 4 ? 4 : R == 2 ? 6 : 8) hs_lowd_kernel(HalfStep A) {
    __shared__ __align__(16) float4 sm[2][kHsChunk];
    __shared__ double s_red[kHsThreads / 32];
    __shared__ int s_flag;
    __shared__ long long s_next[2];
    if (blockIdx.x == 0 && threadIdx.x == 0) A.st->work[A.side ^ 1] = 0u;
    if (ld_volatile(&A.st->stop)) return;
    if (A.gate && ld_volatile(A.gate) != A.gate_val) return;
    const int64_t n_items = (int64_t)A.tiles * A.splits;
    int64_t item = blockIdx.x;
    for (int it = 0; item < n_items; ++it) {
        // two slots: a slow thread still reading the previous claim is never overwritten
        if (threadIdx.x == 0)
            s_next[it & 1] = (long long)gridDim.x + (long long)atomicAdd(&A.st->work[A.side], 1u);
        const int tile = (int)(item / A.splits);
        const int split = (int)(item % A.splits);
        lowd_item<D, R, false, true>(A, tile, split, sm);
        finish_tile<kHsThreads, kHsThreads * R, 0>(A, tile, threadIdx.x, s_red, &s_flag);
        __syncthreads();
        item = s_next[it & 1];
    }
}

// --------------------------------------------------------- generic-d path
// For 3 < d <= 64 (CUDA-core FMA path). Column table: per column DP + 4
// floats, [Y_0 .. Y_{DP-1}, G, 0, 0, 0] (Y = 2 c kappa y', zero past d). Row
// table: [rows][DP] floats x' (zero past d). Thread t owns rows t and t + 128
// of the tile; the dot products run as packed f32x2 FMAs over coordinate pairs.
// Work items are handed out dynamically, as in hs_lowd_kernel.
template <int DP>
__global__ void __launch_bounds__(kGnThreads, 2) hs_generic_kernel(HalfStep A) {
    constexpr int ST = DP + 4;
    constexpr int CH4 = kGnChunk * ST / 4;  // float4 per chunk
    __shared__ __align__(16) float4 sm[2][CH4];
    __shared__ double s_red[kGnThreads / 32];
    __shared__ int s_flag;
    __shared__ long long s_next[2];
    if (blockIdx.x == 0 && threadIdx.x == 0) A.st->work[A.side ^ 1] = 0u;  // as in hs_lowd_kernel
    if (ld_volatile(&A.st->stop)) return;
    const int tid = threadIdx.x;
    const int64_t n_items = (int64_t)A.tiles * A.splits;

    int64_t item = blockIdx.x;
    for (int it = 0; item < n_items; ++it) {
        if (tid == 0)
            s_next[it & 1] = (long long)gridDim.x + (long long)atomicAdd(&A.st->work[A.side], 1u);
        const int tile = (int)(item / A.splits);
        const int split = (int)(item % A.splits);

        float2 xp[kGnRows][DP / 2];
        float m[kGnRows], tot[kGnRows];
        float2 acc[kGnRows];
#pragma unroll
        for (int k = 0; k < kGnRows; ++k) {
            const int64_t row = (int64_t)tile * kGnTile + k * kGnThreads + tid;
            const float2 *src = reinterpret_cast<const float2 *>(A.rowtab + row * (int64_t)DP);
#pragma unroll
            for (int q = 0; q < DP / 2; ++q) xp[k][q] = row < A.rows ? src[q] : make_float2(0.f, 0.f);
            m[k] = kNegBig;
            acc[k] = make_float2(0.f, 0.f);
            tot[k] = 0.f;
        }

        const int64_t c0 = (int64_t)split * A.cols_per_split;
        const int64_t span = min(c0 + A.cols_per_split, A.cols_pad) - c0;  // multiple of 8
        const int nch = (int)((span + kGnChunk - 1) / kGnChunk);
        const float4 *src = A.coltab + c0 * (ST / 4);

#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
            float4 *buf = sm[ch & 1];
            const int ncols = (int)min((int64_t)kGnChunk, span - (int64_t)ch * kGnChunk);
            for (int u = tid; u < ncols * (ST / 4); u += kGnThreads) buf[u] = src[(int64_t)ch * CH4 + u];
            __syncthreads();
            const float *bf = reinterpret_cast<const float *>(buf);
#pragma unroll 1
            for (int j = 0; j < ncols; j += 4) {
#pragma unroll
                for (int k = 0; k < kGnRows; ++k) {
                    float t[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 *col = reinterpret_cast<const float4 *>(bf + (j + u) * ST);
                        float2 s = make_float2(0.f, 0.f);
#pragma unroll
                        for (int q = 0; q < DP / 4; ++q) {
                            const float4 yv = col[q];
                            s = __ffma2_rn(xp[k][2 * q], make_float2(yv.x, yv.y), s);
                            s = __ffma2_rn(xp[k][2 * q + 1], make_float2(yv.z, yv.w), s);
                        }
                        t[u] = bf[(j + u) * ST + DP] + (s.x + s.y);
                    }
                    const float cm = fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3]));
                    if (__any_sync(0xffffffffu, cm > m[k] + kLazyMax)) {
                        const float mx = fmaxf(cm, m[k]);
                        const float sc = ex2_approx(m[k] - mx);
                        acc[k] = __fmul2_rn(acc[k], make_float2(sc, sc));
                        tot[k] *= sc;
                        m[k] = mx;
                    }
                    const float2 nm = make_float2(-m[k], -m[k]);
                    const float2 u0 = __fadd2_rn(make_float2(t[0], t[1]), nm);
                    const float2 u1 = __fadd2_rn(make_float2(t[2], t[3]), nm);
                    acc[k] = __fadd2_rn(acc[k], make_float2(ex2_approx(u0.x), ex2_approx(u0.y)));
                    acc[k] = __fadd2_rn(acc[k], make_float2(ex2_approx(u1.x), ex2_approx(u1.y)));
                }
            }
#pragma unroll
            for (int k = 0; k < kGnRows; ++k) {
                tot[k] += acc[k].x + acc[k].y;
                acc[k] = make_float2(0.f, 0.f);
            }
            __syncthreads();
        }

        const int64_t stride = (int64_t)A.tiles * kGnTile;
#pragma unroll
        for (int k = 0; k < kGnRows; ++k) {
            const int64_t row = (int64_t)tile * kGnTile + k * kGnThreads + tid;
            if (row < A.rows) A.part[split * stride + row] = make_float2(m[k], tot[k]);
        }
        finish_tile<kGnThreads, kGnTile, 0>(A, tile, threadIdx.x, s_red, &s_flag);
        __syncthreads();
        item = s_next[it & 1];
    }
}

// ----------------------------------------------------------------- launchers
template <int R>
static const void *lowd_fn(int dim) {
    if (dim == 1) return (const void *)hs_lowd_kernel<1, R>;
    if (dim == 2) return (const void *)hs_lowd_kernel<2, R>;
    return (const void *)hs_lowd_kernel<3, R>;
}

// kind 0: low-d (dim = d in 1..3, rpt = rows per thread 1/2/4/8);
// kind 1: generic (dim = DP in {8,16,32,64}, rpt ignored).
// The kernel for a launch shape; nullptr for a shape that has no instantiation
// (the tile size, hence the partials' layout, depends on rpt).
static const void *halfstep_fn(int kind, int dim, int rpt) {
    if (kind == 0) {
        if (rpt == 8) return lowd_fn<8>(dim);
        if (rpt == 4) return lowd_fn<4>(dim);
        if (rpt == 2) return lowd_fn<2>(dim);
        if (rpt == 1) return lowd_fn<1>(dim);
        return nullptr;
    }
    if (dim == 8) return (const void *)hs_generic_kernel<8>;
    if (dim == 16) return (const void *)hs_generic_kernel<16>;
    if (dim == 32) return (const void *)hs_generic_kernel<32>;
    return (const void *)hs_generic_kernel<64>;
}

int halfstep_blocks_per_sm(int kind, int dim, int rpt) {
    int nb = 0;
    const int threads = kind == 0 ? kHsThreads : kGnThreads;
    const void *fn = halfstep_fn(kind, dim, rpt);
    if (!fn) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, 0) !=
        cudaSuccess)
        return 0;
    return nb;
}

cudaError_t launch_halfstep(int kind, int dim, int rpt, const HalfStep &A, int grid,
                            cudaStream_t s) {
    const int threads = kind == 0 ? kHsThreads : kGnThreads;
    const void *fn = halfstep_fn(kind, dim, rpt);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {(void *)&A};
    return cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, 0, s);
}

}  // namespace ot
