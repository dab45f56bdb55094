// sparse.cu -- block-sparse fine updates for d <= 3, following "FlashSinkhorn
// 2: Block-Sparse Entropic Optimal Transport", sections 3, 3.2, A.3, B.1, B.3.
//
// Points are put in Morton order once per solve (a 30-bit code from the joint
// bounding box, sorted with the point index as the tie-break), so that blocks
// of B consecutive points are spatially compact. Every fine iteration then
//  1. takes each block's potential maximum (block_max_kernel);
//  2. screens every block pair (I, J) with the bound
//        M_IJ <= |I| |J| exp((F_I + G_J - c D_IJ) / eps),
//     D_IJ the squared distance between the two blocks' bounding boxes, against
//     rho_IJ = delta * min(smallest nonzero a in I, smallest nonzero b in J)
//     (screen_kernel, float64, one byte per pair);
//  3. verifies the candidates by their exact mass over the B x B point pairs
//     and, in the same pass, runs the f-update over the admitted ones
//     (hs_verify_kernel: the half-step's own float32 exponentials, float64 row
//     terms; a row block left without an admitted tile is updated over every
//     column by a fallback hs_sparse_kernel launch);
//  4. lists the admitted tiles of every column block from the transposed mask
//     (transpose_bytes_kernel, mask_list_kernel);
//  5. runs the g-update over the admitted tiles only (hs_sparse_kernel: the
//     d <= 3 half-step with a gathered column stream); a block with no
//     admitted tile reduces over every column.
// The mask omits at most delta a_i per tile from row i (delta b_j from
// column j), so with delta = tol / (4 max(NB, MB)) at most tol/4 of the mass.
#include <float.h>

#include <algorithm>

#include "finish.cuh"
#include "lowd.cuh"
#include "runtime.h"

namespace ot {

// ------------------------------------------------------------ Morton order
__device__ __forceinline__ unsigned float_order(float v) {
    const unsigned b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// lohi[k] = min, lohi[3 + k] = max of coordinate k (order-preserving bits)
__global__ void box_kernel(const float *p, int64_t cnt, int d, unsigned *lohi) {
    unsigned lo[3] = {0xffffffffu, 0xffffffffu, 0xffffffffu}, hi[3] = {0u, 0u, 0u};
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < cnt;
         i += (int64_t)gridDim.x * blockDim.x) {
        for (int k = 0; k < d; ++k) {
            const unsigned o = float_order(p[i * d + k]);
            lo[k] = min(lo[k], o);
            hi[k] = max(hi[k], o);
        }
    }
    for (int k = 0; k < d; ++k) {
        const unsigned l = __reduce_min_sync(0xffffffffu, lo[k]);
        const unsigned h = __reduce_max_sync(0xffffffffu, hi[k]);
        if ((threadIdx.x & 31) == 0) {
            atomicMin(lohi + k, l);
            atomicMax(lohi + 3 + k, h);
        }
    }
}

// keys[i] = code(p_i) << 32 | i for i < cnt, all ones for the padding up to n2.
// code: bit t of q_k is bit t*d + (d-1-k); q_k = floor((v - lo_k) * s_k)
// clamped to [0, 2^bits - 1], s_k = 2^bits / (hi_k - lo_k) (0: q_k = 0).
__global__ void morton_kernel(const float *p, int64_t cnt, int64_t n2, MortonArgs M,
                              unsigned long long *keys) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n2) return;
    if (i >= cnt) {
        keys[i] = ~0ull;
        return;
    }
    const double top = (double)((1ll << M.bits) - 1);
    unsigned long long code = 0;
    for (int k = 0; k < M.d; ++k) {
        long long q = 0;
        if (M.s[k] > 0.0) {
            const double t = floor(__dmul_rn(__dsub_rn((double)p[i * M.d + k], M.lo[k]), M.s[k]));
            q = t < 0.0 ? 0 : t > top ? (long long)top : (long long)t;
        }
        for (int b = 0; b < M.bits; ++b)
            if ((q >> b) & 1) code |= 1ull << (b * M.d + (M.d - 1 - k));
    }
    keys[i] = (code << 32) | (unsigned long long)i;
}

// Bitonic sort of n2 (a power of two) 64-bit keys: segments of up to 2048
// keys in shared memory, the strides >= 2048 in global passes.
constexpr int kSortSeg = 2048;

__global__ void __launch_bounds__(1024) bitonic_seg_kernel(unsigned long long *keys, int seg,
                                                           long long kmerge) {
    __shared__ unsigned long long s[kSortSeg];
    const long long base = (long long)blockIdx.x * seg;
    for (int i = threadIdx.x; i < seg; i += blockDim.x) s[i] = keys[base + i];
    __syncthreads();
    auto step = [&](long long k, int j) {
        for (int t = threadIdx.x; t < seg / 2; t += blockDim.x) {
            const int i = 2 * t - (t & (j - 1));
            const bool asc = ((base + i) & k) == 0;
            const unsigned long long a = s[i], b = s[i + j];
            if ((a > b) == asc) {
                s[i] = b;
                s[i + j] = a;
            }
        }
        __syncthreads();
    };
    if (kmerge == 0) {
        for (long long k = 2; k <= seg; k <<= 1)
            for (int j = (int)(k >> 1); j > 0; j >>= 1) step(k, j);
    } else {
        for (int j = seg >> 1; j > 0; j >>= 1) step(kmerge, j);
    }
    for (int i = threadIdx.x; i < seg; i += blockDim.x) keys[base + i] = s[i];
}

__global__ void bitonic_global_kernel(unsigned long long *keys, long long n2, long long k,
                                      long long j) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n2 / 2) return;
    const long long i = 2 * t - (t & (j - 1));
    const bool asc = (i & k) == 0;
    const unsigned long long a = keys[i], b = keys[i + j];
    if ((a > b) == asc) {
        keys[i] = b;
        keys[i + j] = a;
    }
}

// perm[r] = the index in the r-th key; the points, weights and (optional)
// potentials in that order
__global__ void gather_kernel(const unsigned long long *keys, int64_t cnt, int d, const float *p,
                              const float *w, const float *pot, int64_t *perm, float *ps,
                              float *ws, float *pots) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= cnt) return;
    const int64_t idx = (int64_t)(keys[r] & 0xffffffffull);
    perm[r] = idx;
    for (int k = 0; k < d; ++k) ps[r * d + k] = p[idx * d + k];
    ws[r] = w[idx];
    if (pot) pots[r] = pot[idx];
}

__global__ void scatter_kernel(const float *in, const int64_t *perm, int64_t cnt, float *out) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r < cnt) out[perm[r]] = in[r];
}

// --------------------------------------------------------- block summaries
// One warp per block: bounding box, smallest nonzero weight, point count.
__global__ void block_static_kernel(const float *ps, const float *ws, int64_t cnt, int d, int B,
                                    int64_t nblk, BlockSum *bs) {
    const int64_t blk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (blk >= nblk) return;
    const int64_t i0 = blk * B, i1 = min(i0 + B, cnt);
    float lo[3] = {FLT_MAX, FLT_MAX, FLT_MAX}, hi[3] = {-FLT_MAX, -FLT_MAX, -FLT_MAX};
    float wmin = INFINITY;
    for (int64_t i = i0 + lane; i < i1; i += 32) {
        for (int k = 0; k < d; ++k) {
            lo[k] = fminf(lo[k], ps[i * d + k]);
            hi[k] = fmaxf(hi[k], ps[i * d + k]);
        }
        const float w = ws[i];
        if (w > 0.f) wmin = fminf(wmin, w);
    }
    for (int off = 16; off > 0; off >>= 1) {
        for (int k = 0; k < 3; ++k) {
            lo[k] = fminf(lo[k], __shfl_xor_sync(0xffffffffu, lo[k], off));
            hi[k] = fmaxf(hi[k], __shfl_xor_sync(0xffffffffu, hi[k], off));
        }
        wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, off));
    }
    if (lane == 0) {
        BlockSum s;
        for (int k = 0; k < 3; ++k) {
            s.lo[k] = k < d ? (double)lo[k] : 0.0;
            s.hi[k] = k < d ? (double)hi[k] : 0.0;
        }
        s.pmax = -INFINITY;
        s.lnw = isinf(wmin) ? INFINITY : log((double)wmin);
        s.l2w = isinf(wmin) ? INFINITY : log2((double)wmin);
        s.lncnt = log((double)(i1 - i0));
        bs[blk] = s;
    }
}

// One warp per block: the largest potential (-inf for a massless block) and
// log2 sum_j 2^(kappa pot_j) (float64), the column factor of the verification's
// row-level bound.
__global__ void block_max_kernel(const float *pot, int64_t cnt, int B, int64_t nblk, double kappa,
                                 BlockSum *bs) {
    const int64_t blk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (blk >= nblk) return;
    const int64_t i0 = blk * B, i1 = min(i0 + B, cnt);
    float mx = -INFINITY;
    for (int64_t i = i0 + lane; i < i1; i += 32) mx = fmaxf(mx, pot[i]);
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    double sum = 0.0;
    if (mx != -INFINITY)
        for (int64_t i = i0 + lane; i < i1; i += 32)
            if (pot[i] != -INFINITY) sum += exp2(kappa * ((double)pot[i] - (double)mx));
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
        bs[blk].pmax = (double)mx;
        bs[blk].l2gsum = mx == -INFINITY ? -INFINITY : kappa * (double)mx + log2(sum);
    }
}

// ------------------------------------------------------------------ screen
// Grid (ceil(MB / 256), ceil(NB / kScreenRows)): thread t holds column block
// q = 256 blockIdx.x + t, the block's kScreenRows row blocks come from shared
// memory. The test, in float64 with explicit roundings:
//     (F_p + G_q - c D_pq) / eps > ln delta + min(ln amin_p, ln bmin_q) - ln|I_p| - ln|J_q|.
constexpr int kScreenThreads = 256, kScreenRows = 32;

__global__ void __launch_bounds__(kScreenThreads) screen_kernel(ScreenArgs S) {
    if (ld_volatile(&S.st->stop)) return;  // a stopped solve keeps its last mask
    __shared__ BlockSum rs[kScreenRows];
    __shared__ unsigned long long s_tot[kScreenThreads / 32];
    const int tid = threadIdx.x;
    const int64_t q = (int64_t)blockIdx.x * kScreenThreads + tid;
    const int64_t p0 = (int64_t)blockIdx.y * kScreenRows;
    const int nr = (int)min((int64_t)kScreenRows, S.nb - p0);
    if (tid < nr) rs[tid] = S.rs[p0 + tid];
    const bool valid = q < S.mb;
    BlockSum cq{};
    if (valid) cq = S.cs[q];
    __syncthreads();
    long long mine = 0;
    for (int r = 0; r < nr; ++r) {
        const BlockSum &rp = rs[r];
        bool cand = false;
        if (valid && rp.pmax != -INFINITY && cq.pmax != -INFINITY) {
            double D = 0.0;
            for (int k = 0; k < S.d; ++k) {
                double gap = 0.0;
                const double g1 = __dsub_rn(rp.lo[k], cq.hi[k]);
                const double g2 = __dsub_rn(cq.lo[k], rp.hi[k]);
                if (g1 > gap) gap = g1;
                if (g2 > gap) gap = g2;
                D = __dadd_rn(D, __dmul_rn(gap, gap));
            }
            const double lhs =
                __ddiv_rn(__dsub_rn(__dadd_rn(rp.pmax, cq.pmax), __dmul_rn(S.c, D)), S.eps);
            const double rhs = S.ln_delta + fmin(rp.lnw, cq.lnw) - rp.lncnt - cq.lncnt;
            cand = lhs > rhs;
        }
        if (valid) S.mask[(p0 + r) * S.mb + q] = cand ? 1 : 0;
        const int c = __syncthreads_count(cand);
        if (tid == 0 && c > 0) atomicAdd(reinterpret_cast<unsigned long long *>(S.cnt + p0 + r),
                                         (unsigned long long)c);
        mine += cand;
    }
    if (valid && mine > 0)
        atomicAdd(reinterpret_cast<unsigned long long *>(S.cnt_t + q), (unsigned long long)mine);
    unsigned long long w = mine;
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if ((tid & 31) == 0) s_tot[tid >> 5] = w;
    __syncthreads();
    if (tid == 0) {
        unsigned long long t = 0;
        for (int k = 0; k < kScreenThreads / 32; ++k) t += s_tot[k];
        if (t) atomicAdd(S.total, t);
    }
}

// Start of a block-sparse iteration: zero the per-block counts and the tile
// counters (nothing once the solve has stopped, so the last mask's counts stay).
__global__ void sparse_prep_kernel(int64_t *cnt, int64_t nb, int64_t *cnt_t, int64_t mb,
                                   unsigned long long *ctr, int nctr, const State *st) {
    if (ld_volatile(&st->stop)) return;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb + mb + nctr;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nb) cnt[i] = 0;
        else if (i < nb + mb) cnt_t[i - nb] = 0;
        else ctr[i - nb - mb] = 0ull;
    }
}

// After the screen: dense or sparse updates for this iteration (kModeSparse,
// kModeDense; kModeStopped once the stop test has passed), counted per kind.
__global__ void decide_kernel(const unsigned long long *cand, double limit, const State *st,
                              int *mode, unsigned long long *n_mode, int count) {
    if (ld_volatile(&st->stop)) {
        *mode = kModeStopped;
        return;
    }
    const int md = (double)*cand > limit ? kModeDense : kModeSparse;
    *mode = md;
    if (count) {
        n_mode[md] += 1ull;
        mode[1] = md;  // the kind of the last counted iteration
    }
}

// ------------------------------------------------------------ verification
// Work items (row block p, segment of its candidate list; V.segs segments per
// row block, claimed dynamically, so a row block with many candidates does not
// leave a tail). The candidates come as compressed rows (cptr, clist) in
// column order, taken kVfWindow at a time. Each candidate tile q is tested
// against log2 rho = log2 delta + min(log2 amin_p, log2 bmin_q):
//  1. a row-level bound, one warp per tile: with dist_i the distance from
//     x_i to q's bounding box (so C_ij >= c dist_i^2 for every j of q),
//         M <= sum_i 2^(kappa (f_i - c dist_i^2)) * sum_{j in q} 2^(kappa g_j),
//     the column factor computed once per block and iteration (l2gsum);
//     a tile whose bound stays below rho by kVfMargin (base-2 units, far
//     above the float32 rounding of the bound) is rejected here: its exact
//     mass is below rho as well, so the admitted set is the same, at B
//     exponentials per tile instead of B^2 (measured at n = m = 1e6: 1.76M
//     of 3.67M candidates left for the exact test, 1.83M with |J| 2^(kappa
//     max g) as the column factor; a bound through the
//     column side as well, or over 32-point sub-blocks of the column tile,
//     left 7 % / 11 % fewer but cost more time than it saved);
//  2. the exact mass of the others (taken in list order), 256 / B tiles per
//     256-column step: per row i, the running (max m_i, sum s_i) of 2^(t_ij)
//     (t = G_j + x'_i.Y_j, as in the half-step); with the row term b_i = kappa
//     f_i - c kappa |x'_i|^2 (float64), log2 M = log2 sum_i s_i 2^(b_i + m_i),
//     and the tile stays admitted when log2 M > log2 rho. An admitted tile's
//     (m_i, s_i) joins the row's running sum: the segment's share of the
//     f-update, written as a split partial and merged by finish_tile.
// A rejected tile's byte is cleared and the counts are corrected. This kernel is
// the f half-step of a block-sparse iteration (HalfStep A, side 0).
constexpr int kVfWindow = 1024;
constexpr float kVfMargin = 0.05f;

template <int D, int R>
__global__ void __launch_bounds__(kHsThreads, R == 2 ? 5 : 8) hs_verify_kernel(HalfStep A, VerifyArgs V) {
    constexpr int kB = kHsThreads * R;
    __shared__ __align__(16) float4 sbuf[2][kHsChunk];
    __shared__ int s_list[kVfWindow], s_exact[kVfWindow];
    __shared__ float s_xr[kB][3], s_fr[kB];
    __shared__ int s_nexact;
    __shared__ float s_max[kHsChunk / kB][kHsThreads / 32], s_sum[kHsChunk / kB][kHsThreads / 32];
    __shared__ int s_kept;
    __shared__ long long s_next[2];
    __shared__ uint8_t s_keep[kVfWindow];
    __shared__ int s_wcnt[kHsThreads / 32];
    __shared__ double s_red[kHsThreads / 32];
    __shared__ int s_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float4 *rt4 = reinterpret_cast<const float4 *>(V.rowtab);
    const double kappa = V.prm->kappa, c = V.prm->c;
    const float kf = (float)kappa, cf = (float)c;
    if (blockIdx.x == 0 && threadIdx.x == 0) A.st->work[A.side ^ 1] = 0u;  // as in hs_lowd_kernel
    if (ld_volatile(&A.st->stop)) return;
    if (A.gate && ld_volatile(A.gate) != A.gate_val) return;

    const long long n_items = V.nb * (long long)V.segs;
    long long item = blockIdx.x;
    for (int it = 0; item < n_items; ++it) {
        if (tid == 0)
            s_next[it & 1] = (long long)gridDim.x + (long long)atomicAdd(&A.st->work[A.side], 1u);
        const long long p = item / V.segs;
        const int seg = (int)(item % V.segs);
        const int64_t c0 = V.cptr[p], cp = V.cptr[p + 1] - c0;
        const int64_t k0 = c0 + cp * seg / V.segs, k1 = c0 + cp * (seg + 1) / V.segs;
        // the block's points (caller's coordinates) and potentials for the row-level bound
        for (int r = tid; r < kB; r += kHsThreads) {
            const int64_t row = p * kB + r;
            const bool in = row < V.rows;
#pragma unroll
            for (int k = 0; k < 3; ++k) s_xr[r][k] = (in && k < D) ? V.pts[row * D + k] : 0.f;
            s_fr[r] = in ? V.pot[row] : -INFINITY;
        }
        float2 xd[R][3];
        double base[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t row = p * kB + k * kHsThreads + tid;
            const float4 x = row < V.rows ? rt4[row] : make_float4(0.f, 0.f, 0.f, 0.f);
            xd[k][0] = make_float2(x.x, x.x);
            xd[k][1] = make_float2(x.y, x.y);
            xd[k][2] = make_float2(x.z, x.z);
            const double nrm = (double)x.x * x.x + (double)x.y * x.y + (double)x.z * x.z + (double)x.w * x.w;
            base[k] = row < V.rows ? kappa * (double)V.pot[row] - c * kappa * nrm : -INFINITY;
        }
        // this segment's share of the f-update: (running max, sum) over its admitted tiles
        float mr[R], tr[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            mr[k] = kNegBig;
            tr[k] = 0.f;
        }
        if (tid == 0) s_kept = 0;
        for (int64_t w0 = k0; w0 < k1; w0 += kVfWindow) {
            // this window of the segment's candidate columns
            const int total = (int)min((int64_t)kVfWindow, k1 - w0);
            for (int t = tid; t < total; t += kHsThreads) s_list[t] = V.clist[w0 + t];
            __syncthreads();

            // 1. row-level bound, one warp per candidate tile
            for (int t = warp; t < total; t += kHsThreads / 32) {
                const int64_t q = s_list[t];
                const BlockSum &cq = V.cs[q];
                float lo[3], hi[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    lo[k] = (float)cq.lo[k];
                    hi[k] = (float)cq.hi[k];
                }
                float u[kB / 32], mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < kB / 32; ++k) {
                    const int r = lane + 32 * k;
                    float dist = 0.f;
#pragma unroll
                    for (int e = 0; e < D; ++e) {
                        const float gap = fmaxf(0.f, fmaxf(lo[e] - s_xr[r][e], s_xr[r][e] - hi[e]));
                        dist = fmaf(gap, gap, dist);
                    }
                    u[k] = s_fr[r] == -INFINITY ? -INFINITY : kf * (s_fr[r] - cf * dist);
                    mx = fmaxf(mx, u[k]);
                }
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                float sum = 0.f;
                if (mx != -INFINITY) {
#pragma unroll
                    for (int k = 0; k < kB / 32; ++k)
                        if (u[k] != -INFINITY) sum += ex2_approx(u[k] - mx);
                }
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane == 0) {
                    const double lb = (mx == -INFINITY || cq.l2gsum == -INFINITY)
                                          ? -INFINITY : (double)mx + log2((double)sum) + cq.l2gsum;
                    const double lrho = V.l2_delta + fmin(V.rs[p].l2w, cq.l2w);
                    const bool keep = lb + kVfMargin > lrho;
                    s_keep[t] = keep;
                    if (!keep) {
                        V.mask[p * V.mb + q] = 0;
                        atomicAdd(reinterpret_cast<unsigned long long *>(V.cnt_t + q), ~0ull);
                    }
                }
            }
            __syncthreads();
            {   // the survivors in list order (the f-update sums its tiles in a fixed order)
                constexpr int kPer = kVfWindow / kHsThreads;
                int mine = 0;
#pragma unroll
                for (int u = 0; u < kPer; ++u) mine += (tid * kPer + u < total) && s_keep[tid * kPer + u];
                int incl = mine;
                for (int off = 1; off < 32; off <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                if (lane == 31) s_wcnt[warp] = incl;
                __syncthreads();
                int pos = incl - mine;
                for (int k = 0; k < warp; ++k) pos += s_wcnt[k];
#pragma unroll
                for (int u = 0; u < kPer; ++u)
                    if ((tid * kPer + u < total) && s_keep[tid * kPer + u]) s_exact[pos++] = s_list[tid * kPer + u];
                if (tid == kHsThreads - 1) s_nexact = pos;
                __syncthreads();
            }
            const int n_exact = s_nexact;
            if (tid == 0 && n_exact) atomicAdd(V.exact, (unsigned long long)n_exact);

            // 2. exact mass of the remaining tiles, 256 / B tiles per step (one
            // 256-column chunk), the next step's columns loaded while this one runs
            constexpr int kTpc = kHsChunk / kB;
            const int nsteps = (n_exact + kTpc - 1) / kTpc;
            auto fetch = [&](int step, int u) -> float4 {
                const int t = step * kTpc + u / kB;
                if (t >= n_exact) return dead4(u);
                const int64_t col = (int64_t)s_exact[t] * kB + (u % kB);
                return col < V.cols_pad ? V.coltab[col] : dead4(u);
            };
            float4 p0 = make_float4(0.f, 0.f, 0.f, 0.f), p1 = p0;
            if (nsteps > 0) {
                p0 = fetch(0, tid);
                p1 = fetch(0, tid + kHsThreads);
            }
            for (int step = 0; step < nsteps; ++step) {
                float4 *buf = sbuf[step & 1];
                buf[tid] = p0;
                buf[tid + kHsThreads] = p1;
                __syncthreads();
                if (step + 1 < nsteps) {
                    p0 = fetch(step + 1, tid);
                    p1 = fetch(step + 1, tid + kHsThreads);
                }
                float wv[kTpc][R];
                float tv[kTpc][R], mv[kTpc][R];
#pragma unroll
                for (int tt = 0; tt < kTpc; ++tt) {
                    float m[R], tot[R];
                    float2 nm[R], acc[R], acc2[R];
#pragma unroll
                    for (int k = 0; k < R; ++k) {
                        m[k] = kNegBig;
                        nm[k] = make_float2(-kNegBig, -kNegBig);
                        acc[k] = acc2[k] = make_float2(0.f, 0.f);
                        tot[k] = 0.f;
                    }
                    if (step * kTpc + tt < n_exact) {
#pragma unroll 1
                        for (int j = 0; j < kB; j += 8) {
                            float4 v[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) v[u] = buf[tt * kB + j + u];
                            lowd_step8<D, R, true>(v, xd, m, nm, acc, acc2, tot);
                        }
                    }
                    float wmax = -INFINITY;
#pragma unroll
                    for (int k = 0; k < R; ++k) {
                        tot[k] += (acc[k].x + acc[k].y) + (acc2[k].x + acc2[k].y);
                        tv[tt][k] = tot[k];
                        mv[tt][k] = m[k];
                        wv[tt][k] = (tot[k] > 0.f && base[k] != -INFINITY)
                                        ? (float)(base[k] + (double)m[k]) : -INFINITY;
                        wmax = fmaxf(wmax, wv[tt][k]);
                    }
                    for (int off = 16; off > 0; off >>= 1)
                        wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, off));
                    if (lane == 0) s_max[tt][warp] = wmax;
                }
                __syncthreads();
                float W[kTpc];
#pragma unroll
                for (int tt = 0; tt < kTpc; ++tt) {
                    W[tt] = s_max[tt][0];
                    for (int k = 1; k < kHsThreads / 32; ++k) W[tt] = fmaxf(W[tt], s_max[tt][k]);
                    float sum = 0.f;
                    if (W[tt] != -INFINITY) {
#pragma unroll
                        for (int k = 0; k < R; ++k)
                            if (wv[tt][k] != -INFINITY) sum += tv[tt][k] * ex2_approx(wv[tt][k] - W[tt]);
                    }
                    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                    if (lane == 0) s_sum[tt][warp] = sum;
                }
                __syncthreads();
#pragma unroll
                for (int tt = 0; tt < kTpc; ++tt) {
                    if (step * kTpc + tt >= n_exact) continue;
                    const int64_t q = s_exact[step * kTpc + tt];
                    // one lane per warp takes the decision (float64 log2), the warp shares it
                    int adm = 0;
                    if (lane == 0) {
                        float S = 0.f;
                        for (int k = 0; k < kHsThreads / 32; ++k) S += s_sum[tt][k];
                        const double lm = (W[tt] == -INFINITY || !(S > 0.f))
                                              ? -INFINITY : (double)W[tt] + log2((double)S);
                        adm = lm > V.l2_delta + fmin(V.rs[p].l2w, V.cs[q].l2w);
                    }
                    if (__shfl_sync(0xffffffffu, adm, 0)) {  // admitted: the tile joins this segment's f-update
#pragma unroll
                        for (int k = 0; k < R; ++k) {
                            if (!(tv[tt][k] > 0.f)) continue;
                            if (mv[tt][k] > mr[k]) {
                                tr[k] = tr[k] * ex2_approx(mr[k] - mv[tt][k]) + tv[tt][k];
                                mr[k] = mv[tt][k];
                            } else {
                                tr[k] += tv[tt][k] * ex2_approx(mv[tt][k] - mr[k]);
                            }
                        }
                        if (tid == 0) ++s_kept;
                    } else if (tid == 0) {
                        V.mask[p * V.mb + q] = 0;
                        atomicAdd(reinterpret_cast<unsigned long long *>(V.cnt_t + q), ~0ull);
                    }
                }
            }
            __syncthreads();  // s_list and s_exact are rewritten by the next window
        }
        __syncthreads();
        if (tid == 0) {
            const int kept = s_kept;
            if (kept) {
                atomicAdd(reinterpret_cast<unsigned long long *>(V.cnt + p), (unsigned long long)kept);
                atomicAdd(V.total, (unsigned long long)kept);
            }
        }
        const int64_t stride = (int64_t)A.tiles * kB;
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t row = p * kB + k * kHsThreads + tid;
            if (row < A.rows) A.part[seg * stride + row] = make_float2(mr[k], tr[k]);
        }
        // the last segment merges; a row block left with no admitted tile is
        // skipped here and updated over every column by the fallback launch
        finish_tile<kHsThreads, kB, 0>(A, (int)p, tid, s_red, &s_flag, V.cnt);
        __syncthreads();
        item = s_next[it & 1];
    }
}

// --------------------------------------------------- mask -> column lists
// One block per row of a byte matrix [rows][cols]: the columns of the nonzero
// bytes of row r, in increasing order, go to list[ptr[r] ..].
constexpr int kListThreads = 256;

__global__ void __launch_bounds__(kListThreads) mask_list_kernel(const uint8_t *mask, int64_t rows,
                                                                 int64_t cols, const int64_t *ptr,
                                                                 int *list) {
    __shared__ int s_w[kListThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        int64_t at = ptr[r];
        for (int64_t c0 = 0; c0 < cols; c0 += kListThreads) {
            const int64_t c = c0 + tid;
            const bool on = c < cols && mask[r * cols + c] != 0;
            const unsigned bal = __ballot_sync(0xffffffffu, on);
            if (lane == 0) s_w[warp] = __popc(bal);
            __syncthreads();
            int off = 0, tot = 0;
            for (int k = 0; k < kListThreads / 32; ++k) {
                if (k < warp) off += s_w[k];
                tot += s_w[k];
            }
            if (on) list[at + off + __popc(bal & ((1u << lane) - 1u))] = (int)c;
            at += tot;
            __syncthreads();
        }
    }
}

// out[c][r] = in[r][c] for a byte matrix, 64 x 64 tiles
__global__ void __launch_bounds__(256) transpose_bytes_kernel(const uint8_t *in, int64_t rows,
                                                              int64_t cols, uint8_t *out) {
    __shared__ uint8_t t[64][65];
    const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int rr = i >> 6, cc = i & 63;
        t[rr][cc] = (r0 + rr < rows && c0 + cc < cols) ? in[(r0 + rr) * cols + c0 + cc] : 0;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int cc = i >> 6, rr = i & 63;
        if (c0 + cc < cols && r0 + rr < rows) out[(c0 + cc) * rows + r0 + rr] = t[rr][cc];
    }
}

// --------------------------------------------------------- sparse half-step
// The d <= 3 half-step over each row block's admitted column tiles; work
// items (row block, split of its tile list) are claimed dynamically and merged
// by finish_tile, exactly as in hs_lowd_kernel.
template <int D, int R>
__global__ void __launch_bounds__(kHsThreads, R == 2 ? 4 : 8) hs_sparse_kernel(HalfStep A) {
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
        if (threadIdx.x == 0)
            s_next[it & 1] = (long long)gridDim.x + (long long)atomicAdd(&A.st->work[A.side], 1u);
        const int tile = (int)(item / A.splits);
        const int split = (int)(item % A.splits);
        if (A.sp_fallback && __ldcg(A.sp_fallback + tile) != 0) {  // not a fallback block
            __syncthreads();
            item = s_next[it & 1];
            continue;
        }
        sparse_item<D, R>(A, tile, split, sm);
        finish_tile<kHsThreads, kHsThreads * R, 0>(A, tile, threadIdx.x, s_red, &s_flag);
        __syncthreads();
        item = s_next[it & 1];
    }
}

// ----------------------------------------------------------------- launchers
template <int R>
static const void *sparse_fn(int d) {
    if (d == 1) return (const void *)hs_sparse_kernel<1, R>;
    if (d == 2) return (const void *)hs_sparse_kernel<2, R>;
    return (const void *)hs_sparse_kernel<3, R>;
}

template <int R>
static const void *verify_fn(int d) {
    if (d == 1) return (const void *)hs_verify_kernel<1, R>;
    if (d == 2) return (const void *)hs_verify_kernel<2, R>;
    return (const void *)hs_verify_kernel<3, R>;
}

static const void *sparse_kernel_fn(int which, int d, int rpt) {
    if (rpt == 1) return which ? verify_fn<1>(d) : sparse_fn<1>(d);
    if (rpt == 2) return which ? verify_fn<2>(d) : sparse_fn<2>(d);
    return nullptr;
}

int sparse_blocks_per_sm(int which, int d, int rpt) {
    const void *fn = sparse_kernel_fn(which, d, rpt);
    int nb = 0;
    if (!fn || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kHsThreads, 0) != cudaSuccess)
        return 0;
    return nb;
}

cudaError_t launch_box(const float *p, int64_t cnt, int d, unsigned *lohi, cudaStream_t s) {
    const int64_t blocks = std::min<int64_t>((cnt + 255) / 256, 1184);
    box_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, s>>>(p, cnt, d, lohi);
    return cudaGetLastError();
}

cudaError_t launch_morton_sort(const float *p, int64_t cnt, int64_t n2, const MortonArgs &M,
                               unsigned long long *keys, cudaStream_t s) {
    morton_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, s>>>(p, cnt, n2, M, keys);
    const int seg = (int)std::min<int64_t>(kSortSeg, n2);
    const int threads = std::max(1, std::min(1024, seg / 2));
    const unsigned nseg = (unsigned)(n2 / seg);
    bitonic_seg_kernel<<<nseg, threads, 0, s>>>(keys, seg, 0);
    for (long long k = 2ll * seg; k <= n2; k <<= 1) {
        for (long long j = k >> 1; j >= seg; j >>= 1)
            bitonic_global_kernel<<<(unsigned)((n2 / 2 + 255) / 256), 256, 0, s>>>(keys, n2, k, j);
        bitonic_seg_kernel<<<nseg, threads, 0, s>>>(keys, seg, k);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather(const unsigned long long *keys, int64_t cnt, int d, const float *p,
                          const float *w, const float *pot, int64_t *perm, float *ps, float *ws,
                          float *pots, cudaStream_t s) {
    gather_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, s>>>(keys, cnt, d, p, w, pot, perm, ps,
                                                                ws, pots);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const float *in, const int64_t *perm, int64_t cnt, float *out,
                           cudaStream_t s) {
    scatter_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, s>>>(in, perm, cnt, out);
    return cudaGetLastError();
}

cudaError_t launch_block_static(const float *ps, const float *ws, int64_t cnt, int d, int B,
                                BlockSum *bs, cudaStream_t s) {
    const int64_t nblk = (cnt + B - 1) / B;
    block_static_kernel<<<(unsigned)((nblk * 32 + 255) / 256), 256, 0, s>>>(ps, ws, cnt, d, B, nblk, bs);
    return cudaGetLastError();
}

cudaError_t launch_block_max(const float *pot, int64_t cnt, int B, double kappa, BlockSum *bs,
                             cudaStream_t s) {
    const int64_t nblk = (cnt + B - 1) / B;
    block_max_kernel<<<(unsigned)((nblk * 32 + 255) / 256), 256, 0, s>>>(pot, cnt, B, nblk, kappa, bs);
    return cudaGetLastError();
}

cudaError_t launch_sparse_prep(int64_t *cnt, int64_t nb, int64_t *cnt_t, int64_t mb,
                               unsigned long long *ctr, int nctr, const State *st, cudaStream_t s) {
    const int64_t total = nb + mb + nctr;
    const unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, 1184);
    sparse_prep_kernel<<<std::max(grid, 1u), 256, 0, s>>>(cnt, nb, cnt_t, mb, ctr, nctr, st);
    return cudaGetLastError();
}

cudaError_t launch_decide(const unsigned long long *cand, double limit, const State *st, int *mode,
                          unsigned long long *n_mode, int count, cudaStream_t s) {
    decide_kernel<<<1, 1, 0, s>>>(cand, limit, st, mode, n_mode, count);
    return cudaGetLastError();
}

cudaError_t launch_screen(const ScreenArgs &S, cudaStream_t s) {
    const dim3 grid((unsigned)((S.mb + kScreenThreads - 1) / kScreenThreads),
                    (unsigned)((S.nb + kScreenRows - 1) / kScreenRows));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    screen_kernel<<<grid, kScreenThreads, 0, s>>>(S);
    return cudaGetLastError();
}

cudaError_t launch_verify(int d, int rpt, const HalfStep &A, const VerifyArgs &V, int grid,
                          cudaStream_t s) {
    const void *fn = sparse_kernel_fn(1, d, rpt);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {(void *)&A, (void *)&V};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kHsThreads), args, 0, s);
}

cudaError_t launch_mask_list(const uint8_t *mask, int64_t rows, int64_t cols, const int64_t *ptr,
                             int *list, cudaStream_t s) {
    const int64_t grid = std::min<int64_t>(rows, 65535);
    mask_list_kernel<<<(unsigned)std::max<int64_t>(grid, 1), kListThreads, 0, s>>>(mask, rows, cols,
                                                                                  ptr, list);
    return cudaGetLastError();
}

cudaError_t launch_transpose_bytes(const uint8_t *in, int64_t rows, int64_t cols, uint8_t *out,
                                   cudaStream_t s) {
    const dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    transpose_bytes_kernel<<<grid, 256, 0, s>>>(in, rows, cols, out);
    return cudaGetLastError();
}

cudaError_t launch_halfstep_sparse(int d, int rpt, const HalfStep &A, int grid, cudaStream_t s) {
    const void *fn = sparse_kernel_fn(0, d, rpt);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {(void *)&A};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kHsThreads), args, 0, s);
}

}  // namespace ot
