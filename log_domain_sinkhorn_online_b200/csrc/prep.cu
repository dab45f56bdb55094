// prep.cu -- scale resolution and per-stage tables.
//
// The cost scale is resolved once on the whole problem and captured by the plan
// (moscot PR #846, "materialize transport-matrix rows instead of pushing
// indicator columns", section Fix: a subset must never re-derive it).
//  - "mean": the mean over all n*m pairs of ||x_i - y_j||^2 has the closed form
//      mean|x|^2 + mean|y|^2 - 2 mean(x) . mean(y),
//    evaluated from float64 coordinate sums (O((n+m)d)).
//  - "max_cost": one pass over all pairs (fp32 differences, order-free max).
// All sums use a fixed reduction order, so repeated runs agree bit for bit.
#include "common.cuh"

#include <algorithm>

namespace ot {

constexpr int kStatThreads = 256;

// Per-coordinate column sums of a [cnt, d] float array: block (bx, k) sums
// coordinate k over its point range into part[k*nb + bx] (and squares into
// part2). flags: bit0 non-finite value, bit1 negative value. zero_count counts
// exact zeros (used for weights, d == 1).
__global__ void coord_stats_kernel(const float *__restrict__ v, int64_t cnt, int d,
                                   int64_t per_block, double *part, double *part2, int *flags,
                                   unsigned long long *zero_count) {
    __shared__ double s1[kStatThreads / 32], s2[kStatThreads / 32];
    const int k = blockIdx.y, tid = threadIdx.x;
    const int64_t p0 = (int64_t)blockIdx.x * per_block;
    const int64_t p1 = min(p0 + per_block, cnt);
    double a1 = 0.0, a2 = 0.0;
    int fl = 0;
    unsigned long long zc = 0;
    for (int64_t p = p0 + tid; p < p1; p += kStatThreads) {
        const float val = v[p * d + k];
        if (!isfinite(val)) fl |= 1;
        if (val < 0.0f) fl |= 2;
        if (val == 0.0f) ++zc;
        a1 += (double)val;
        a2 += (double)val * (double)val;
    }
    for (int off = 16; off > 0; off >>= 1) {
        a1 += __shfl_xor_sync(0xffffffffu, a1, off);
        a2 += __shfl_xor_sync(0xffffffffu, a2, off);
    }
    if ((tid & 31) == 0) {
        s1[tid >> 5] = a1;
        s2[tid >> 5] = a2;
    }
    if (fl) atomicOr(flags, fl);
    if (zc && zero_count) atomicAdd(zero_count, zc);
    __syncthreads();
    if (tid == 0) {
        double t1 = 0.0, t2 = 0.0;
        for (int w = 0; w < kStatThreads / 32; ++w) {
            t1 += s1[w];
            t2 += s2[w];
        }
        part[(int64_t)k * gridDim.x + blockIdx.x] = t1;
        part2[(int64_t)k * gridDim.x + blockIdx.x] = t2;
    }
}

// Sums the block partials of coord_stats in block order: out[k] = sum, out2[k]
// = sum of squares, for k < d.
__global__ void sum_parts_kernel(const double *part, const double *part2, int nb, int d,
                                 double *out, double *out2) {
    const int k = blockIdx.x;
    if (threadIdx.x != 0 || k >= d) return;
    double t1 = 0.0, t2 = 0.0;
    for (int b = 0; b < nb; ++b) {
        t1 += part[(int64_t)k * nb + b];
        t2 += part2[(int64_t)k * nb + b];
    }
    out[k] = t1;
    out2[k] = t2;
}

// ---------------------------------------------------------- max-cost pass
// max over all pairs of ||x_i - y_j||^2 (fp32 coordinate differences). Each thread owns 4 rows; columns stream through shared
// memory. The max is order-free, so the float-as-uint atomicMax is exact and
// deterministic (values are >= 0).
constexpr int kMaxThreads = 128, kMaxRows = 4, kMaxChunk = 64;

__global__ void __launch_bounds__(kMaxThreads) max_cost_kernel(const float *__restrict__ x,
                                                               const float *__restrict__ y,
                                                               int64_t n, int64_t m, int d,
                                                               unsigned *out_bits) {
    __shared__ float sy[kMaxChunk * kMaxD];
    __shared__ float s_red[kMaxThreads / 32];
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)blockIdx.x * kMaxThreads * kMaxRows;
    float best = 0.0f;
    for (int64_t c0 = 0; c0 < m; c0 += kMaxChunk) {
        const int cn = (int)min((int64_t)kMaxChunk, m - c0);
        __syncthreads();
        for (int u = tid; u < cn * d; u += kMaxThreads) sy[u] = y[c0 * d + u];
        __syncthreads();
        for (int r = 0; r < kMaxRows; ++r) {
            const int64_t i = r0 + r * kMaxThreads + tid;
            if (i >= n) break;
            const float *xi = x + i * d;
            for (int j = 0; j < cn; ++j) {
                float s = 0.0f;
                for (int q = 0; q < d; ++q) {
                    const float t = xi[q] - sy[j * d + q];
                    s = fmaf(t, t, s);
                }
                best = fmaxf(best, s);
            }
        }
    }
    for (int off = 16; off > 0; off >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
    if ((tid & 31) == 0) s_red[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
        float b = 0.0f;
        for (int w = 0; w < kMaxThreads / 32; ++w) b = fmaxf(b, s_red[w]);
        atomicMax(out_bits, __float_as_uint(b));
    }
}

// ----------------------------------------------------------------- params
__global__ void set_params_kernel(Params *prm, double eps, double c, double tol, double *hist,
                                  int64_t hist_off, int64_t hist_len) {
    prm->eps = eps;
    prm->kappa = kLog2e / eps;
    prm->c = c;
    prm->tol = tol;
    prm->hist = hist;
    prm->hist_off = hist_off;
    prm->hist_len = hist_len;
}

__global__ void reset_state_kernel(State *st) {
    st->stop = 0;
    st->wait_timeout = 0;
    st->iter_done = 0;
    st->conv_iter = -1;
    st->resid[0] = st->resid[1] = -1.0;
    st->tiles_done[0] = st->tiles_done[1] = 0;
    st->work[0] = st->work[1] = 0;
}

// ----------------------------------------------------------------- tables
// For one cloud p [cnt, d] with potential pot [cnt] (the potential that the
// OTHER half-step reads as its column term), at the current stage's kappa, c:
//  rowtab [cnt_pad][dp]: p' = p - o in fp32, zero past d and past cnt;
//  coltab: Y = 2 c kappa p', G = kappa (pot - c |p'|^2) (|p'|^2 in float64 of
//    the fp32 p'), padding columns Y = 0, G = -inf.
//    layout 0 (d <= 3, dp == 4): column pair (2q, 2q+1) -> 8 floats
//      [Y0 Y0' Y1 Y1' Y2 Y2' G G'];
//    layout 1 (generic): [cnt_pad][dp + 4] = [Y_0 .. Y_{dp-1}, G, 0, 0, 0].
__global__ void build_tables_kernel(const float *__restrict__ p, const float *__restrict__ pot,
                                    int64_t cnt, int64_t cnt_pad, int d, int dp,
                                    const double *__restrict__ o, const Params *__restrict__ prm,
                                    float *rowtab, float *coltab, int layout) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= cnt_pad) return;
    const double kappa = prm->kappa, c = prm->c;
    const bool real = i < cnt;
    double nrm = 0.0;
    for (int q = 0; q < dp; ++q) {
        const float v = (real && q < d) ? (float)((double)p[i * d + q] - o[q]) : 0.0f;
        rowtab[i * dp + q] = v;
        nrm += (double)v * (double)v;
    }
    float G = -INFINITY;
    if (real) {
        const float pv = pot[i];
        G = (pv == -INFINITY) ? -INFINITY : (float)(kappa * ((double)pv - c * nrm));
    }
    if (layout == 0) {
        float *base = coltab + (i >> 1) * 8 + (i & 1);
        for (int q = 0; q < 3; ++q) base[2 * q] = (float)(2.0 * c * kappa * (double)rowtab[i * dp + q]);
        base[6] = G;
    } else {
        float *base = coltab + i * (dp + 4);
        for (int q = 0; q < dp; ++q) base[q] = (float)(2.0 * c * kappa * (double)rowtab[i * dp + q]);
        base[dp] = G;
        base[dp + 1] = base[dp + 2] = base[dp + 3] = 0.0f;
    }
}


// ----------------------------------------------------------------- launchers
// Column sums (and sums of squares) of v [cnt, d] into out[d], out2[d], in a
// fixed order; part/part2 hold at least d * 1024 doubles each.
cudaError_t launch_coord_stats(const float *v, int64_t cnt, int d, double *part, double *part2,
                               double *out, double *out2, int *flags,
                               unsigned long long *zero_count, cudaStream_t s) {
    const int64_t per_block = std::max<int64_t>(4096, (cnt + 1023) / 1024);
    const int nb = (int)std::max<int64_t>(1, (cnt + per_block - 1) / per_block);
    coord_stats_kernel<<<dim3(nb, d), kStatThreads, 0, s>>>(v, cnt, d, per_block, part, part2,
                                                            flags, zero_count);
    sum_parts_kernel<<<d, 32, 0, s>>>(part, part2, nb, d, out, out2);
    return cudaGetLastError();
}

// d <= 3: max_j ||x'_i - y'_j||^2 = |x'_i|^2 + max_j (|y'_j|^2 - 2 x'_i . y'_j) on the
// shifted coordinates (fp32, packed f32x2 FMAs, 3-input max): thread owns 8
// rows, 256 columns per shared-memory chunk, stored as column pairs
// [y0 y0' y1 y1' y2 y2' |y|^2 |y'|^2].
template <int D>
__global__ void __launch_bounds__(128) max_cost_lowd_kernel(const float *__restrict__ x,
                                                            const float *__restrict__ y,
                                                            int64_t n, int64_t m,
                                                            const double *__restrict__ o,
                                                            unsigned *out_bits) {
    constexpr int R = 8, CH = 256;
    __shared__ __align__(16) float4 sm[CH];
    __shared__ float s_red[4];
    const int tid = threadIdx.x;
    float ov[3] = {0.f, 0.f, 0.f};
    for (int q = 0; q < D; ++q) ov[q] = (float)o[q];
    float2 xm[R][3];
    float nx[R], best[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const int64_t i = ((int64_t)blockIdx.x * R + k) * 128 + tid;
        float v[3] = {0.f, 0.f, 0.f};
        if (i < n)
            for (int q = 0; q < D; ++q) v[q] = x[i * D + q] - ov[q];
        nx[k] = v[0] * v[0] + v[1] * v[1] + v[2] * v[2];
        for (int q = 0; q < 3; ++q) xm[k][q] = make_float2(-2.f * v[q], -2.f * v[q]);
        best[k] = -INFINITY;
    }
    for (int64_t c0 = 0; c0 < m; c0 += CH) {
        __syncthreads();
        for (int u = tid; u < CH / 2; u += 128) {
            float a[3] = {0.f, 0.f, 0.f}, b[3] = {0.f, 0.f, 0.f};
            const int64_t j = c0 + 2 * u;
            float na = -INFINITY, nb = -INFINITY;  // padding columns never win
            if (j < m) {
                for (int q = 0; q < D; ++q) a[q] = y[j * D + q] - ov[q];
                na = a[0] * a[0] + a[1] * a[1] + a[2] * a[2];
            }
            if (j + 1 < m) {
                for (int q = 0; q < D; ++q) b[q] = y[(j + 1) * D + q] - ov[q];
                nb = b[0] * b[0] + b[1] * b[1] + b[2] * b[2];
            }
            sm[2 * u] = make_float4(a[0], b[0], a[1], b[1]);
            sm[2 * u + 1] = make_float4(a[2], b[2], na, nb);
        }
        __syncthreads();
        const int cn = (int)min((int64_t)CH, m - c0);
        for (int q8 = 0; q8 < cn; q8 += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = sm[q8 + u];
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 t[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const float4 lo = v[2 * pp], hi = v[2 * pp + 1];
                    float2 tt = __ffma2_rn(make_float2(lo.x, lo.y), xm[k][0], make_float2(hi.z, hi.w));
                    if (D >= 2) tt = __ffma2_rn(make_float2(lo.z, lo.w), xm[k][1], tt);
                    if (D >= 3) tt = __ffma2_rn(make_float2(hi.x, hi.y), xm[k][2], tt);
                    t[pp] = tt;
                }
                best[k] = fmax3(best[k], fmax3(t[0].x, t[0].y, t[1].x), fmax3(t[1].y, t[2].x, t[2].y));
                best[k] = fmax3(best[k], t[3].x, t[3].y);
            }
        }
    }
    float b = 0.0f;
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const int64_t i = ((int64_t)blockIdx.x * R + k) * 128 + tid;
        if (i < n) b = fmaxf(b, fmaxf(best[k] + nx[k], 0.0f));
    }
    for (int off = 16; off > 0; off >>= 1) b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, off));
    if ((tid & 31) == 0) s_red[tid >> 5] = b;
    __syncthreads();
    if (tid == 0) atomicMax(out_bits, __float_as_uint(fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]))));
}

cudaError_t launch_max_cost(const float *x, const float *y, int64_t n, int64_t m, int d,
                            const double *o, unsigned *out_bits, cudaStream_t s) {
    if (d <= 3) {
        const unsigned grid = (unsigned)((n + 8 * 128 - 1) / (8 * 128));
        if (d == 1) max_cost_lowd_kernel<1><<<grid, 128, 0, s>>>(x, y, n, m, o, out_bits);
        else if (d == 2) max_cost_lowd_kernel<2><<<grid, 128, 0, s>>>(x, y, n, m, o, out_bits);
        else max_cost_lowd_kernel<3><<<grid, 128, 0, s>>>(x, y, n, m, o, out_bits);
        return cudaGetLastError();
    }
    const int64_t rows_per_block = (int64_t)kMaxThreads * kMaxRows;
    max_cost_kernel<<<(unsigned)((n + rows_per_block - 1) / rows_per_block), kMaxThreads, 0, s>>>(
        x, y, n, m, d, out_bits);
    return cudaGetLastError();
}

cudaError_t launch_set_params(Params *prm, double eps, double c, double tol, double *hist,
                              int64_t hist_off, int64_t hist_len, cudaStream_t s) {
    set_params_kernel<<<1, 1, 0, s>>>(prm, eps, c, tol, hist, hist_off, hist_len);
    return cudaGetLastError();
}

cudaError_t launch_reset_state(State *st, cudaStream_t s) {
    reset_state_kernel<<<1, 1, 0, s>>>(st);
    return cudaGetLastError();
}

cudaError_t launch_tables(const float *p, const float *pot, int64_t cnt, int64_t cnt_pad, int d,
                          int dp, const double *o, const Params *prm, float *rowtab,
                          float *coltab, int layout, cudaStream_t s) {
    build_tables_kernel<<<(unsigned)((cnt_pad + 255) / 256), 256, 0, s>>>(
        p, pot, cnt, cnt_pad, d, dp, o, prm, rowtab, coltab, layout);
    return cudaGetLastError();
}

}  // namespace ot
