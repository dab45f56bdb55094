// noalloc.cu -- ot_marginal_residual_noalloc: the marginal residual computed
// without allocating any memory.
//
// Some callers cannot allocate device memory at the point where they need a
// residual: a process whose device memory is entirely owned by another
// allocator (a framework's caching pool, a fixed budget reserved at start-up),
// or a latency-sensitive loop in which cudaMalloc/cudaFree would stall every
// stream of the device. For them this variant of the residual row pass takes
// its scratch from a fixed array that lives in the library's device image
// instead of a plan's workspace, and needs no plan: the caller passes the
// inputs and the potentials and gets the two sums back.
//
// The arithmetic per entry is the same plan entry as everywhere else,
// T_ij = exp((f_i + g_j - C_ij)/eps), with the exponent built in float64, here
// from coordinate differences read straight from x and y (no column table), and
// each row's sum kept inside one block, so the result is deterministic.
#include <cmath>
#include <mutex>

#include "ot_sinkhorn.h"
#include "runtime.h"

namespace ot {

// one partial per block of 8 rows for clouds of up to OT_NOALLOC_MAX_POINTS
// points, plus the two results
constexpr int kNaRows = 8, kNaThreads = 256;
constexpr int64_t kNaPartials = OT_NOALLOC_MAX_POINTS / kNaRows;
constexpr int64_t kNaScratch = kNaPartials + 2;

// Device scratch shared by every call on a device, kept until the process exits
// (1 MiB + 16 bytes). Host code must not pass this name to a kernel: on the host
// it is only a stand-in; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) double g_na_scratch[kNaScratch];

__device__ __forceinline__ float na_exp2_split(double e2) {
    if (!(e2 > -152.0)) return 0.0f;
    if (e2 >= 128.0) return INFINITY;
    const int k = __double2int_rn(e2);
    const float p = ex2_approx((float)(e2 - (double)k));
    if (k >= -125) return __int_as_float(__float_as_int(p) + (k << 23));
    return p * __int_as_float((k + 64 + 127) << 23) * 5.42101086242752217e-20f;
}

// part[block] = sum over the block's rows i of |sum_j T_ij - w_i|, rows = (pts,
// pot, w), columns = (cpts, cpot); kappa = log2(e)/eps, c = inv_scale_cost.
template <int D>
__global__ void __launch_bounds__(kNaThreads) na_rowsum_kernel(
    const float *__restrict__ pts, const float *__restrict__ pot, const float *__restrict__ w,
    const float *__restrict__ cpts, const float *__restrict__ cpot, int64_t rows, int64_t cols,
    int d, double kappa, double c, double *part) {
    __shared__ double sx[kNaRows][D > 0 ? D : kMaxD], sf[kNaRows];
    __shared__ double sred[kNaThreads / 32][kNaRows];
    const int tid = threadIdx.x;
    const int dd = D > 0 ? D : d;
    const int64_t r0 = (int64_t)blockIdx.x * kNaRows;
    if (tid < kNaRows) {
        const int64_t i = r0 + tid;
        for (int q = 0; q < dd; ++q) sx[tid][q] = i < rows ? (double)pts[i * dd + q] : 0.0;
        const float pv = i < rows ? pot[i] : -INFINITY;
        sf[tid] = pv == -INFINITY ? -INFINITY : kappa * (double)pv;
    }
    __syncthreads();
    double acc[kNaRows];
#pragma unroll
    for (int r = 0; r < kNaRows; ++r) acc[r] = 0.0;
    for (int64_t j = tid; j < cols; j += kNaThreads) {
        const float gv = cpot[j];
        if (gv == -INFINITY) continue;
        const double kg = kappa * (double)gv;
        double yj[D > 0 ? D : kMaxD];
        for (int q = 0; q < dd; ++q) yj[q] = (double)cpts[j * dd + q];
#pragma unroll
        for (int r = 0; r < kNaRows; ++r) {
            double s = 0.0;
            for (int q = 0; q < dd; ++q) {
                const double t = sx[r][q] - yj[q];
                s = fma(t, t, s);
            }
            acc[r] += (double)na_exp2_split(sf[r] + kg - kappa * c * s);
        }
    }
#pragma unroll
    for (int r = 0; r < kNaRows; ++r) {
        double v = acc[r];
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if ((tid & 31) == 0) sred[tid >> 5][r] = v;
    }
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int r = 0; r < kNaRows; ++r) {
            const int64_t i = r0 + r;
            if (i >= rows) break;
            double v = 0.0;
            for (int wv = 0; wv < kNaThreads / 32; ++wv) v += sred[wv][r];
            t += fabs(v - (double)w[i]);
        }
        part[blockIdx.x] = t;
    }
}

// out = sum of part[0..cnt) in a fixed order (one block)
__global__ void __launch_bounds__(1024) na_sum_kernel(const double *part, int64_t cnt, double *out) {
    __shared__ double s[1024];
    double a = 0.0;
    for (int64_t i = threadIdx.x; i < cnt; i += 1024) a += part[i];
    s[threadIdx.x] = a;
    __syncthreads();
    for (int st = 512; st > 0; st >>= 1) {
        if (threadIdx.x < st) s[threadIdx.x] += s[threadIdx.x + st];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = s[0];
}

static cudaError_t na_pass(const float *pts, const float *pot, const float *w, const float *cpts,
                           const float *cpot, int64_t rows, int64_t cols, int d, double kappa,
                           double c, double *scratch, double *out, cudaStream_t s) {
    const unsigned grid = (unsigned)((rows + kNaRows - 1) / kNaRows);
    switch (d) {
        case 1: na_rowsum_kernel<1><<<grid, kNaThreads, 0, s>>>(pts, pot, w, cpts, cpot, rows, cols, d, kappa, c, scratch); break;
        case 2: na_rowsum_kernel<2><<<grid, kNaThreads, 0, s>>>(pts, pot, w, cpts, cpot, rows, cols, d, kappa, c, scratch); break;
        case 3: na_rowsum_kernel<3><<<grid, kNaThreads, 0, s>>>(pts, pot, w, cpts, cpot, rows, cols, d, kappa, c, scratch); break;
        default: na_rowsum_kernel<0><<<grid, kNaThreads, 0, s>>>(pts, pot, w, cpts, cpot, rows, cols, d, kappa, c, scratch); break;
    }
    na_sum_kernel<<<1, 1024, 0, s>>>(scratch, grid, out);
    return cudaGetLastError();
}

}  // namespace ot

namespace {

constexpr int kNaMaxDevices = 64;
std::mutex g_na_mutex;
double *g_na_addr[kNaMaxDevices] = {};  // device address of g_na_scratch, per device

}  // namespace

// The scratch's device address is looked up once per device, on the first call
// made with that device current (cudaGetSymbolAddress, return code checked).
extern "C" int ot_marginal_residual_noalloc(const float *x, const float *y, const float *a,
                                            const float *b, const float *f, const float *g,
                                            int64_t n, int64_t m, int32_t d, double eps,
                                            double inv_scale_cost, double *row_l1,
                                            double *col_l1, void *stream) {
    using namespace ot;
    NvtxRange nvtx_range("ot_marginal_residual_noalloc");
    if (!x || !y || !a || !b || !f || !g) return set_error(OT_ERR_INVALID_ARG, "null array pointer");
    if (n < 1 || m < 1) return set_error(OT_ERR_INVALID_ARG, "n and m must be >= 1");
    if (n > OT_NOALLOC_MAX_POINTS || m > OT_NOALLOC_MAX_POINTS)
        return set_error(OT_ERR_UNSUPPORTED,
                         "n=%lld, m=%lld: the allocation-free residual takes at most %d points "
                         "per cloud (use ot_marginal_residual on a plan)",
                         (long long)n, (long long)m, OT_NOALLOC_MAX_POINTS);
    if (d < 1 || d > kMaxD) return set_error(d < 1 ? OT_ERR_INVALID_ARG : OT_ERR_UNSUPPORTED, "d=%d outside 1..%d", d, kMaxD);
    if (!(eps > 0.0) || !std::isfinite(eps)) return set_error(OT_ERR_INVALID_ARG, "eps must be > 0 and finite");
    if (!(inv_scale_cost > 0.0) || !std::isfinite(inv_scale_cost))
        return set_error(OT_ERR_INVALID_ARG, "inv_scale_cost must be > 0 and finite");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(OT_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kNaMaxDevices) return set_error(OT_ERR_UNSUPPORTED, "device index %d too large", dev);
    double *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_na_mutex);
        if (!g_na_addr[dev]) {
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_na_scratch);
            if (e != cudaSuccess || !ptr)
                return set_error(OT_ERR_CUDA, "cudaGetSymbolAddress of the scratch failed: %s",
                                 cudaGetErrorString(e));
            g_na_addr[dev] = static_cast<double *>(ptr);
        }
        scratch = g_na_addr[dev];
    }
    cudaStream_t s = (cudaStream_t)stream;
    const double kappa = kLog2e / eps;
    double *res = scratch + kNaPartials;
    e = na_pass(x, f, a, y, g, n, m, d, kappa, inv_scale_cost, scratch, res, s);
    if (e == cudaSuccess) e = na_pass(y, g, b, x, f, m, n, d, kappa, inv_scale_cost, scratch, res + 1, s);
    double host[2] = {0.0, 0.0};
    if (e == cudaSuccess) e = cudaMemcpyAsync(host, res, sizeof host, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(OT_ERR_CUDA, "allocation-free residual failed: %s", cudaGetErrorString(e));
    if (row_l1) *row_l1 = host[0];
    if (col_l1) *col_l1 = host[1];
    return OT_OK;
}
