// rows.cu -- plan entries: row materializer, exact min_row, marginal residual.
//
// Every entry of the plan is T_ij = exp((f_i + g_j - C_ij)/eps) (moscot PR
// #846, "materialize transport-matrix rows instead of pushing indicator
// columns", section Fix), produced by ONE device function, plan_entry(), so the
// min_row threshold and the values it is compared with come from the same
// float path ("Behavioural changes": the old threshold and values came from two
// paths and could empty a row).
//
// Precision. In base 2 with kappa = log2(e)/eps and the shifted coordinates
// x' = x - o, y' = y - o held in float64:
//   e2_ij = A_i + B_j + sum_q P_iq y'_jq,
//   A_i = kappa (f_i - c |x'_i|^2), B_j = kappa (g_j - c |y'_j|^2), P_i = 2 c kappa x'_i,
// all in float64 (FlashSinkhorn 2, section D.3: accurate evaluation is done in
// FP64). The sum is formed on t = kShift + e2 rather than on e2: kShift = 1.5 *
// 2^29 + 126 keeps t in [2^29, 2^30), where a float64 step is 2^-23, so every
// operation rounds e2 to a multiple of 2^-23 (at most 2^-24 off, ~2e-7 relative
// in T after the five operations) and the low 32 bits of t are the integer
// (126 + e2) * 2^23 -- the range reduction is then two integer operations: the
// fraction of e2 goes into the mantissa of a float in [1, 2), whose MUFU ex2
// (relative error ~2^-22) is scaled by 2^floor(e2) through the exponent field.
// The range takes two float64 compares and an integer min: for e2 in
// [-126, 386) t lies in [kBase, kBase + 512) (kBase = 1.5 * 2^29), where the low
// word is exact; the integer min caps it at e2 = 128, where the exponent field
// saturates to +inf exactly; below -126 T is returned as 0 (entries under
// 2^-126 = 1.2e-38, the smallest normal float, are flushed; a massless side,
// potential -inf, lands there) and from 386 on as +inf. Per entry: d + 1 float64
// FMAs/adds, two float64 compares, three integer operations, two selects, one
// ex2. Where a tile bound proves e2 < 128 for all its entries, the row passes
// use exp2_shifted_capped: one integer compare of the high word replaces both
// float64 compares, the cap and a select, with the same value bit for bit.
// The row passes accumulate each row's terms 8 at a time in float32 and those
// partial sums in float64 (maxima and counts exactly).
#include <type_traits>

#include "runtime.h"

namespace ot {

constexpr double kShift = 805306368.0 + 126.0;  // 1.5 * 2^29 + 126
constexpr double kShiftLo = kShift - 126.0;     // e2 >= -126 (else 0)
constexpr double kShiftHi = kShift + 386.0;     // e2 < 386 (else +inf)

// T = 2^e2 from t = kShift + e2 (see above).
__device__ __forceinline__ float exp2_shifted(double t) {
    const unsigned q = min((unsigned)__double2loint(t), 254u << 23);  // (126 + e2) * 2^23, capped
    const unsigned mant = (q & 0x7FFFFFu) | 0x3F800000u;              // 1 + frac(e2), in [1, 2)
    const float p = ex2_approx(__uint_as_float(mant));                 // 2^(1 + frac(e2)), in [2, 4]
    // exponent field + floor(e2) - 1: q - mant = (floor(e2) - 1) * 2^23
    const float v = __uint_as_float(__float_as_uint(p) + q - mant);
    const float r = t >= kShiftLo ? v : 0.0f;
    return t < kShiftHi ? r : INFINITY;
}

// The same for an e2 known to lie below 128 (a tile whose bound says so): the
// high word of t is that of kShift - 126 exactly when e2 >= -126 (t in
// [2^29 * 1.5, 2^29 * 1.5 + 512)), which takes the place of both range tests
// and of the cap; the value is bit for bit that of exp2_shifted.
constexpr unsigned kBaseHi = 0x41C80000u;  // high word of 1.5 * 2^29
__device__ __forceinline__ float exp2_shifted_capped(double t) {
    const unsigned lo = (unsigned)__double2loint(t);
    const unsigned mant = (lo & 0x7FFFFFu) | 0x3F800000u;
    const float p = ex2_approx(__uint_as_float(mant));
    const float v = __uint_as_float(__float_as_uint(p) + lo - mant);
    return (unsigned)__double2hiint(t) == kBaseHi ? v : 0.0f;
}

// the one float path for a plan entry: row data (A' = A + kShift, P[d]),
// column data (y'[d], B)
template <int D>
__device__ __forceinline__ float plan_entry(double Ash, const double *P, const double *col, int d) {
    const int dd = D > 0 ? D : d;
    double t = Ash + col[dd];
#pragma unroll
    for (int q = 0; q < (D > 0 ? D : 1); ++q) {
        if (D > 0) t = fma(P[q], col[q], t);
    }
    if (D == 0)
        for (int q = 0; q < dd; ++q) t = fma(P[q], col[q], t);
    return exp2_shifted(t);
}

// plan_entry for an entry known to lie below 2^128 (d <= 3)
template <int D>
__device__ __forceinline__ float plan_entry_capped(double Ash, const double *P, const double *col) {
    double t = Ash + col[D];
#pragma unroll
    for (int q = 0; q < D; ++q) t = fma(P[q], col[q], t);
    return exp2_shifted_capped(t);
}

// Column table in float64: dcol[j*(d+1) + q] = y'_jq (q < d), dcol[j*(d+1) + d] = B_j,
// for the column perm[j] (perm NULL: column j).
__global__ void build_dcol_kernel(const float *__restrict__ p, const float *__restrict__ pot,
                                  int64_t cnt, int d, const double *__restrict__ o,
                                  const Params *__restrict__ prm, const int64_t *__restrict__ perm,
                                  double *dcol) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= cnt) return;
    const int64_t src = perm ? perm[j] : j;
    const double kappa = prm->kappa, c = prm->c;
    double nrm = 0.0;
    for (int q = 0; q < d; ++q) {
        const double v = (double)p[src * d + q] - o[q];
        dcol[j * (d + 1) + q] = v;
        nrm += v * v;
    }
    const float pv = pot[src];
    dcol[j * (d + 1) + d] = (pv == -INFINITY) ? -INFINITY : kappa * ((double)pv - c * nrm);
}

// Summary of each chunk of kRpChunk consecutive columns of the column table
// (d <= 3), for the tile screen of the row passes: csum[7c .. 7c+2] and
// [7c+3 .. 7c+5] the chunk's box in y' (0 past d), csum[7c+6] = max over its
// columns of kappa g_j = B_j + kappa c |y'_j|^2 (-inf if every column is
// massless). One warp per chunk.
constexpr int kRpChunkC = 256;
__global__ void chunk_summary_kernel(const double *__restrict__ dcol, int64_t cnt, int d,
                                     const Params *__restrict__ prm, double *csum) {
    const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = (cnt + kRpChunkC - 1) / kRpChunkC;
    if (chunk >= nchunks) return;
    const double kc = prm->kappa * prm->c;
    double lo[3] = {INFINITY, INFINITY, INFINITY}, hi[3] = {-INFINITY, -INFINITY, -INFINITY};
    double gmax = -INFINITY;
    const int64_t j1 = min(cnt, (chunk + 1) * kRpChunkC);
    for (int64_t j = chunk * kRpChunkC + lane; j < j1; j += 32) {
        double nrm = 0.0;
        for (int q = 0; q < d; ++q) {
            const double v = dcol[j * (d + 1) + q];
            lo[q] = fmin(lo[q], v);
            hi[q] = fmax(hi[q], v);
            nrm += v * v;
        }
        const double B = dcol[j * (d + 1) + d];
        if (B != -INFINITY) gmax = fmax(gmax, B + kc * nrm);
    }
    for (int off = 16; off > 0; off >>= 1) {
        for (int q = 0; q < 3; ++q) {
            lo[q] = fmin(lo[q], __shfl_xor_sync(0xffffffffu, lo[q], off));
            hi[q] = fmax(hi[q], __shfl_xor_sync(0xffffffffu, hi[q], off));
        }
        gmax = fmax(gmax, __shfl_xor_sync(0xffffffffu, gmax, off));
    }
    if (lane == 0) {
        for (int q = 0; q < 3; ++q) {
            csum[chunk * 7 + q] = q < d ? lo[q] : 0.0;
            csum[chunk * 7 + 3 + q] = q < d ? hi[q] : 0.0;
        }
        csum[chunk * 7 + 6] = gmax;
    }
}

// perm[r] = off + the point index in the r-th sorted Morton key
__global__ void perm_from_keys_kernel(const unsigned long long *keys, int64_t cnt, int64_t off,
                                      int64_t *perm) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r < cnt) perm[r] = off + (int64_t)(keys[r] & 0xffffffffull);
}

// Row data of one row: A' = A + kShift and P (d values).
__device__ __forceinline__ void load_row(const float *pts, const float *pot, int64_t i, int d,
                                         const double *o, double kappa, double c, double *A,
                                         double *P) {
    double nrm = 0.0;
    for (int q = 0; q < d; ++q) {
        const double v = (double)pts[i * d + q] - o[q];
        P[q] = 2.0 * c * kappa * v;
        nrm += v * v;
    }
    const float pv = pot[i];
    *A = (pv == -INFINITY) ? -INFINITY : kappa * ((double)pv - c * nrm) + kShift;
}

// ------------------------------------------------------------ materializer
// Block: 256 threads x 4 consecutive columns (1024 columns). A block keeps its
// columns' float64 data in registers (d <= 3) and walks a range of up to 256
// rows of the row list, staged 32 at a time through shared memory; each row is
// one coalesced float4 evict-first store per thread. The kernel is bound by
// the latency of each entry's float64 chain, so occupancy matters more than
// rows in flight: 4 blocks per SM with 2 rows unrolled (measured at 4096 x 1e5,
// d = 3: 2.63 TB/s written, against 2.29 at 3 blocks per SM, 4 rows).
constexpr int kMtThreads = 256, kMtStage = 32, kMtRowsPerBlock = 256;

template <int D>
__global__ void __launch_bounds__(kMtThreads, 4) materialize_kernel(MatArgs M) {
    __shared__ double sA[kMtStage], sP[kMtStage][D > 0 ? D : kMaxD];
    __shared__ int sValid[kMtStage];
    const int tid = threadIdx.x;
    const int d = D > 0 ? D : M.d;
    const int64_t j0 = ((int64_t)blockIdx.x * kMtThreads + tid) * 4;
    const int ncol = j0 < M.m ? (int)min((int64_t)4, M.m - j0) : 0;
    constexpr int DS = (D > 0 ? D : 1) + 1;
    double cd[4][DS];
    if (D > 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int q = 0; q < DS; ++q)
                cd[u][q] = u < ncol ? M.dcol[(j0 + u) * DS + q] : (q == DS - 1 ? -INFINITY : 0.0);
    }
    const int64_t rb0 = (int64_t)blockIdx.y * kMtRowsPerBlock;
    const int64_t rb1 = min(rb0 + kMtRowsPerBlock, M.k);
    for (int64_t s0 = rb0; s0 < rb1; s0 += kMtStage) {
        __syncthreads();
        if (tid < kMtStage) {
            const int64_t r = s0 + tid;
            int ok = 0;
            if (r < rb1) {
                const int64_t i = M.row_idx[r];
                if (i >= 0 && i < M.n) {
                    ok = 1;
                    load_row(M.x, M.f, i, d, M.o, M.prm->kappa, M.prm->c, &sA[tid], sP[tid]);
                } else {
                    atomicExch(M.bad, 1);
                }
            }
            sValid[tid] = ok;
        }
        __syncthreads();
        if (ncol == 0) continue;
        const int nr = (int)min((int64_t)kMtStage, rb1 - s0);
        const bool full = M.vec && ncol == 4;
        float *dst = M.out + s0 * M.m + j0;
#pragma unroll 2
        for (int rr = 0; rr < nr; ++rr, dst += M.m) {
            if (!sValid[rr]) continue;  // the same for every thread of the block
            float t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                // a column past m carries B = -inf and gives 0, never stored
                if (D > 0)
                    t[u] = plan_entry<D>(sA[rr], sP[rr], cd[u], d);
                else
                    t[u] = u < ncol ? plan_entry<0>(sA[rr], sP[rr], M.dcol + (j0 + u) * (d + 1), d)
                                    : 0.0f;
            }
            if (full) {
                __stcs(reinterpret_cast<float4 *>(dst), make_float4(t[0], t[1], t[2], t[3]));
            } else {
                for (int u = 0; u < ncol; ++u) __stcs(dst + u, t[u]);
            }
        }
    }
}

// Materializer for d > 3: the float64 exponent's dot product as a register-
// tiled product, as in rowpass_wide_kernel (its comment has the layout): a
// block takes 64 entries of the row list and a range of kMwChunks chunks of 64
// columns; each thread forms a 4 x 4 tile of entries in the order of
// plan_entry (the same values bit for bit) and stores 4 consecutive columns of
// each of its rows (one float4 streaming store when the row is aligned).
constexpr int kMwRows = 64, kMwCols = 64, kMwChunks = 16;

int64_t matwide_smem_bytes(int d) { return (int64_t)(d * (kMwRows + kMwCols) + kMwRows * 3 + kMwCols) * 8; }

__global__ void __launch_bounds__(256, 3) materialize_wide_kernel(MatArgs M) {
    extern __shared__ __align__(16) double msm[];
    const int d = M.d;
    double *sPt = msm;                    // [d][64]
    double *sYt = sPt + d * kMwRows;      // [d][64]
    double *sA = sYt + d * kMwCols;       // [64]
    double *sB = sA + kMwRows;            // [64]
    int64_t *sRow = reinterpret_cast<int64_t *>(sB + kMwCols);  // [64] output row, -1: skip
    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int64_t t0 = (int64_t)blockIdx.y * kMwRows;
    if (tid < kMwRows) {
        const int64_t t = t0 + tid;
        double P[kMaxD];
        double A = -INFINITY;
        int64_t out_row = -1;
        if (t < M.k) {
            const int64_t i = M.row_idx[t];
            if (i >= 0 && i < M.n) {
                load_row(M.x, M.f, i, d, M.o, M.prm->kappa, M.prm->c, &A, P);
                out_row = t;
            } else {
                atomicExch(M.bad, 1);
            }
        }
        if (out_row < 0)
            for (int q = 0; q < d; ++q) P[q] = 0.0;
        sA[tid] = A;
        sRow[tid] = out_row;
        for (int q = 0; q < d; ++q) sPt[q * kMwRows + tid] = P[q];
    }
    const int DS = d + 1;
    const int64_t cbeg = (int64_t)blockIdx.x * kMwChunks * kMwCols;
    const int64_t cend = min(M.m, cbeg + (int64_t)kMwChunks * kMwCols);
    for (int64_t c0 = cbeg; c0 < cend; c0 += kMwCols) {
        __syncthreads();  // the previous chunk is no longer read (and the rows are staged)
        for (int c = tid >> 5; c < kMwCols; c += 8) {
            const int64_t j = c0 + c;
            for (int q = tid & 31; q < DS; q += 32) {
                const double v = j < M.m ? M.dcol[j * DS + q] : (q == d ? -INFINITY : 0.0);
                if (q < d)
                    sYt[q * kMwCols + (c ^ ((q & 15) << 2))] = v;
                else
                    sB[c] = v;
            }
        }
        __syncthreads();
        double acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = sA[4 * rg + r] + sB[4 * cg + c];
#pragma unroll 2
        for (int q = 0; q < d; ++q) {
            const double *pq = &sPt[q * kMwRows + 4 * rg];
            const double2 p0 = *reinterpret_cast<const double2 *>(pq);
            const double2 p1 = *reinterpret_cast<const double2 *>(pq + 2);
            const double *yq = &sYt[q * kMwCols + ((4 * cg) ^ ((q & 15) << 2))];
            const double2 y0 = *reinterpret_cast<const double2 *>(yq);
            const double2 y1 = *reinterpret_cast<const double2 *>(yq + 2);
            const double pr[4] = {p0.x, p0.y, p1.x, p1.y}, yc[4] = {y0.x, y0.y, y1.x, y1.y};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fma(pr[r], yc[c], acc[r][c]);
        }
        const int64_t j0 = c0 + 4 * cg;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t orow = sRow[4 * rg + r];
            if (orow < 0 || j0 >= M.m) continue;
            float t[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) t[c] = exp2_shifted(acc[r][c]);
            float *dst = M.out + orow * M.m + j0;
            if (M.vec && j0 + 4 <= M.m) {
                __stcs(reinterpret_cast<float4 *>(dst), make_float4(t[0], t[1], t[2], t[3]));
            } else {
                for (int c = 0; c < 4 && j0 + c < M.m; ++c) __stcs(dst + c, t[c]);
            }
        }
    }
}

// ------------------------------------------------------- row-complete passes
// A pass visits every entry of a range of rows and reduces each row:
//   OP_MAX:   rowmax[i] = max_j T_ij                       (min_row, pass A)
//   OP_COUNT: counts[i] = #{j : T_ij >= thr} if w_i > 0    (min_row, pass B)
//   OP_SUM:   part[block] = sum over its rows of |sum_j T_ij - w_i|  (residual)
// "Rows" may be either cloud: the column residual runs the same pass with the
// roles of (x, f, a) and (y, g, b) swapped, since T is symmetric in them.
//
// d <= 3: a block of 8 warps owns 32 rows, 4 per warp, whose float64 data sit
// in registers; the columns' float64 records (y'[d], B) stream through shared
// memory 256 at a time (the next chunk prefetched into registers), so a column
// is read from L2 once per 32 rows and from shared memory once per 4 entries.
// 3 blocks per SM (85 registers): the entry is a chain of dependent float64
// operations, and more resident warps hide it better than more rows per warp
// (measured at n = m = 1e5: 4 rows x 3 blocks 32 % of the MUFU rate for the
// residual pass, 8 rows x 2 blocks 30 %).
// Lane l takes columns l, l + 32, ... of each chunk for all 4 rows of its warp,
// so every row's reduction stays in one warp, in a fixed lane order
// (deterministic). Sums: the 8 terms of a row in one chunk add up in float32,
// those partial sums in float64. With R.rperm the pass's positions are taken
// through that permutation (results still land at the row's own index); the
// column order is whatever the column table holds.
enum { OP_MAX = 0, OP_COUNT = 1, OP_SUM = 2 };
constexpr int kRpThreads = 256, kRpWarps = kRpThreads / 32, kRpR = 4, kRpChunk = kRpChunkC;
constexpr int kRpRows = kRpWarps * kRpR;  // rows per block, d <= 3 (32)
constexpr int kRgRows = 64;               // rows per block, d > 3
constexpr int kRpWin = 8192;              // chunks screened at a time (one bit each)

// Tile screen (d <= 3, R.csum set). The pass's rows come in Morton order
// (R.rperm), so a block's 32 rows are close together, and so are the columns
// of a chunk (the column table is in Morton order too). For rows I and the
// columns J of a chunk,
//   e2_ij = kappa (f_i + g_j) - kappa c |x'_i - y'_j|^2
//        <= kappa max_I f + kappa max_J g - kappa c dist(box(x'_I), box(y'_J))^2,
// and a chunk whose bound is below -127 is skipped: every entry of it is below
// 2^-126, where the entry function returns exactly 0 (the margin of one unit of
// e2 is far above the float64 rounding of the bound and of the entry), so row
// sums, maxima and counts at a threshold above 0 are the same as with every
// chunk visited. The block bounds its rows first (lane 0 of each warp, then one
// thread), then every thread screens kRpWin chunks at a time into a bit mask.
template <int D, int OP>
__global__ void __launch_bounds__(kRpThreads, 3) rowpass_kernel(RowPassArgs R) {
    constexpr int DS = D + 1;                 // doubles per column record
    constexpr int DP = D == 1 ? 2 : 4;        // padded stride in shared memory
    constexpr int PER = (kRpChunk * DS + kRpThreads - 1) / kRpThreads;  // prefetched doubles
    __shared__ __align__(16) double sc[kRpChunk * DP];
    __shared__ double sRed[kRpWarps][kRpR];
    __shared__ double sBox[kRpWarps + 1][7];  // per warp, then the block: lo[3], hi[3], kappa max f
    __shared__ unsigned sLive[kRpWin / 32], sSafe[kRpWin / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rw = R.row_begin + (int64_t)blockIdx.x * kRpRows + (int64_t)warp * kRpR;  // positions
    double Ash[kRpR], P[kRpR][D];
#pragma unroll
    for (int r = 0; r < kRpR; ++r) {
        if (rw + r < R.row_end) {
            const int64_t i = R.rperm ? R.rperm[rw + r] : rw + r;
            load_row(R.pts, R.pot, i, D, R.o, R.prm->kappa, R.prm->c, &Ash[r], P[r]);
        } else {
            Ash[r] = -INFINITY;
#pragma unroll
            for (int q = 0; q < D; ++q) P[r][q] = 0.0;
        }
    }
    if (R.csum) {
        if (lane == 0) {
            double b[7] = {INFINITY, INFINITY, INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
            for (int r = 0; r < kRpR; ++r) {
                if (rw + r >= R.row_end) break;
                const int64_t i = R.rperm ? R.rperm[rw + r] : rw + r;
                for (int q = 0; q < D; ++q) {
                    const double v = (double)R.pts[i * D + q] - R.o[q];
                    b[q] = fmin(b[q], v);
                    b[3 + q] = fmax(b[3 + q], v);
                }
                const float pv = R.pot[i];
                if (pv != -INFINITY) b[6] = fmax(b[6], R.prm->kappa * (double)pv);
            }
            for (int q = 0; q < 7; ++q) sBox[warp][q] = b[q];
        }
        __syncthreads();
        if (tid == 0) {
            for (int q = 0; q < 7; ++q) {
                double v = sBox[0][q];
                for (int w = 1; w < kRpWarps; ++w)
                    v = (q < 3) ? fmin(v, sBox[w][q]) : fmax(v, sBox[w][q]);
                sBox[kRpWarps][q] = v;
            }
        }
    }
    float mx[kRpR];
    int cnt[kRpR];
    double sum[kRpR];
#pragma unroll
    for (int r = 0; r < kRpR; ++r) {
        mx[r] = 0.0f;  // entries are >= 0, and a row has at least one
        cnt[r] = 0;
        sum[r] = 0.0;
    }
    // chunk c's records are elements [c * 256 * DS, (c + 1) * 256 * DS) of dcol;
    // thread t holds elements t, t + 256, ... of the next one
    const int64_t total = R.cols * DS;
    double pre[PER];
    auto fetch = [&](int64_t c0) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t e = c0 * DS + tid + (int64_t)k * kRpThreads;
            pre[k] = (tid + k * kRpThreads < kRpChunk * DS && e < total) ? __ldg(R.dcol + e)
                     : ((tid + k * kRpThreads) % DS == D ? -INFINITY : 0.0);
        }
    };
    const int64_t nchunks = (R.cols + kRpChunk - 1) / kRpChunk;
    const double kc = R.prm->kappa * R.prm->c;
    unsigned nvis = 0;  // chunks evaluated (the same in every thread)
    for (int64_t w0 = 0; w0 < nchunks; w0 += kRpWin) {
        const int nw = (int)min((int64_t)kRpWin, nchunks - w0);
        __syncthreads();  // the previous window's mask and chunk are no longer read
        for (int k = tid; k < ((nw + 31) & ~31); k += kRpThreads) {
            bool live = k < nw, safe = false;
            if (live && R.csum) {
                const double *cs = R.csum + (w0 + k) * 7;
                const double *bb = sBox[kRpWarps];
                double d2 = 0.0;
#pragma unroll
                for (int q = 0; q < D; ++q) {
                    const double gap = fmax(0.0, fmax(cs[q] - bb[3 + q], bb[q] - cs[3 + q]));
                    d2 = fma(gap, gap, d2);
                }
                const double bound = bb[6] + cs[6] - kc * d2;
                live = bound >= -127.0;
                safe = bound < 127.0;  // no entry reaches 2^128: the capped entry applies
            }
            const unsigned bal = __ballot_sync(0xffffffffu, live);
            const unsigned bsafe = __ballot_sync(0xffffffffu, safe);
            if (lane == 0) {
                sLive[k >> 5] = bal;
                sSafe[k >> 5] = bsafe;
            }
        }
        __syncthreads();
        auto next_live = [&](int k) {  // first chunk >= k of the window that is visited, or nw
            while (k < nw) {
                const unsigned word = sLive[k >> 5] >> (k & 31);
                if (word) return k + __ffs(word) - 1;
                k = (k | 31) + 1;
            }
            return nw;
        };
        int k = next_live(0);
        if (k < nw) fetch((w0 + k) * kRpChunk);
        while (k < nw) {
            const int64_t c0 = (w0 + k) * kRpChunk;
            ++nvis;
            __syncthreads();  // the previous chunk is no longer read
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = tid + u * kRpThreads;
                if (e < kRpChunk * DS) sc[(e / DS) * DP + (e % DS)] = pre[u];
            }
            __syncthreads();
            const int kn = next_live(k + 1);
            if (kn < nw) fetch((w0 + kn) * kRpChunk);
            // the chunk's entries; CAPPED: the tile bound keeps them below 2^128
            auto run_chunk = [&](auto capped) {
                constexpr bool CAPPED = decltype(capped)::value;
                float part[kRpR];
#pragma unroll
                for (int r = 0; r < kRpR; ++r) part[r] = 0.0f;
#pragma unroll 2
                for (int s2 = 0; s2 < kRpChunk / 32; ++s2) {
                    const int cc = s2 * 32 + lane;
                    double col[DP];
                    if (DP == 2) {
                        const double2 v = *reinterpret_cast<const double2 *>(&sc[cc * DP]);
                        col[0] = v.x;
                        col[1] = v.y;
                    } else {
                        const double2 v0 = *reinterpret_cast<const double2 *>(&sc[cc * DP]);
                        const double2 v1 = *reinterpret_cast<const double2 *>(&sc[cc * DP + 2]);
                        col[0] = v0.x;
                        col[1] = v0.y;
                        col[2] = v1.x;
                        col[3] = v1.y;
                    }
                    const bool live = c0 + cc < R.cols;
#pragma unroll
                    for (int r = 0; r < kRpR; ++r) {
                        const float t = CAPPED ? plan_entry_capped<D>(Ash[r], P[r], col)
                                               : plan_entry<D>(Ash[r], P[r], col, D);
                        if (OP == OP_MAX) mx[r] = fmaxf(mx[r], t);
                        if (OP == OP_COUNT) cnt[r] += (live && t >= R.thr) ? 1 : 0;
                        if (OP == OP_SUM) part[r] += t;
                    }
                }
                if (OP == OP_SUM) {
#pragma unroll
                    for (int r = 0; r < kRpR; ++r) sum[r] += (double)part[r];
                }
            };
            if ((sSafe[k >> 5] >> (k & 31)) & 1u)
                run_chunk(std::true_type{});
            else
                run_chunk(std::false_type{});
            k = kn;
        }
    }
    if (tid == 0 && R.visited) atomicAdd(R.visited, (unsigned long long)nvis);
    // per-row reductions across the warp (fixed order), then per block
#pragma unroll
    for (int r = 0; r < kRpR; ++r) {
        double v = OP == OP_SUM ? sum[r] : OP == OP_COUNT ? (double)cnt[r] : (double)mx[r];
        for (int off = 16; off > 0; off >>= 1) {
            const double o2 = __shfl_xor_sync(0xffffffffu, v, off);
            v = OP == OP_MAX ? fmax(v, o2) : v + o2;
        }
        if (lane == 0) {
            const int64_t pos = rw + r;
            double res = 0.0;
            if (pos < R.row_end) {
                const int64_t i = R.rperm ? R.rperm[pos] : pos;
                const float wi = R.w[i];
                if (OP == OP_MAX) R.rowmax[i] = (float)v;
                if (OP == OP_COUNT) R.counts[i] = wi > 0.0f ? (int64_t)v : 0;
                if (OP == OP_SUM) res = fabs(v - (double)wi);
            }
            sRed[warp][r] = res;
        }
    }
    if (OP == OP_SUM) {
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int w = 0; w < kRpWarps; ++w)
                for (int r = 0; r < kRpR; ++r) t += sRed[w][r];
            R.part[blockIdx.x] = t;
        }
    }
}

// d > 3: register-tiled float64 dot products. A block owns 64 rows (A' = A +
// kShift in sA, P transposed in sPt[q][r]) and streams the columns 64 at a
// time (y' transposed into sYt[q][.], swizzled, B into sB[c]; dynamic shared
// memory, two chunk buffers: the next chunk's records are copied straight to
// shared memory with cp.async while the current one is computed); thread t
// takes rows 4 (t / 16) + {0..3} and columns 4 (t % 16) + {0..3} of the chunk
// and forms t = A' + B + sum_q P_q y'_q in the order of plan_entry (so the
// same value bit for bit), then the entry and its reduction: per (q, thread)
// two 16-byte loads of P (shared by the 16 threads of the rows) and two of y'
// for 16 float64 FMAs. A row is reduced over the 16 threads of its half warp in
// a fixed order. 2 blocks per SM (120 registers; measured at workload 3: the
// residual 47 -> 40 ms and min_row 52 -> 41 ms against a single chunk buffer
// at 3 blocks per SM).
constexpr int kWdCols = 64;

int64_t wide_smem_bytes(int d) { return (int64_t)(d * (kRgRows + 2 * kWdCols) + kRgRows * 2 + 2 * kWdCols) * 8; }

template <int OP>
__global__ void __launch_bounds__(kRpThreads, 2) rowpass_wide_kernel(RowPassArgs R) {
    extern __shared__ __align__(16) double wsm[];
    const int d = R.d;
    double *sPt = wsm;                    // [d][64]
    double *sYt2 = sPt + d * kRgRows;     // [2][d][64]
    double *sA = sYt2 + 2 * d * kWdCols;  // [64]
    double *sB2 = sA + kRgRows;           // [2][64]
    double *sRed = sB2 + 2 * kWdCols;     // [64]
    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int64_t r0 = R.row_begin + (int64_t)blockIdx.x * kRgRows;
    if (tid < kRgRows) {
        const int64_t i = r0 + tid;
        double P[kMaxD];
        double A = -INFINITY;
        if (i < R.row_end) {
            load_row(R.pts, R.pot, i, d, R.o, R.prm->kappa, R.prm->c, &A, P);
        } else {
            for (int q = 0; q < d; ++q) P[q] = 0.0;
        }
        sA[tid] = A;
        for (int q = 0; q < d; ++q) sPt[q * kRgRows + tid] = P[q];
    }
    float mx[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int cnt[4] = {0, 0, 0, 0};
    double sum[4] = {0.0, 0.0, 0.0, 0.0};
    const int DS = d + 1;
    auto stage = [&](int64_t c0, int buf) {
        double *sYt = sYt2 + buf * d * kWdCols, *sB = sB2 + buf * kWdCols;
        for (int c = tid >> 5; c < kWdCols; c += kRpThreads / 32) {
            const int64_t j = c0 + c;
            for (int q = tid & 31; q < DS; q += 32) {
                double *dst = q < d ? &sYt[q * kWdCols + (c ^ ((q & 15) << 2))] : &sB[c];
                if (j < R.cols) {
                    const unsigned sa = (unsigned)__cvta_generic_to_shared(dst);
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(R.dcol + j * DS + q) : "memory");
                } else {
                    *dst = q == d ? -INFINITY : 0.0;
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    stage(0, 0);
    int buf = 0;
    for (int64_t c0 = 0; c0 < R.cols; c0 += kWdCols, buf ^= 1) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();  // chunk c0 is staged, and the other buffer is no longer read
        if (c0 + kWdCols < R.cols) stage(c0 + kWdCols, buf ^ 1);
        const double *sYt = sYt2 + buf * d * kWdCols, *sB = sB2 + buf * kWdCols;
        double acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = sA[4 * rg + r] + sB[4 * cg + c];
#pragma unroll 4
        for (int q = 0; q < d; ++q) {
            const double *pq = &sPt[q * kRgRows + 4 * rg];
            const double2 p0 = *reinterpret_cast<const double2 *>(pq);
            const double2 p1 = *reinterpret_cast<const double2 *>(pq + 2);
            const double *yq = &sYt[q * kWdCols + ((4 * cg) ^ ((q & 15) << 2))];
            const double2 y0 = *reinterpret_cast<const double2 *>(yq);
            const double2 y1 = *reinterpret_cast<const double2 *>(yq + 2);
            const double pr[4] = {p0.x, p0.y, p1.x, p1.y}, yc[4] = {y0.x, y0.y, y1.x, y1.y};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fma(pr[r], yc[c], acc[r][c]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float part = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float t = exp2_shifted(acc[r][c]);
                if (OP == OP_MAX) mx[r] = fmaxf(mx[r], t);
                if (OP == OP_COUNT) cnt[r] += (c0 + 4 * cg + c < R.cols && t >= R.thr) ? 1 : 0;
                if (OP == OP_SUM) part += t;
            }
            if (OP == OP_SUM) sum[r] += (double)part;
        }
    }
    // each row over the 16 threads of its half warp, in a fixed order
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        double v = OP == OP_SUM ? sum[r] : OP == OP_COUNT ? (double)cnt[r] : (double)mx[r];
        for (int off = 8; off > 0; off >>= 1) {
            const double o2 = __shfl_xor_sync(0xffffffffu, v, off);
            v = OP == OP_MAX ? fmax(v, o2) : v + o2;
        }
        if (cg == 0) {
            const int rr = 4 * rg + r;
            const int64_t i = r0 + rr;
            double res = 0.0;
            if (i < R.row_end) {
                const float wi = R.w[i];
                if (OP == OP_MAX) R.rowmax[i] = (float)v;
                if (OP == OP_COUNT) R.counts[i] = wi > 0.0f ? (int64_t)v : 0;
                if (OP == OP_SUM) res = fabs(v - (double)wi);
            }
            sRed[rr] = res;
        }
    }
    if (OP == OP_SUM) {
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int r = 0; r < kRgRows; ++r) t += sRed[r];
            R.part[blockIdx.x] = t;
        }
    }
}

// ------------------------------------------------------------ low-rank rows
// Two more row flavours (moscot PR #846, "Fix"), both a small matrix product:
//   MODE 0, low-rank coupling:  out[t, j] = sum_k Q[i,k] R[j,k] / g[k]
//   MODE 1, low-rank cost:      out[t, j] = exp((f_i + g_j - c (cost1[i].cost2[j] + bias)) / eps)
// with i = row_idx[t]. A block owns 128 columns and up to 512 rows of the row
// list: it stages its columns' factors once, then walks 64-row tiles; its 256
// threads are 8 row groups x 32 column groups and each owns 8 rows x 4 columns
// of a tile; both factor blocks sit K-major in shared memory (rows read as
// broadcasts, columns as one 16-byte load per thread and k). The coupling accumulates in float32
// (its factors are nonnegative: relative error <= r 2^-24); the cost
// accumulates its dot products in float64 and assembles the exponent like the
// point-cloud rows (exp2_shifted).
constexpr int kLrRows = 64, kLrCols = 128, kLrThreads = 256, kLrRowsPerBlock = 512;

template <typename T, int MODE>
__global__ void __launch_bounds__(kLrThreads) lowrank_rows_kernel(LrArgs L) {
    extern __shared__ __align__(16) uint8_t lr_smem[];
    T *sR = reinterpret_cast<T *>(lr_smem);    // [r][kLrRows]
    T *sC = sR + (size_t)L.r * kLrRows;         // [r][kLrCols]
    const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5;
    const int64_t j0 = (int64_t)blockIdx.x * kLrCols;
    // this block's columns, once
    for (int e = tid; e < L.r * kLrCols; e += kLrThreads) {
        const int cc = e / L.r, q = e % L.r;  // consecutive threads: consecutive k of one column
        const int64_t j = j0 + cc;
        sC[q * kLrCols + cc] = j < L.m ? (T)L.fb[j * L.r + q] : (T)0;
    }
    const int64_t tb = (int64_t)blockIdx.y * kLrRowsPerBlock;
    const int64_t te = min(tb + kLrRowsPerBlock, L.k);
    const int64_t jb = j0 + cg * 4;
    for (int64_t t0 = tb; t0 < te; t0 += kLrRows) {
        __syncthreads();  // the previous tile's row factors are no longer read
        // row factors (a row list entry outside [0, n) is reported and yields no row)
        for (int e = tid; e < L.r * kLrRows; e += kLrThreads) {
            const int rr = e / L.r, q = e % L.r;
            const int64_t t = t0 + rr;
            T v = (T)0;
            if (t < te) {
                const int64_t i = L.row_idx[t];
                if (i >= 0 && i < L.n) {
                    v = (T)L.fa[i * L.r + q];
                    if (MODE == 0) v = v / (T)L.g[q];
                } else if (q == 0) {
                    atomicExch(L.bad, 1);
                }
            }
            sR[q * kLrRows + rr] = v;
        }
        __syncthreads();
        T acc[8][4];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = (T)0;
        for (int q = 0; q < L.r; ++q) {
            T av[8], bv[4];
#pragma unroll
            for (int a = 0; a < 8; ++a) av[a] = sR[q * kLrRows + rg * 8 + a];
#pragma unroll
            for (int b = 0; b < 4; ++b) bv[b] = sC[q * kLrCols + cg * 4 + b];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fma(av[a], bv[b], acc[a][b]);
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int64_t t = t0 + rg * 8 + a;
            if (t >= te) break;
            const int64_t i = L.row_idx[t];
            if (i < 0 || i >= L.n) continue;
            float o[4];
            double Ai = 0.0;
            if (MODE == 1) {
                const float fv = L.f[i];
                Ai = fv == -INFINITY ? -1e15 : L.kappa * (double)fv;
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (MODE == 0) {
                    o[b] = (float)acc[a][b];
                } else {
                    const int64_t j = jb + b < L.m ? jb + b : L.m - 1;
                    const float gv = L.gp[j];
                    const double Bj = gv == -INFINITY ? -1e15 : L.kappa * (double)gv;
                    o[b] = exp2_shifted(fma(-L.kc, (double)acc[a][b] + L.bias, (Ai + kShift) + Bj));
                }
            }
            float *dst = L.out + t * L.m + jb;
            if (L.vec && jb + 4 <= L.m) {
                __stcs(reinterpret_cast<float4 *>(dst), make_float4(o[0], o[1], o[2], o[3]));
            } else {
                for (int b = 0; b < 4 && jb + b < L.m; ++b) __stcs(dst + b, o[b]);
            }
        }
    }
}

size_t lowrank_smem_bytes(int mode, int r) {
    return (size_t)r * (kLrRows + kLrCols) * (mode == 0 ? sizeof(float) : sizeof(double));
}

cudaError_t launch_lowrank_rows(int mode, const LrArgs &L, cudaStream_t s) {
    if (L.k <= 0 || L.m <= 0) return cudaSuccess;
    const size_t smem = lowrank_smem_bytes(mode, L.r);
    const void *fn = mode == 0 ? (const void *)lowrank_rows_kernel<float, 0>
                               : (const void *)lowrank_rows_kernel<double, 1>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t max_y = 65535;
    for (int64_t r0 = 0; r0 < L.k; r0 += max_y * kLrRowsPerBlock) {
        LrArgs A = L;
        A.row_idx = L.row_idx + r0;
        A.out = L.out + r0 * L.m;
        A.k = std::min<int64_t>(max_y * kLrRowsPerBlock, L.k - r0);
        dim3 grid((unsigned)((L.m + kLrCols - 1) / kLrCols),
                  (unsigned)((A.k + kLrRowsPerBlock - 1) / kLrRowsPerBlock));
        if (mode == 0) lowrank_rows_kernel<float, 0><<<grid, kLrThreads, smem, s>>>(A);
        else lowrank_rows_kernel<double, 1><<<grid, kLrThreads, smem, s>>>(A);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ----------------------------------------------------------- sparse plan
// The kept entries (T_ij >= thr, rows with mass) of kRpRows rows per block in
// compressed-row form. Thread t visits columns t, t + 256, ... in order; per
// 256-column chunk and row, a warp ballot and the warps' counts in shared
// memory give every kept entry its position, so each row's entries land in
// increasing column order from row_ptr[i]. The entries come from the same
// plan_entry() as the count pass that produced row_ptr; a row never writes
// past its own segment, and a row whose kept entries do not fill it exactly
// sets *bad (it cannot happen unless the two passes disagree).
constexpr int kCsrRows = 8;  // rows per block of the compressed-row write

template <int D>
__global__ void __launch_bounds__(kRpThreads) csr_write_kernel(CsrArgs C) {
    constexpr int WARPS = kRpThreads / 32;
    __shared__ double sA[kCsrRows], sP[kCsrRows][D > 0 ? D : kMaxD];
    __shared__ int sCnt[kCsrRows][WARPS];
    __shared__ long long sPos[kCsrRows], sEnd[kCsrRows];
    __shared__ int sLive[kCsrRows];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = C.row_begin + (int64_t)blockIdx.x * kCsrRows;
    const int d = D > 0 ? D : C.d;
    if (tid < kCsrRows) {
        const int64_t i = r0 + tid;
        const int live = i < C.row_end && C.w[i] > 0.0f;
        if (live) {
            load_row(C.pts, C.pot, i, d, C.o, C.prm->kappa, C.prm->c, &sA[tid], sP[tid]);
            sPos[tid] = C.row_ptr[i];
            sEnd[tid] = C.row_ptr[i + 1];
        } else {
            sA[tid] = -INFINITY;
            sPos[tid] = sEnd[tid] = 0;
        }
        sLive[tid] = live;
    }
    __syncthreads();
    const unsigned below = (1u << lane) - 1u;
    constexpr int DS = (D > 0 ? D : 1) + 1;
    for (int64_t j0 = 0; j0 < C.cols; j0 += kRpThreads) {
        const int64_t j = j0 + tid;
        const bool colok = j < C.cols;
        double cd[DS];
        const double *col = C.dcol + (colok ? j : 0) * (d + 1);
        if (D > 0) {
#pragma unroll
            for (int q = 0; q < DS; ++q) cd[q] = col[q];
        }
        float t[kCsrRows];
        unsigned bal[kCsrRows];
#pragma unroll
        for (int r = 0; r < kCsrRows; ++r) {
            t[r] = D > 0 ? plan_entry<D>(sA[r], sP[r], cd, d) : plan_entry<0>(sA[r], sP[r], col, d);
            const bool keep = colok && sLive[r] && t[r] >= C.thr;
            bal[r] = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) sCnt[r][warp] = __popc(bal[r]);
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kCsrRows; ++r) {
            if (!((bal[r] >> lane) & 1u)) continue;
            long long off = sPos[r] + __popc(bal[r] & below);
            for (int w = 0; w < warp; ++w) off += sCnt[r][w];
            if (off < sEnd[r]) {
                C.col_idx[off] = j;
                C.vals[off] = t[r];
            } else {
                atomicExch(C.bad, 1);
            }
        }
        __syncthreads();
        if (tid < kCsrRows) {
            int tot = 0;
            for (int w = 0; w < WARPS; ++w) tot += sCnt[tid][w];
            sPos[tid] += tot;
        }
        __syncthreads();
    }
    if (tid < kCsrRows && sLive[tid] && sPos[tid] != sEnd[tid]) atomicExch(C.bad, 1);
}

// Exclusive scan of the row counts into row_ptr, in three launches: tiles of
// kScanTile counts scanned in place (inclusive, at row_ptr[1..]) with the tile
// totals on the side, the totals scanned by one block, the tile offsets added.
constexpr int kScanThreads = 1024, kScanPer = 4, kScanTile = kScanThreads * kScanPer;

__device__ long long block_incl_scan(long long v, long long *s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        long long w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const long long u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const long long r = v + (warp > 0 ? s_warp[warp - 1] : 0);
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kScanThreads) scan_tiles_kernel(const int64_t *counts, int64_t n,
                                                                   int64_t *row_ptr, int64_t *sums) {
    __shared__ long long s_warp[32];
    const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPer;
    long long v[kScanPer], run = 0;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) {
        v[k] = base + k < n ? counts[base + k] : 0;
        run += v[k];
    }
    const long long excl = block_incl_scan(run, s_warp) - run;
    long long acc = excl;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) {
        acc += v[k];
        if (base + k < n) row_ptr[base + k + 1] = acc;
    }
    if (threadIdx.x == blockDim.x - 1) sums[blockIdx.x] = acc;
    if (blockIdx.x == 0 && threadIdx.x == 0) row_ptr[0] = 0;
}

__global__ void __launch_bounds__(kScanThreads) scan_sums_kernel(int64_t *sums, int64_t nb) {
    __shared__ long long s_warp[32];
    __shared__ long long s_tot;
    long long carry = 0;
    for (int64_t b0 = 0; b0 < nb; b0 += kScanThreads) {
        const int64_t b = b0 + threadIdx.x;
        const long long v = b < nb ? sums[b] : 0;
        const long long incl = block_incl_scan(v, s_warp);
        if (b < nb) sums[b] = carry + incl - v;  // exclusive: the offset of tile b
        if (threadIdx.x == kScanThreads - 1) s_tot = incl;
        __syncthreads();
        carry += s_tot;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kScanThreads) scan_add_kernel(int64_t n, int64_t *row_ptr,
                                                                 const int64_t *sums) {
    if (blockIdx.x == 0) return;  // tile 0 has offset 0
    const long long off = sums[blockIdx.x];
    const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPer;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k)
        if (base + k < n) row_ptr[base + k + 1] += off;
}

// ------------------------------------------------------------ reductions
// min over massful rows of rowmax (smallest index on ties), number of massless
// rows and (after the count pass) nnz. One block; fixed order per thread, then
// a fixed tree, so the result does not depend on timing.
constexpr int kRedThreads = 1024;

__global__ void __launch_bounds__(kRedThreads) min_row_reduce_kernel(const float *rowmax,
                                                                     const float *w, int64_t n,
                                                                     float *thr,
                                                                     int64_t *argmin,
                                                                     int64_t *n_massless) {
    __shared__ float sv[kRedThreads];
    __shared__ int64_t si[kRedThreads], sc[kRedThreads];
    const int tid = threadIdx.x;
    float best = INFINITY;
    int64_t bi = -1, nm = 0;
    for (int64_t i = tid; i < n; i += kRedThreads) {
        if (w[i] > 0.0f) {
            const float v = rowmax[i];
            if (v < best) {
                best = v;
                bi = i;
            }
        } else {
            ++nm;
        }
    }
    sv[tid] = best;
    si[tid] = bi;
    sc[tid] = nm;
    __syncthreads();
    for (int s = kRedThreads / 2; s > 0; s >>= 1) {
        if (tid < s) {
            const float v2 = sv[tid + s];
            const int64_t i2 = si[tid + s];
            if (i2 >= 0 && (si[tid] < 0 || v2 < sv[tid] || (v2 == sv[tid] && i2 < si[tid]))) {
                sv[tid] = v2;
                si[tid] = i2;
            }
            sc[tid] += sc[tid + s];
        }
        __syncthreads();
    }
    if (tid == 0) {
        *thr = sv[0];
        *argmin = si[0];
        *n_massless = sc[0];
    }
}

// out = sum of v[0..cnt) for int64 (exact) or double (fixed order).
template <typename T>
__global__ void __launch_bounds__(kRedThreads) sum_kernel(const T *v, int64_t cnt, T *out) {
    __shared__ T s[kRedThreads];
    const int tid = threadIdx.x;
    T acc = 0;
    for (int64_t i = tid; i < cnt; i += kRedThreads) acc += v[i];
    s[tid] = acc;
    __syncthreads();
    for (int st = kRedThreads / 2; st > 0; st >>= 1) {
        if (tid < st) s[tid] += s[tid + st];
        __syncthreads();
    }
    if (tid == 0) *out = s[0];
}


// ----------------------------------------------------------------- launchers
cudaError_t launch_dcol(const float *p, const float *pot, int64_t cnt, int d, const double *o,
                        const Params *prm, double *dcol, cudaStream_t s, const int64_t *perm) {
    if (cnt <= 0) return cudaSuccess;
    build_dcol_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, s>>>(p, pot, cnt, d, o, prm, perm, dcol);
    return cudaGetLastError();
}

int64_t chunk_count(int64_t cols) { return (cols + kRpChunkC - 1) / kRpChunkC; }

cudaError_t launch_chunk_summary(const double *dcol, int64_t cnt, int d, const Params *prm,
                                 double *csum, cudaStream_t s) {
    const int64_t warps = chunk_count(cnt);
    if (warps <= 0) return cudaSuccess;
    chunk_summary_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(dcol, cnt, d, prm, csum);
    return cudaGetLastError();
}

cudaError_t launch_perm_from_keys(const unsigned long long *keys, int64_t cnt, int64_t off,
                                  int64_t *perm, cudaStream_t s) {
    if (cnt <= 0) return cudaSuccess;
    perm_from_keys_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, s>>>(keys, cnt, off, perm);
    return cudaGetLastError();
}

cudaError_t launch_materialize(const MatArgs &M, cudaStream_t s) {
    const int64_t col_blocks = (M.m + kMtThreads * 4 - 1) / (kMtThreads * 4);
    // at most 65535 row ranges per launch: split long row lists
    const int64_t max_rows = (int64_t)65535 * (M.d > 3 ? kMwRows : kMtRowsPerBlock);
    for (int64_t r = 0; r < M.k; r += max_rows) {
        MatArgs A = M;
        A.row_idx = M.row_idx + r;
        A.out = M.out + r * M.m;
        A.k = min(max_rows, M.k - r);
        dim3 grid((unsigned)col_blocks, (unsigned)((A.k + kMtRowsPerBlock - 1) / kMtRowsPerBlock));
        switch (M.d) {
            case 1: materialize_kernel<1><<<grid, kMtThreads, 0, s>>>(A); break;
            case 2: materialize_kernel<2><<<grid, kMtThreads, 0, s>>>(A); break;
            case 3: materialize_kernel<3><<<grid, kMtThreads, 0, s>>>(A); break;
            default: {
                // d > 3: 64 list entries x 16 chunks of 64 columns per block (up to 66 KB of
                // shared memory at d = 64: the opt-in is per device, so every launch sets it)
                if (cudaFuncSetAttribute(materialize_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)matwide_smem_bytes(kMaxD)) != cudaSuccess)
                    return cudaGetLastError();
                const int64_t wcols = (M.m + (int64_t)kMwChunks * kMwCols - 1) / ((int64_t)kMwChunks * kMwCols);
                dim3 wgrid((unsigned)wcols, (unsigned)((A.k + kMwRows - 1) / kMwRows));
                materialize_wide_kernel<<<wgrid, 256, (size_t)matwide_smem_bytes(M.d), s>>>(A);
                break;
            }
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int OP>
static void rowpass_dispatch(const RowPassArgs &R, int64_t rows, cudaStream_t s) {
    const unsigned grid = (unsigned)rowpass_blocks(rows, R.d);
    switch (R.d) {
        case 1: rowpass_kernel<1, OP><<<grid, kRpThreads, 0, s>>>(R); break;
        case 2: rowpass_kernel<2, OP><<<grid, kRpThreads, 0, s>>>(R); break;
        case 3: rowpass_kernel<3, OP><<<grid, kRpThreads, 0, s>>>(R); break;
        default: {
            // up to 50 KB of shared memory at d = 64: the opt-in is per device, so every
            // launch sets it (a host-side call)
            if (cudaFuncSetAttribute(rowpass_wide_kernel<OP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)wide_smem_bytes(kMaxD)) != cudaSuccess)
                return;  // the caller's cudaGetLastError reports it
            rowpass_wide_kernel<OP><<<grid, kRpThreads, (size_t)wide_smem_bytes(R.d), s>>>(R);
            break;
        }
    }
}

// op: 0 max, 1 count, 2 sum; rows [row_begin, row_end)
cudaError_t launch_rowpass(int op, const RowPassArgs &R, cudaStream_t s) {
    const int64_t rows = R.row_end - R.row_begin;
    if (rows <= 0) return cudaSuccess;
    if (op == OP_MAX) rowpass_dispatch<OP_MAX>(R, rows, s);
    else if (op == OP_COUNT) rowpass_dispatch<OP_COUNT>(R, rows, s);
    else rowpass_dispatch<OP_SUM>(R, rows, s);
    return cudaGetLastError();
}

int64_t rowpass_rows_per_block(int d) { return d <= 3 ? kRpRows : kRgRows; }

int64_t rowpass_blocks(int64_t rows, int d) {
    const int64_t per = rowpass_rows_per_block(d);
    return (rows + per - 1) / per;
}

cudaError_t launch_min_row_reduce(const float *rowmax, const float *w, int64_t n, float *thr,
                                  int64_t *argmin, int64_t *n_massless, cudaStream_t s) {
    min_row_reduce_kernel<<<1, kRedThreads, 0, s>>>(rowmax, w, n, thr, argmin, n_massless);
    return cudaGetLastError();
}

cudaError_t launch_sum_i64(const int64_t *v, int64_t cnt, int64_t *out, cudaStream_t s) {
    sum_kernel<int64_t><<<1, kRedThreads, 0, s>>>(v, cnt, out);
    return cudaGetLastError();
}

cudaError_t launch_csr_write(const CsrArgs &C, cudaStream_t s) {
    const int64_t rows = C.row_end - C.row_begin;
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kCsrRows - 1) / kCsrRows);
    switch (C.d) {
        case 1: csr_write_kernel<1><<<grid, kRpThreads, 0, s>>>(C); break;
        case 2: csr_write_kernel<2><<<grid, kRpThreads, 0, s>>>(C); break;
        case 3: csr_write_kernel<3><<<grid, kRpThreads, 0, s>>>(C); break;
        default: csr_write_kernel<0><<<grid, kRpThreads, 0, s>>>(C); break;
    }
    return cudaGetLastError();
}

int64_t scan_tmp_count(int64_t n) { return (n + kScanTile - 1) / kScanTile + 1; }

cudaError_t launch_row_ptr_scan(const int64_t *counts, int64_t n, int64_t *row_ptr, int64_t *tmp,
                                cudaStream_t s) {
    const int64_t nb = std::max<int64_t>((n + kScanTile - 1) / kScanTile, 1);
    scan_tiles_kernel<<<(unsigned)nb, kScanThreads, 0, s>>>(counts, n, row_ptr, tmp);
    scan_sums_kernel<<<1, kScanThreads, 0, s>>>(tmp, nb);
    scan_add_kernel<<<(unsigned)nb, kScanThreads, 0, s>>>(n, row_ptr, tmp);
    return cudaGetLastError();
}

cudaError_t launch_sum_f64(const double *v, int64_t cnt, double *out, cudaStream_t s) {
    sum_kernel<double><<<1, kRedThreads, 0, s>>>(v, cnt, out);
    return cudaGetLastError();
}

}  // namespace ot
