// lowd.cuh -- the d <= 3 work item shared by the per-half-step kernel and the
// device-resident loop kernel. See halfstep.cu for the design of the update.
#pragma once
#include "common.cuh"

namespace ot {

// Column-table load: CG = true bypasses L1 (the table may have been rewritten
// earlier in the same kernel by other blocks, as in the device-resident loop).
template <bool CG>
__device__ __forceinline__ float4 ld4(const float4 *p) {
    return CG ? __ldcg(p) : *p;
}

// One step of 8 columns (four column pairs v[0..7] of the column table) for
// the R rows of this thread: the exponents t = G_j + x'.Y_j as packed f32x2
// FMAs, the lazily refreshed running maximum (warp vote), the exponentials and
// the two accumulator pairs per row. SPEC: the exponentials are taken against
// the current maximum before the vote, and again in the rare step that
// refreshes, so the ex2 pipe does not wait for the vote.
template <int D, int R, bool SPEC>
__device__ __forceinline__ void lowd_step8(const float4 (&v)[8], const float2 (&xd)[R][3],
                                           float (&m)[R], float2 (&nm)[R], float2 (&acc)[R],
                                           float2 (&acc2)[R], float (&tot)[R]) {
    constexpr int kHsRows = R;
#pragma unroll
    for (int k = 0; k < kHsRows; ++k) {
        float2 t[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float4 lo = v[2 * p], hi = v[2 * p + 1];
            float2 tt = __ffma2_rn(make_float2(lo.x, lo.y), xd[k][0],
                                   make_float2(hi.z, hi.w));
            if (D >= 2) tt = __ffma2_rn(make_float2(lo.z, lo.w), xd[k][1], tt);
            if (D >= 3) tt = __ffma2_rn(make_float2(hi.x, hi.y), xd[k][2], tt);
            t[p] = tt;
        }
        const float cm = fmax3(fmax3(t[0].x, t[0].y, t[1].x), fmax3(t[1].y, t[2].x, t[2].y),
                               fmaxf(t[3].x, t[3].y));
        float2 e[4];
        if (SPEC) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 u = __fadd2_rn(t[p], nm[k]);
                e[p] = make_float2(ex2_approx(u.x), ex2_approx(u.y));
            }
        }
        if (__any_sync(0xffffffffu, cm > m[k] + kLazyMax)) {  // rare: refresh (warp vote)
            const float mx = fmaxf(cm, m[k]);
            const float sc = ex2_approx(m[k] - mx);
            acc[k] = __fmul2_rn(acc[k], make_float2(sc, sc));
            acc2[k] = __fmul2_rn(acc2[k], make_float2(sc, sc));
            tot[k] *= sc;
            m[k] = mx;
            nm[k] = make_float2(-mx, -mx);
            if (SPEC) {
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 u = __fadd2_rn(t[p], nm[k]);
                    e[p] = make_float2(ex2_approx(u.x), ex2_approx(u.y));
                }
            }
        }
        if (!SPEC) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 u = __fadd2_rn(t[p], nm[k]);
                e[p] = make_float2(ex2_approx(u.x), ex2_approx(u.y));
            }
        }
        acc[k] = __fadd2_rn(acc[k], e[0]);
        acc2[k] = __fadd2_rn(acc2[k], e[1]);
        acc[k] = __fadd2_rn(acc[k], e[2]);
        acc2[k] = __fadd2_rn(acc2[k], e[3]);
    }
}

// One work item (row tile, column split) of the d <= 3 half-step: streams the
// split's columns through shared memory and writes (running max, sum) per row
// to A.part. Rows: thread t owns rows t + 128 k, k < R.
// SPEC (see lowd_step8) needs a few more registers (measured: +2.5% of the
// MUFU rate at n = 1e5..3e5 per launch, +2..5% in the loop kernel at n =
// 8000..16000 when it has the registers to avoid spills).
template <int D, int R, bool CG, bool SPEC>
__device__ __forceinline__ void lowd_item(const HalfStep &A, int tile, int split,
                                          float4 (*sm)[kHsChunk]) {
    constexpr int kHsRows = R;
    constexpr int kHsTile = kHsThreads * R;
    const int tid = threadIdx.x;
    const float4 *rt4 = reinterpret_cast<const float4 *>(A.rowtab);

    float2 xd[kHsRows][3];
    float m[kHsRows], tot[kHsRows];
    float2 nm[kHsRows], acc[kHsRows], acc2[kHsRows];
#pragma unroll
    for (int k = 0; k < kHsRows; ++k) {
        const int64_t row = (int64_t)tile * kHsTile + k * kHsThreads + tid;
        const float4 p = row < A.rows ? rt4[row] : make_float4(0.f, 0.f, 0.f, 0.f);
        xd[k][0] = make_float2(p.x, p.x);
        xd[k][1] = make_float2(p.y, p.y);
        xd[k][2] = make_float2(p.z, p.z);
        m[k] = kNegBig;
        nm[k] = make_float2(-kNegBig, -kNegBig);
        acc[k] = make_float2(0.f, 0.f);
        acc2[k] = make_float2(0.f, 0.f);
        tot[k] = 0.f;
    }

    const int64_t c0 = (int64_t)split * A.cols_per_split;
    const int64_t span = min(c0 + A.cols_per_split, A.cols_pad) - c0;  // multiple of 8
    const int nch = (int)((span + kHsChunk - 1) / kHsChunk);
    const float4 *src = A.coltab + c0;
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 p0 = tid < span ? ld4<CG>(src + tid) : zero4;
    float4 p1 = tid + kHsThreads < span ? ld4<CG>(src + tid + kHsThreads) : zero4;

#pragma unroll 1
    for (int ch = 0; ch < nch; ++ch) {
        float4 *buf = sm[ch & 1];
        buf[tid] = p0;
        buf[tid + kHsThreads] = p1;
        __syncthreads();
        const int64_t nb = (int64_t)(ch + 1) * kHsChunk;
        if (ch + 1 < nch) {
            p0 = nb + tid < span ? ld4<CG>(src + nb + tid) : zero4;
            p1 = nb + kHsThreads + tid < span ? ld4<CG>(src + nb + kHsThreads + tid) : zero4;
        }
        const int ncols = (int)min((int64_t)kHsChunk, span - (int64_t)ch * kHsChunk);
#pragma unroll 1
        for (int q = 0; q < ncols; q += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = buf[q + u];
            lowd_step8<D, R, SPEC>(v, xd, m, nm, acc, acc2, tot);
        }
#pragma unroll
        for (int k = 0; k < kHsRows; ++k) {
            tot[k] += (acc[k].x + acc[k].y) + (acc2[k].x + acc2[k].y);
            acc[k] = make_float2(0.f, 0.f);
            acc2[k] = make_float2(0.f, 0.f);
        }
    }

    const int64_t stride = (int64_t)A.tiles * kHsTile;
#pragma unroll
    for (int k = 0; k < kHsRows; ++k) {
        const int64_t row = (int64_t)tile * kHsTile + k * kHsThreads + tid;
        if (row < A.rows) A.part[split * stride + row] = make_float2(m[k], tot[k]);
    }
}


// ------------------------------------------------------ block-sparse item
// Column-table entry that adds nothing: chunk slot u holds the even (u even)
// or the odd half of a column pair; the odd half carries G = -inf.
__device__ __forceinline__ float4 dead4(int u) {
    return (u & 1) ? make_float4(0.f, 0.f, -INFINITY, -INFINITY) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// One work item of the block-sparse half-step ("FlashSinkhorn 2: Block-Sparse
// Entropic Optimal Transport", section 3.2): the B = 128 R rows of row block
// `tile` reduce over list positions [k0, k1) of the block's admitted column
// tiles (A.sp_idx[A.sp_ptr[tile] ..], B columns each), or over every column
// tile when the block has none. A chunk of 256 columns gathers 256 / B tiles.
// Writes (running max, sum) per row to A.part, as lowd_item does.
template <int D, int R>
__device__ __forceinline__ void sparse_item(const HalfStep &A, int tile, int split,
                                            float4 (*sm)[kHsChunk]) {
    constexpr int kB = kHsThreads * R;
    constexpr int kTpc = kHsChunk / kB;  // column tiles per chunk
    const int tid = threadIdx.x;
    const float4 *rt4 = reinterpret_cast<const float4 *>(A.rowtab);

    float2 xd[R][3];
    float m[R], tot[R];
    float2 nm[R], acc[R], acc2[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const int64_t row = (int64_t)tile * kB + k * kHsThreads + tid;
        const float4 p = row < A.rows ? rt4[row] : make_float4(0.f, 0.f, 0.f, 0.f);
        xd[k][0] = make_float2(p.x, p.x);
        xd[k][1] = make_float2(p.y, p.y);
        xd[k][2] = make_float2(p.z, p.z);
        m[k] = kNegBig;
        nm[k] = make_float2(-kNegBig, -kNegBig);
        acc[k] = make_float2(0.f, 0.f);
        acc2[k] = make_float2(0.f, 0.f);
        tot[k] = 0.f;
    }

    const int64_t lp0 = A.sp_ptr ? A.sp_ptr[tile] : 0;
    const int64_t cnt_p = A.sp_ptr ? A.sp_ptr[tile + 1] - lp0 : 0;  // no list: every tile
    const int64_t cnt = cnt_p > 0 ? cnt_p : (int64_t)A.sp_coltiles;
    const int64_t k0 = cnt * split / A.splits, k1 = cnt * (split + 1) / A.splits;
    const int nch = (int)((k1 - k0 + kTpc - 1) / kTpc);
    auto fetch = [&](int ch, int u) -> float4 {
        const int64_t k = k0 + (int64_t)ch * kTpc + u / kB;
        if (k >= k1) return dead4(u);
        const int64_t id = cnt_p > 0 ? (int64_t)__ldg(A.sp_idx + lp0 + k) : k;
        const int64_t c = id * kB + (u % kB);
        return c < A.cols_pad ? A.coltab[c] : dead4(u);
    };
    float4 p0 = make_float4(0.f, 0.f, 0.f, 0.f), p1 = p0;
    if (nch > 0) {
        p0 = fetch(0, tid);
        p1 = fetch(0, tid + kHsThreads);
    }
#pragma unroll 1
    for (int ch = 0; ch < nch; ++ch) {
        float4 *buf = sm[ch & 1];
        buf[tid] = p0;
        buf[tid + kHsThreads] = p1;
        __syncthreads();
        if (ch + 1 < nch) {
            p0 = fetch(ch + 1, tid);
            p1 = fetch(ch + 1, tid + kHsThreads);
        }
        const int ncols = (int)min((int64_t)kTpc, k1 - k0 - (int64_t)ch * kTpc) * kB;
#pragma unroll 1
        for (int q = 0; q < ncols; q += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = buf[q + u];
            lowd_step8<D, R, true>(v, xd, m, nm, acc, acc2, tot);
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            tot[k] += (acc[k].x + acc[k].y) + (acc2[k].x + acc2[k].y);
            acc[k] = make_float2(0.f, 0.f);
            acc2[k] = make_float2(0.f, 0.f);
        }
    }

    const int64_t stride = (int64_t)A.tiles * kB;
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const int64_t row = (int64_t)tile * kB + k * kHsThreads + tid;
        if (row < A.rows) A.part[split * stride + row] = make_float2(m[k], tot[k]);
    }
}

}  // namespace ot
