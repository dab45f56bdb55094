// halfstep_tc.cu -- fused log-domain Sinkhorn half-step for 16 <= d <= 64 with the
// x . y contraction on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// The update is the streaming log-sum-exp of "FlashSinkhorn 2: Block-Sparse
// Entropic Optimal Transport", section 2.1 (tiled reductions, tensor-core
// products, O((n+m)d) memory). In base-2 units the exponent of pair (i, j) is
//     t_ij = G_j + x'_i . Y_j,   Y_j = 2 c kappa y'_j,   G_j = kappa (g_j - c |y'_j|^2),
// and the whole of t_ij comes out of ONE bf16 tensor-core contraction with
// fp32 accumulation: with the two-term splits x' = x1 + x2, Y = Y1 + Y2 and
// the three-term split G = G1 + G2 + G3 (each term a bf16),
//     row operand    [ x1 | x1 | x2 | 1 1 1 | 0 ... ]
//     column operand [ Y1 | Y2 | Y1 | G1 G2 G3 | 0 ... ]
// (K = 3d + 3, padded to a multiple of 16). The dropped x2.Y2 term and the bf16
// roundings leave a relative cost error near 2^-16 (single-pass tf32 was
// measured at 1.2e-4 of max C on the potentials -- over the bar -- this split at
// 1.8e-6). The row constant -c kappa |x'_i|^2 is added once per row, in
// float64, by the shared tile finalizer.
//
// Block: 18 warps. Warp 16's elected lane issues the TMA loads of the row tile
// (once per work item) and of 128-column chunks of the column operand into a
// 3-stage (2 for K > 192) shared-memory ring, 128B-swizzled K-major; warp 17's
// issues tcgen05.mma into one of four TMEM accumulators (128 lanes x 128 fp32
// columns each). Warps 0-15 are the epilogue, four per accumulator: warp w
// drains buffer w/4 (TMEM lanes 32*(w%4)..+31, its rows; all 128 columns of
// chunks w/4, w/4 + 4, ... of each work item) with the lazily-rescaled max /
// ex2 / sum per row, so the summation order depends on the item alone;
// the four buffers' states of a row merge in shared memory at the end of a work
// item. Each SM sub-partition holds one warp per buffer, a chunk apart in time,
// so one warp's waits and loads overlap another's exponentials. Work items are
// claimed dynamically by the producer (its first one is its block index, the
// next ones come from the side's atomic counter) and handed to the MMA warp and
// the epilogue through a four-slot ring in shared memory guarded by mbarriers
// (a static stride left SMs idle 16 % of a launch: per-block times spread from
// 672 to 874 us at 40000 x 50000, d = 50). Every wait on
// an mbarrier is bounded; on timeout the block records State::wait_timeout,
// drains what it issued (again bounded), frees its TMEM and returns. No TMA
// load uses cluster multicast.
#include <cuda.h>

#include "finish.cuh"
#include "runtime.h"

namespace ot {
namespace tc {

constexpr int M = 128;               // rows per tile (MMA M)
constexpr int N = 128;               // columns per chunk (MMA N)
constexpr int EPI_WARPS = 16;         // 4 per SM sub-partition
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int THREADS = (EPI_WARPS + 2) * 32;  // + TMA warp + MMA warp
constexpr int SLAB = 64;             // bf16 per 128-byte swizzle row
constexpr int SLAB_BYTES = M * 128;  // one slab of a 128-row operand tile (16 KB)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for the phase with parity `parity` to complete. Returns false
// (and raises *abort) after `limit` polls (2^22 in production) or when another
// role aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          uint32_t limit) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if ((it & 255u) == 255u && *abort) return false;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// K-major, 128-byte-swizzled operand: 8-row atoms of 128 B, atoms 1024 B apart
// (SBO), LBO unused (1), descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t smem_desc(const void *p) {
    const uint64_t addr = smem_u32(p);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: bf16 A and B, f32 D, both K-major, M x N.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                           ((uint32_t)(M >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");  // it reads shared memory: keep it after the barrier waits
}

// arrives once on `bar` when every MMA issued so far by this thread completes
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }


// Warp-wide wait: lane 0 polls, the other lanes wait converged in the shuffle
// (512 threads polling would compete with TMA and MMA for shared memory).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort,
                                               uint32_t limit) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, limit) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait that ignores the abort flag: used only to drain work this block
// already issued before it frees its resources.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, uint32_t limit) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return;
    }
}

// tcgen05.wait::ld that also marks the loaded registers as written here, so the
// compiler cannot read them before the wait
__device__ __forceinline__ void tmem_wait_ld(float (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
                   "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]),
                   "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]),
                   "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]), "+f"(v[24]),
                   "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]), "+f"(v[30]),
                   "+f"(v[31])
                 :
                 : "memory");
}

constexpr int NBUF = 4;  // TMEM accumulators (4 x 128 fp32 columns = all 512)
constexpr int RING = 4;  // work items published by the producer ahead of the MMA warp and the epilogue
constexpr int TMA_WARP = EPI_WARPS, MMA_WARP = EPI_WARPS + 1;
static_assert(EPI_WARPS == 4 * NBUF, "one group of four epilogue warps per accumulator buffer");

// Shared-memory plan (dynamic; base rounded up to 1024 B for the 128B swizzle).
template <int KS>
struct Smem {
    static constexpr int STAGES = KS <= 3 ? 3 : 2;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = KS * SLAB_BYTES;
    static constexpr int BAR_OFF = B_OFF + STAGES * KS * SLAB_BYTES;
    // full[S], empty[S], tfull[NBUF], tempty[NBUF], afull, aempty, drain, ifull[RING], iempty[RING]
    static constexpr int NBAR = 2 * STAGES + 2 * NBUF + 3 + 2 * RING;
    // tmem addr, abort, flag, decide, 16 doubles, RING item slots, the epilogue's item
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int ITEMS_OFF = MISC_OFF + 144;
    static constexpr int MERGE_OFF = MISC_OFF + 256;      // float2 [EPI_WARPS/4][M]
    static constexpr int BYTES = MERGE_OFF + (EPI_WARPS / 4) * M * 8;
    // at least 116 KB, so that one block holds an SM (it takes all 512 TMEM columns)
    static constexpr int ALLOC = (BYTES + 1024) > 116 * 1024 ? BYTES + 1024 : 116 * 1024;
};

template <int KS>
__global__ void __launch_bounds__(THREADS, 1)
hs_tc_kernel(HalfStep A, const __grid_constant__ CUtensorMap tmA,
             const __grid_constant__ CUtensorMap tmB, int ksteps) {
    using L = Smem<KS>;
    constexpr int STAGES = L::STAGES;
    extern __shared__ uint8_t smem_raw[];
    // the other side's work-item counter (as in the CUDA-core half-steps)
    if (blockIdx.x == 0 && threadIdx.x == 0) A.st->work[A.side ^ 1] = 0u;
    if (ld_volatile(&A.st->stop)) return;
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = sm + L::A_OFF;
    uint8_t *sB = sm + L::B_OFF;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *afull = tempty + NBUF;
    uint64_t *aempty = afull + 1;
    uint64_t *drain = aempty + 1;
    uint64_t *ifull = drain + 1;
    uint64_t *iempty = ifull + RING;
    volatile long long *s_items = reinterpret_cast<volatile long long *>(sm + L::ITEMS_OFF);
    volatile long long *s_item_epi = s_items + RING;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::MISC_OFF);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 4);
    int *s_flag = reinterpret_cast<int *>(sm + L::MISC_OFF + 8);
    volatile int *s_decide = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 12);
    double *s_red = reinterpret_cast<double *>(sm + L::MISC_OFF + 16);
    float2 *s_merge = reinterpret_cast<float2 *>(sm + L::MERGE_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);  // the four warps (one per lane quarter) that drain buffer b
        }
        mbar_init(afull, 1);
        mbar_init(aempty, 1);
        mbar_init(drain, 1);
        for (int q = 0; q < RING; ++q) {
            mbar_init(&ifull[q], 1);   // the producer, after writing the slot
            mbar_init(&iempty[q], 2);  // the MMA lane and the epilogue, after reading it
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {  // all 512 TMEM columns: NBUF accumulators of N fp32 columns x 128 lanes
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(s_tmem)),
                     "r"(NBUF * N));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int64_t n_items = (int64_t)A.tiles * A.splits;
    const uint32_t lim = A.wait_polls;

    if (warp == TMA_WARP) {
        // -------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t g = 0, item_no = 0, issued[STAGES] = {};
            bool ok = true, a_out = false;
            int64_t item = blockIdx.x;
            for (uint32_t iq = 0; ok; ++iq, ++item_no) {
                // publish the item (or the end) to the MMA warp and the epilogue
                const int slot = (int)(iq % RING);
                if (iq >= (uint32_t)RING && !(ok = mbar_wait(&iempty[slot], ((iq / RING) - 1) & 1, s_abort, lim)))
                    break;
                s_items[slot] = item < n_items ? item : -1;
                mbar_arrive(&ifull[slot]);
                if (item >= n_items) break;
                // claim the next item now; its value is needed only after this item's loads
                const int64_t next = (int64_t)gridDim.x + (int64_t)atomicAdd(&A.st->work[A.side], 1u);
                const int tile = (int)(item / A.splits), split = (int)(item % A.splits);
                const int64_t c0 = (int64_t)split * A.cols_per_split;
                const int nch = (int)((min(c0 + A.cols_per_split, A.cols_pad) - c0) / N);
                // the row tile is overwritten only after every MMA of the previous item
                if (item_no > 0 && !(ok = mbar_wait(aempty, (item_no - 1) & 1, s_abort, lim))) break;
                mbar_expect_tx(afull, KS * SLAB_BYTES);
                for (int s = 0; s < KS; ++s)
                    tma_load_2d(sA + s * SLAB_BYTES, &tmA, afull, s * SLAB, (int)(tile * M + A.row_off));
                a_out = true;
                for (int ch = 0; ch < nch && ok; ++ch, ++g) {
                    const int st = g % STAGES;
                    if (g >= (uint32_t)STAGES && !(ok = mbar_wait(&empty[st], ((g / STAGES) - 1) & 1, s_abort, lim)))
                        break;
                    // failure tests only: block 0 leaves its first chunk unloaded, so the
                    // MMA warp's wait on it gives up
                    if (g == 0 && A.withhold && blockIdx.x == 0) continue;
                    mbar_expect_tx(&full[st], KS * SLAB_BYTES);
                    uint8_t *dst = sB + st * KS * SLAB_BYTES;
                    for (int s = 0; s < KS; ++s)
                        tma_load_2d(dst + s * SLAB_BYTES, &tmB, &full[st], s * SLAB, (int)(c0 + (int64_t)ch * N));
                    ++issued[st];
                }
                item = next;
            }
            if (!ok) {  // wait (bounded) for the loads this block put in flight
                if (a_out) mbar_drain(afull, (item_no & 1) ^ 0, lim);
                for (int st = 0; st < STAGES; ++st)
                    if (issued[st]) mbar_drain(&full[st], (issued[st] - 1) & 1, lim);
                atomicExch(&A.st->wait_timeout, 1);
            }
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------ MMA issue
        if (lane == 0) {
            uint32_t g = 0, item_no = 0, ub[NBUF] = {};  // ub: uses of each accumulator
            bool ok = true, issued_any = false;
            for (uint32_t iq = 0; ok; ++iq, ++item_no) {
                const int slot = (int)(iq % RING);
                if (!(ok = mbar_wait(&ifull[slot], (iq / RING) & 1, s_abort, lim))) break;
                const int64_t item = s_items[slot];
                mbar_arrive(&iempty[slot]);
                if (item < 0) break;
                const int split = (int)(item % A.splits);
                const int64_t c0 = (int64_t)split * A.cols_per_split;
                const int nch = (int)((min(c0 + A.cols_per_split, A.cols_pad) - c0) / N);
                if (!(ok = mbar_wait(afull, item_no & 1, s_abort, lim))) break;
                for (int ch = 0; ch < nch; ++ch, ++g) {
                    // accumulator by the chunk's index in its item, so that which epilogue
                    // warps sum which columns does not depend on the schedule
                    const int st = g % STAGES, b = ch % NBUF;
                    if (!(ok = mbar_wait(&full[st], (g / STAGES) & 1, s_abort, lim))) break;
                    if (ub[b] > 0 && !(ok = mbar_wait(&tempty[b], (ub[b] - 1) & 1, s_abort, lim))) break;
                    ++ub[b];
                    tc_fence_after();
                    const uint8_t *bst = sB + st * KS * SLAB_BYTES;
                    // fully unrolled over the template bound: with a loop over the runtime
                    // count the issue of one tcgen05.mma took ~120 cycles (half the
                    // tensor rate of a 128 x 128 x 16 MMA); unrolled it keeps up
#pragma unroll
                    for (int k = 0; k < 4 * KS; ++k) {
                        if (k >= ksteps) break;
                        const int slab = k >> 2;
                        const uint64_t adv = (uint64_t)((k & 3) * 2);  // 32 bytes per K step of 16
                        mma_bf16(tmem + (uint32_t)(b * N), smem_desc(sA + slab * SLAB_BYTES) + adv,
                                 smem_desc(bst + slab * SLAB_BYTES) + adv, k > 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit(&empty[st]);
                    mma_commit(&tfull[b]);
                }
                if (ok) mma_commit(aempty);
            }
            if (!ok) {
                if (issued_any) {  // wait (bounded) until the issued MMAs are done
                    mma_commit(drain);
                    mbar_drain(drain, 0, lim);
                }
                atomicExch(&A.st->wait_timeout, 1);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        // Warp w drains accumulator buffer h = w / 4 for TMEM lanes 32 (w % 4)..+31:
        // the chunks ch = h, h + 4, ... of every work item (the MMA warp puts chunk
        // ch in buffer ch % 4), all 128 columns, as four 32-column loads with the
        // next one in flight. Each SM sub-partition thus holds one warp of each of the
        // four buffers, a chunk apart in time, so one warp's waits and loads
        // overlap another's exponentials.
        const int q = warp & 3, h = warp >> 2;  // TMEM lane quarter, accumulator buffer
        const int r = q * 32 + lane;  // row of the tile owned by this thread
        const int etid = threadIdx.x;  // 0 .. EPI_THREADS-1
        const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * N);
        uint32_t uses = 0;  // uses of buffer h so far
        for (uint32_t iq = 0;; ++iq) {
            // thread 0 takes the next item from the producer and hands it to the others
            if (etid == 0) {
                const int slot = (int)(iq % RING);
                long long it = -1;
                if (mbar_wait(&ifull[slot], (iq / RING) & 1, s_abort, lim)) {
                    it = s_items[slot];
                    mbar_arrive(&iempty[slot]);
                }
                *s_item_epi = it;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
            const int64_t item = *s_item_epi;
            if (item < 0) break;
            const int tile = (int)(item / A.splits), split = (int)(item % A.splits);
            const int64_t c0 = (int64_t)split * A.cols_per_split;
            const int nch = (int)((min(c0 + A.cols_per_split, A.cols_pad) - c0) / N);
            float m = kNegBig, tot = 0.0f;
            float2 nm = make_float2(-kNegBig, -kNegBig);
            float2 acc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
            float va[32], vb[32];
            bool ok = true;
            for (int ch = h; ch < nch && ok; ch += NBUF) {
                ok = mbar_wait_warp(&tfull[h], uses & 1, s_abort, lim);
                if (!ok) break;
                tc_fence_after();
                tmem_ld32(tlane, va);
                tmem_wait_ld(va);
#pragma unroll 1
                for (int sc = 0; sc < N / 32; ++sc) {
                    const bool more = sc + 1 < N / 32;
                    if (more) tmem_ld32(tlane + (uint32_t)((sc + 1) * 32), vb);
                    // running maximum, refreshed lazily (terms stay <= 2^8)
                    float p[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        p[j] = fmax3(fmax3(va[8 * j], va[8 * j + 1], va[8 * j + 2]),
                                     fmax3(va[8 * j + 3], va[8 * j + 4], va[8 * j + 5]),
                                     fmaxf(va[8 * j + 6], va[8 * j + 7]));
                    const float cm = fmax3(p[0], p[1], fmaxf(p[2], p[3]));
                    if (__any_sync(0xffffffffu, cm > m + kLazyMax)) {
                        const float mx = fmaxf(cm, m);
                        const float sc2 = ex2_approx(m - mx);
#pragma unroll
                        for (int u = 0; u < 4; ++u) acc[u] = __fmul2_rn(acc[u], make_float2(sc2, sc2));
                        tot *= sc2;
                        m = mx;
                        nm = make_float2(-mx, -mx);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float2 u0 = __fadd2_rn(make_float2(va[2 * j], va[2 * j + 1]), nm);
                        acc[j & 3] = __fadd2_rn(acc[j & 3], make_float2(ex2_approx(u0.x), ex2_approx(u0.y)));
                    }
                    float cs = 0.0f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        cs += acc[u].x + acc[u].y;
                        acc[u] = make_float2(0.f, 0.f);
                    }
                    tot += cs;
                    if (more) {
                        tmem_wait_ld(vb);
#pragma unroll
                        for (int i = 0; i < 32; ++i) va[i] = vb[i];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[h]);
                ++uses;
            }
            // merge the four buffers' partial states of each row, then the column splits
            s_merge[h * M + r] = make_float2(m, tot);
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
            // one thread samples the abort flag, so every epilogue thread takes
            // the same path through the named barriers that follow
            if (etid == 0) *s_decide = *s_abort;
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
            const bool aborted = *s_decide != 0;
            if (!aborted && h == 0) {
                float M2 = m;
                for (int u = 1; u < EPI_WARPS / 4; ++u) M2 = fmaxf(M2, s_merge[u * M + r].x);
                float S2 = tot * ex2_approx(m - M2);
                for (int u = 1; u < EPI_WARPS / 4; ++u) {
                    const float2 o = s_merge[u * M + r];
                    S2 += o.y * ex2_approx(o.x - M2);
                }
                const int64_t row = (int64_t)tile * M + r;
                if (row < A.rows) A.part[(int64_t)split * A.tiles * M + row] = make_float2(M2, S2);
            }
            if (aborted) break;
            finish_tile<EPI_THREADS, M, 1>(A, tile, etid, s_red, s_flag);
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NBUF * N));
}

}  // namespace tc

// ----------------------------------------------------------------- tables
// For one cloud p [cnt, d] with potential pot (the column term the OTHER
// half-step reads), at the stage's kappa and c, rows padded to `pad` (multiple
// of 128) and K to `kp` bf16 (multiple of 64):
//   rowtab [pad][dpf] fp32 p' = p - o (for the row constant, float64 norm)
//   arow   [pad][kp] bf16 [ p1 | p1 | p2 | 1 1 1 | 0 ]   (this cloud as rows)
//   bcol   [pad][kp] bf16 [ Y1 | Y2 | Y1 | G1 G2 G3 | 0 ] (this cloud as columns),
// Y = 2 c kappa p', G = kappa (pot - c |p'|^2); padding points get zero rows
// and G = -inf (they add nothing).
__global__ void build_tc_tables_kernel(const float *__restrict__ p, const float *__restrict__ pot,
                                       int64_t cnt, int64_t pad, int d, int dpf, int kp,
                                       const double *__restrict__ o, const Params *__restrict__ prm,
                                       float *rowtab, __nv_bfloat16 *arow, __nv_bfloat16 *bcol) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= pad) return;
    const double kappa = prm->kappa, c = prm->c;
    const bool real = i < cnt;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.0f);
    __nv_bfloat16 *ar = arow + i * kp, *bc = bcol + i * kp;
    double nrm = 0.0;
    for (int q = 0; q < dpf; ++q) {
        const float v = (real && q < d) ? (float)((double)p[i * d + q] - o[q]) : 0.0f;
        rowtab[i * dpf + q] = v;
        nrm += (double)v * (double)v;
        if (q >= d) continue;
        const __nv_bfloat16 v1 = __float2bfloat16_rn(v);
        const __nv_bfloat16 v2 = __float2bfloat16_rn(v - __bfloat162float(v1));
        const double Y = 2.0 * c * kappa * (double)v;
        const __nv_bfloat16 y1 = __double2bfloat16(Y);
        const __nv_bfloat16 y2 = __double2bfloat16(Y - (double)__bfloat162float(y1));
        ar[q] = v1;
        ar[d + q] = v1;
        ar[2 * d + q] = v2;
        bc[q] = y1;
        bc[d + q] = y2;
        bc[2 * d + q] = y1;
    }
    double G = -INFINITY;
    if (real) {
        const float pv = pot[i];
        G = (pv == -INFINITY) ? -INFINITY : kappa * ((double)pv - c * nrm);
    }
    const __nv_bfloat16 g1 = __double2bfloat16(G);
    const double r1 = isfinite(G) ? G - (double)__bfloat162float(g1) : 0.0;
    const __nv_bfloat16 g2 = __double2bfloat16(r1);
    const __nv_bfloat16 g3 = __double2bfloat16(r1 - (double)__bfloat162float(g2));
    const __nv_bfloat16 one = __float2bfloat16_rn(real ? 1.0f : 0.0f);
    ar[3 * d] = one;
    ar[3 * d + 1] = one;
    ar[3 * d + 2] = one;
    bc[3 * d] = g1;
    bc[3 * d + 1] = g2;
    bc[3 * d + 2] = g3;
    for (int q = 3 * d + 3; q < kp; ++q) {
        ar[q] = zero;
        bc[q] = zero;
    }
}

// ----------------------------------------------------------------- launchers
int tc_ksteps(int d) { return (3 * d + 3 + 15) / 16; }
int tc_slabs(int d) { return (tc_ksteps(d) + 3) / 4; }

template <int KS>
static cudaError_t tc_prepare() {
    return cudaFuncSetAttribute(tc::hs_tc_kernel<KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tc::Smem<KS>::ALLOC);
}

cudaError_t tc_setup(int d) {
    switch (tc_slabs(d)) {
        case 1: return tc_prepare<1>();
        case 2: return tc_prepare<2>();
        case 3: return tc_prepare<3>();
        case 4: return tc_prepare<4>();
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_halfstep_tc(int d, const HalfStep &A, const CUtensorMap *tmA,
                               const CUtensorMap *tmB, int grid, cudaStream_t s) {
    const int ks = tc_slabs(d), ksteps = tc_ksteps(d);
    void *args[] = {(void *)&A, (void *)tmA, (void *)tmB, (void *)&ksteps};
    const void *fn = ks == 1 ? (const void *)tc::hs_tc_kernel<1>
                   : ks == 2 ? (const void *)tc::hs_tc_kernel<2>
                   : ks == 3 ? (const void *)tc::hs_tc_kernel<3>
                             : (const void *)tc::hs_tc_kernel<4>;
    const int bytes = ks == 1 ? tc::Smem<1>::ALLOC : ks == 2 ? tc::Smem<2>::ALLOC
                    : ks == 3 ? tc::Smem<3>::ALLOC : tc::Smem<4>::ALLOC;
    return cudaLaunchKernel(fn, dim3(grid), dim3(tc::THREADS), args, bytes, s);
}

cudaError_t launch_tc_tables(const float *p, const float *pot, int64_t cnt, int64_t pad, int d,
                             int dpf, int kp, const double *o, const Params *prm, float *rowtab,
                             void *arow, void *bcol, cudaStream_t s) {
    build_tc_tables_kernel<<<(unsigned)((pad + 127) / 128), 128, 0, s>>>(
        p, pot, cnt, pad, d, dpf, kp, o, prm, rowtab, static_cast<__nv_bfloat16 *>(arow),
        static_cast<__nv_bfloat16 *>(bcol));
    return cudaGetLastError();
}

// Tensor map of a [rows][kp] bf16 operand table: boxes of 64 x 128, 128B swizzle.
int make_operand_map(CUtensorMap *map, void *base, int64_t rows, int kp) {
    using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return -1;
        encode = reinterpret_cast<EncodeFn>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)kp, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kp * 2};
    const cuuint32_t box[2] = {(cuuint32_t)tc::SLAB, (cuuint32_t)tc::M};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : (int)r;
}

}  // namespace ot
