// api.cu -- host runtime behind the C ABI declared in include/ot_sinkhorn.h.
//
// Argument checks, one-time scale resolution (captured by the plan, moscot PR
// #846 "materialize transport-matrix rows instead of pushing indicator
// columns", section Fix), workspace sizing, launch shapes, and the iteration
// driver: the f/g half-step pair is replayed as a CUDA graph in chunks of
// check_every iterations on an internal stream; the host reads back only
// scalars (the device stop flag, the in-loop residual, the iteration count).
#include <cmath>
#include <cstdarg>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <new>
#include <atomic>
#include <vector>

#include "ot_sinkhorn.h"
#include "ot_sinkhorn_testing.h"
#include "runtime.h"

using namespace ot;

namespace {

thread_local char g_err[512] = "no error";

// failure tests (include/ot_sinkhorn_testing.h): which bounded device wait to
// make give up, 0 = none
std::atomic<int> g_wait_fault{0};

}  // namespace

// Records the calling thread's error text; returns code (shared by every
// entry point of the library).
int ot::set_error(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

namespace {

#define fail ot::set_error

#define OT_CU(call)                                                                      \
    do {                                                                                 \
        cudaError_t e_ = (call);                                                         \
        if (e_ != cudaSuccess)                                                           \
            return fail(e_ == cudaErrorMemoryAllocation ? OT_ERR_OOM : OT_ERR_CUDA,       \
                        "%s failed: %s", #call, cudaGetErrorString(e_));                 \
    } while (0)

int64_t round_up(int64_t v, int64_t q) { return (v + q - 1) / q * q; }

// small device-side scalars of a plan
struct DevScalars {
    int flags[4];                 // x, y, a, b: bit0 non-finite, bit1 negative
    unsigned long long zeros[2];  // zero weights in a, b
    unsigned max_bits;            // max-cost pass result (float bits)
    int bad;                      // row kernels: an index out of range
    float thr;
    int pad;
    int64_t argmin, n_massless, nnz;
    double r_sum[2];
    double sums[4][kMaxD];        // sum x, sum x^2, sum y, sum y^2 (per coordinate)
    double wsum[4];               // sum a, -, sum b, -
    unsigned long long visited;   // row passes: column chunks evaluated since the call began
};

// block-sparse mode: device counters of one iteration
struct SparseCtr {
    unsigned long long cand, adm;  // candidate and admitted tiles of the current mask
    unsigned long long exact;      // candidates whose exact mass was evaluated
    unsigned long long n_mode[2];  // iterations run sparse / dense (whole solve)
    int mode[2];                   // this iteration's kind (kMode*), the last counted kind
    unsigned lohi[6];              // joint bounding box (order-preserving float bits)
};

// pinned host mirror for read-backs
struct HostScalars {
    DevScalars s;
    State st;
    SparseCtr sc, sc_prev;
    double o[kMaxD];
};

struct Side {          // one cloud's half of the problem
    int64_t cnt, pad;  // points, padded to kColPad
    int64_t lo, rows;  // the rows this plan updates: [lo, lo + rows) (all of them unless sharded)
    float *rowtab;     // [pad][dp]
    float *coltab;     // layout per kind
    int tiles, splits, grid;
    int64_t cps;       // columns per split of the OTHER side's table
    int rpt, tile;     // rows per thread and rows per tile of this side's half-step
    void *arow, *bcol; // tensor-core path: bf16 operand tables [pad][kp] (rows, columns)
};

}  // namespace

struct ot_plan {
    int device = 0;
    const float *x = nullptr, *y = nullptr, *a = nullptr, *b = nullptr;
    float *f = nullptr, *g = nullptr;
    int64_t n = 0, m = 0;
    int d = 0, kind = 0, dim = 0, dp = 0;
    double eps = 0.0, c = 1.0;
    double mean_sq = 0.0;  // mean over all pairs of ||x_i - y_j||^2 (closed form)
    int64_t n_massless_rows = 0, n_massless_cols = 0;
    // workspace (one allocation, carved)
    char *ws = nullptr;
    size_t ws_bytes = 0, ws_rows_bytes = 0;  // as obtained from the pool
    Params *prm = nullptr;
    State *st = nullptr;
    double *o = nullptr;
    DevScalars *ds = nullptr;
    double *part1 = nullptr, *part2 = nullptr;  // coordinate-stat partials
    float *fspare = nullptr;
    float2 *part = nullptr;
    unsigned *tile_cnt = nullptr;
    double *tile_resid = nullptr;
    Side sx{}, sy{};
    // lazily allocated for the row kernels
    char *ws_rows = nullptr;
    double *dcol = nullptr, *rpart = nullptr;
    float *rowmax = nullptr;
    int64_t *counts = nullptr;
    int64_t *scan = nullptr;    // tile totals of the row_ptr scan
    // tile screen of the row passes (d <= 3): Morton orders of the clouds
    int64_t *mperm[2] = {nullptr, nullptr};  // x, y in Morton order (computed once)
    int64_t *rperm = nullptr;                // Morton order of a range of rows (per call)
    unsigned long long *rkeys = nullptr;     // sort keys
    double *csum = nullptr;                  // chunk summaries of the column table
    unsigned *rlohi = nullptr;               // a cloud's box (order-preserving bits)
    bool mperm_ready[2] = {false, false};
    int64_t screen_total = 0;                // row passes: chunks a full visit would evaluate
    int64_t screen_visited = 0;              // and those the last row call evaluated
    bool mort_ready[2] = {false, false};
    MortonArgs mort[2]{};
    HostScalars *hs = nullptr;  // pinned
    int kp = 0;                 // tensor-core path: bf16 K extent of the operand tables
    bool use_loop = false;      // device-resident iterations (loop.cu)
    int loop_grid = 0;
    int loop_rpt = 2;           // rows per thread of the loop kernel (1 or 2)
    unsigned *bar = nullptr;    // grid barrier: count, generation
    double *blk_resid = nullptr;
    // arrays the iterations read: the caller's, or their Morton-ordered copies
    // in block-sparse mode
    const float *sx_pts = nullptr, *sy_pts = nullptr, *sa = nullptr, *sb = nullptr;
    float *sf[2] = {nullptr, nullptr}, *sg = nullptr;
    // block-sparse mode (ot_options.block_sparse)
    bool sparse = false;
    int sp_B = 0, sp_rpt = 1, sp_verify = 1;
    int64_t sp_nb = 0, sp_mb = 0;
    int sp_splits[2] = {1, 1}, sp_grid[2] = {1, 1}, sp_vgrid = 1;
    double sp_delta = 0.0, sp_frac = 0.5, sp_bound = 0.0, asum = 0.0;
    char *ws_sp = nullptr;
    size_t ws_sp_bytes = 0;
    // sharded plan (ot_shard_plan_create): the row ranges [lo, hi) of x and y it updates
    bool shard = false;
    int64_t range[2][2] = {{0, 0}, {0, 0}};
    // ot_sinkhorn_pointcloud_host: the device copies of the caller's host arrays
    char *ws_in = nullptr;
    size_t ws_in_bytes = 0;
    int64_t *perm_x = nullptr, *perm_y = nullptr;
    unsigned long long *keys = nullptr;
    BlockSum *bsx = nullptr, *bsy = nullptr;
    uint8_t *mask = nullptr, *mask_t = nullptr;
    int64_t *cnt = nullptr, *cnt_t = nullptr, *ptr = nullptr, *ptr_t = nullptr, *sp_scan = nullptr;
    int *lst = nullptr, *lst_t = nullptr;
    float2 *sp_part = nullptr;
    unsigned *sp_tcnt = nullptr;
    double *sp_tres = nullptr;
    SparseCtr *sc = nullptr;
    int64_t last_cand = 0, last_adm = 0, last_exact = 0;  // tiles of the last mask an iteration ran on
    uint8_t *mask_out = nullptr;  // where the first mask goes (ot_options.sparse_mask_out), until then
    CUtensorMap tm_arow_x, tm_bcol_y, tm_arow_y, tm_bcol_x;
    cudaStream_t s_int = nullptr;
    cudaEvent_t ev_in = nullptr, ev_out = nullptr;
    cudaGraphExec_t graph[2] = {nullptr, nullptr};  // chunk graphs by start parity
    int graph_len = 0;
    int sm_count = 0;
    // accounting and optional loop timing (events around each chunk)
    int64_t launches = 0;
    bool timing = false;
    std::vector<cudaEvent_t> tev;
    size_t tev_used = 0;
    // block-sparse mode with timing: events around the verification and the
    // sparse half-step launches
    struct Marks {
        std::vector<cudaEvent_t> ev;
        size_t used = 0;
    } tm_verify, tm_hs;
};

namespace {

void plan_free(ot_plan *p) {
    if (!p) return;
    // everything below belongs to the plan's device, which need not be the
    // current one (a plan may be destroyed from any thread, under any device)
    int prev = -1;
    const bool swap = cudaGetDevice(&prev) == cudaSuccess && prev != p->device &&
                      cudaSetDevice(p->device) == cudaSuccess;
    for (auto &gx : p->graph)
        if (gx) cudaGraphExecDestroy(gx);
    for (auto ev : p->tev) cudaEventDestroy(ev);
    for (auto ev : p->tm_verify.ev) cudaEventDestroy(ev);
    for (auto ev : p->tm_hs.ev) cudaEventDestroy(ev);
    // the workspaces and the stream go back to the pool once the plan's work is done
    if (p->s_int) cudaStreamSynchronize(p->s_int);
    pool_device_free(p->ws, p->ws_bytes, p->device);
    pool_device_free(p->ws_rows, p->ws_rows_bytes, p->device);
    pool_device_free(p->ws_sp, p->ws_sp_bytes, p->device);
    pool_device_free(p->ws_in, p->ws_in_bytes, p->device);
    pool_host_free(p->hs, sizeof(HostScalars));
    if (p->ev_in) cudaEventDestroy(p->ev_in);
    if (p->ev_out) cudaEventDestroy(p->ev_out);
    pool_stream_release(p->s_int, p->device);
    if (swap) cudaSetDevice(prev);
    delete p;
}

// Carves aligned sub-buffers out of one allocation (first pass: sizing only).
struct Carver {
    char *base;
    size_t off = 0;
    template <typename T>
    T *take(int64_t count) {
        off = (size_t)round_up((int64_t)off, 256);
        T *ptr = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += (size_t)count * sizeof(T);
        return ptr;
    }
};

// Time of the most loaded SM, in units of one item run at the SM's full ex2
// rate. `items` equal items go to grid = min(items, cap) resident blocks, block
// b taking items b, b + grid, ...; blocks land on SMs round-robin. The SM's
// blocks share its ex2 pipe, which `fill` blocks keep busy: with k < fill
// active blocks it runs at k / fill of its rate. So blocks that hold one item
// more than the others finish in a slower tail.
double sm_time(int64_t items, int64_t cap, int sms, int fill) {
    const int64_t grid = std::min(items, cap);
    const int64_t nb = (grid + sms - 1) / sms;         // blocks on the busiest SM
    const int64_t hi = (items + grid - 1) / grid;      // most items of one block
    const int64_t rem = items - (hi - 1) * grid;       // blocks holding hi items
    const int64_t k_hi = std::min(nb, (rem + sms - 1) / sms);
    double t = 0.0;
    if (hi > 1) t += (double)(nb * (hi - 1)) * fill / (double)std::min<int64_t>(nb, fill);
    t += (double)k_hi * fill / (double)std::min<int64_t>(k_hi, fill);
    return t;
}

// Column splits for one half-step: rows -> tiles of `tile` rows; the column
// table of `cols_pad` columns is cut into `splits` spans (multiples of `gran`).
// Cost model in column-equivalents of one thread's work, an item being
// rpt * (cps + 64 per-item overhead):
//  - static assignment (loop and tensor-core kernels): the busiest SM's time
//    (sm_time);
//  - dynamic assignment (per-launch CUDA-core kernels, which claim items from a
//    counter) with more items than resident blocks: the SMs stay balanced, so
//    the work per SM (no less than `fill` items: fewer do not keep the ex2 pipe
//    busy) plus a tail of about one item (fitted to measurements at n = m =
//    1e5 and 3e5, d = 3); with one wave of items or less, sm_time again
//    (measured at n = m = 8000: 13 splits 35.3 us, 20 splits 38.9 us);
// plus the merge by the block that finishes a tile of `splits` partials per
// row (~8 columns each). Returns the estimate of the best split count, which
// it stores in sd.
double choose_splits(int64_t rows, int64_t cols_pad, int rpt, int tile, int cap, Side &sd,
                     int force_s = 0, int gran = kColPad, int sms = 148, int fill = 3,
                     bool dynamic = false) {
    const int64_t tiles = (rows + tile - 1) / tile;
    double best = 1e300;
    int best_s = 1;
    int64_t best_cps = cols_pad;
    const int64_t max_s = std::min<int64_t>(cols_pad / gran, 4096);
    for (int64_t s = 1; s <= max_s; ++s) {
        const int64_t cps = round_up((cols_pad + s - 1) / s, gran);
        const int64_t s_eff = (cols_pad + cps - 1) / cps;
        if (force_s > 0) {
            if (s != std::min<int64_t>(force_s, max_s)) continue;  // the nearest attainable count
        } else if (s_eff != s) {
            continue;
        }
        const int64_t items = tiles * s_eff;
        const double item = (double)rpt * (double)(cps + 64);
        const double per_sm = (dynamic && items > cap)
                                  ? std::max((double)items / sms, (double)fill) + 1.2
                                  : sm_time(items, cap, sms, fill);
        const double t = per_sm * item + 8.0 * rpt * (double)s_eff;
        if (t < best * 0.995) {
            best = t;
            best_s = (int)s_eff;
            best_cps = cps;
        }
    }
    sd.tiles = (int)tiles;
    sd.splits = best_s;
    sd.cps = best_cps;
    sd.grid = (int)std::min<int64_t>(tiles * best_s, cap);
    sd.rpt = rpt;
    sd.tile = tile;
    return best;
}

// Launch shape of one side's half-step: for d <= 3 also picks the rows per
// thread (8, 4 or 2) with the smallest estimate.
int choose_shape(int kind, int dim, int sms, int64_t rows, int64_t cols_pad, Side &sd,
                 int force_s, int force_rpt) {
    if (kind == 2) {  // tensor cores: one 288-thread block per SM, 128-row tiles, 128-column chunks
        choose_splits(rows, cols_pad, 1, 128, sms, sd, force_s, 128, sms, 1);
        return OT_OK;
    }
    if (kind == 1) {
        const int bps = halfstep_blocks_per_sm(1, dim, kGnRows);
        if (bps <= 0) return fail(OT_ERR_CUDA, "half-step kernel cannot be made resident");
        choose_splits(rows, cols_pad, kGnRows, kGnTile, bps * sms, sd, force_s, kColPad, sms, 3, true);
        return OT_OK;
    }
    double best = 1e300;
    for (int rpt : {8, 4, 2, 1}) {  // 1 only when asked for
        if (force_rpt > 0 ? rpt != force_rpt : rpt == 1) continue;
        const int bps = halfstep_blocks_per_sm(0, dim, rpt);
        if (bps <= 0) continue;
        Side tmp = sd;
        // measured: 2 rows per thread run ~4% faster than 4 or 8 at n = 1e5..3e5
        // (more resident warps hide the ex2 and shared-memory latency)
        const double eff = rpt == 2 ? 1.04 : 1.0;
        const double t =
            choose_splits(rows, cols_pad, rpt, kHsThreads * rpt, bps * sms, tmp, force_s, kColPad, sms, 3,
                          true) / eff;
        if (t < best) {
            best = t;
            sd = tmp;
        }
    }
    if (best >= 1e300) return fail(OT_ERR_CUDA, "half-step kernel cannot be made resident");
    return OT_OK;
}

}  // namespace

namespace {

// Reads the solver state back (synchronises the internal stream).
int read_state(ot_plan *p) {
    OT_CU(cudaMemcpyAsync(&p->hs->st, p->st, sizeof(State), cudaMemcpyDeviceToHost, p->s_int));
    OT_CU(cudaStreamSynchronize(p->s_int));
    return OT_OK;
}

int read_scalars(ot_plan *p) {
    OT_CU(cudaMemcpyAsync(&p->hs->s, p->ds, sizeof(DevScalars), cudaMemcpyDeviceToHost, p->s_int));
    OT_CU(cudaStreamSynchronize(p->s_int));
    return OT_OK;
}

HalfStep make_step(const ot_plan *p, int side, int parity) {
    HalfStep A{};
    const bool f = side == 0;
    const Side &rows = f ? p->sx : p->sy;
    const Side &cols = f ? p->sy : p->sx;
    float *const *fb = p->sf;
    A.coltab = reinterpret_cast<const float4 *>(cols.coltab);
    A.rowtab = rows.rowtab + rows.lo * p->dp;
    A.rows = rows.rows;
    A.row_off = rows.lo;
    A.cols_pad = cols.pad;
    A.cols_per_split = rows.cps;
    A.splits = rows.splits;
    A.tiles = rows.tiles;
    A.tile_rows = rows.tile;
    A.dp = p->dp;
    A.side = side;
    A.part = p->part;
    A.tile_cnt = p->tile_cnt;
    A.tile_resid = p->tile_resid;
    A.w = (f ? p->sa : p->sb) + rows.lo;
    A.pot_old = (f ? fb[parity] : p->sg) + rows.lo;
    A.pot_new = (f ? fb[parity ^ 1] : p->sg) + rows.lo;
    // this side's column table feeds the other half-step; row r of the update is
    // point lo + r (lo is even: pairs of columns share a record in layout 0)
    A.next_col = rows.coltab;
    A.nxt_bf16 = 0;
    if (p->kind == 0) {
        A.nxt_a = 8; A.nxt_l = 1; A.nxt_b = 6;
        A.next_col += (rows.lo >> 1) * 8;
    } else if (p->kind == 1) {
        A.nxt_a = 2 * (p->dp + 4); A.nxt_l = p->dp + 4; A.nxt_b = p->dp;
        A.next_col += rows.lo * (p->dp + 4);
    } else {
        A.next_col = static_cast<float *>(rows.bcol) + (rows.lo * p->kp) / 2;  // bf16 elements
        A.nxt_bf16 = 1;
        A.nxt_a = p->kp; A.nxt_l = 0; A.nxt_b = 3 * p->d;
    }
    A.prm = p->prm;
    A.st = p->st;
    const bool fault = g_wait_fault.load() == 2;
    A.wait_polls = fault ? (1u << 12) : (1u << 22);
    A.withhold = fault ? 1 : 0;
    return A;
}

// Records a timing event on the internal stream (no-op unless timing).
cudaError_t mark(ot_plan *p) {
    if (!p->timing) return cudaSuccess;
    if (p->tev_used == p->tev.size()) {
        cudaEvent_t ev;
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) return e;
        p->tev.push_back(ev);
    }
    return cudaEventRecord(p->tev[p->tev_used++], p->s_int);
}

// The same for one kind of kernel (pairs of events around its launches).
cudaError_t mark_in(ot_plan *p, ot_plan::Marks &mk) {
    if (!p->timing) return cudaSuccess;
    if (mk.used == mk.ev.size()) {
        cudaEvent_t ev;
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) return e;
        mk.ev.push_back(ev);
    }
    return cudaEventRecord(mk.ev[mk.used++], p->s_int);
}

int sum_marks(const ot_plan::Marks &mk, double *ms_out) {
    double t = 0.0;
    for (size_t e = 0; e + 1 < mk.used; e += 2) {
        float ms = 0.0f;
        OT_CU(cudaEventElapsedTime(&ms, mk.ev[e], mk.ev[e + 1]));
        t += ms;
    }
    *ms_out = t;
    return OT_OK;
}

// One half-step: side 0 updates f (rows x, columns y), side 1 updates g.
cudaError_t launch_side(const ot_plan *p, int side, int parity) {
    const Side &sd = side == 0 ? p->sx : p->sy;
    if (p->kind == 2)
        return launch_halfstep_tc(p->d, make_step(p, side, parity),
                                  side == 0 ? &p->tm_arow_x : &p->tm_arow_y,
                                  side == 0 ? &p->tm_bcol_y : &p->tm_bcol_x, sd.grid, p->s_int);
    return launch_halfstep(p->kind, p->dim, sd.rpt, make_step(p, side, parity), sd.grid, p->s_int);
}

cudaError_t launch_iteration(const ot_plan *p, int parity) {
    cudaError_t e = launch_side(p, 0, parity);
    if (e != cudaSuccess) return e;
    return launch_side(p, 1, parity);
}

// ------------------------------------------------------- block-sparse mode
// (csrc/sparse.cu has the kernels and the design)

int64_t next_pow2(int64_t v) {
    int64_t r = 1;
    while (r < v) r <<= 1;
    return r;
}

float float_from_order(unsigned o) {
    const unsigned b = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
    float v;
    std::memcpy(&v, &b, sizeof v);
    return v;
}

// Verification work items per row block: the candidates cluster on a few row
// blocks, so whole row blocks as items left SMs idle at the end of the launch
// (ncu at n = m = 2^18: SMs active 76 % of the elapsed cycles).
constexpr int kVerifySegs = 8;

// Block size, launch shapes and workspace; the Morton order of both clouds and
// the sorted copies of the points, weights and (warm start) potentials; the
// blocks' static summaries. Runs after resolve_scale.
int sparse_setup(ot_plan *p, const ot_options &o, double tol, bool warm) {
    const int64_t n = p->n, m = p->m;
    const int d = p->d;
    int B = o.sparse_block;
    if (B == 0) {
        const int64_t nb = (n + 127) / 128, mb = (m + 127) / 128;
        B = (double)nb * (double)mb <= (double)(1ll << 27) ? 128 : 256;
    }
    p->sp_B = B;
    p->sp_rpt = B / kHsThreads;
    const int64_t nb = (n + B - 1) / B, mb = (m + B - 1) / B;
    p->sp_nb = nb;
    p->sp_mb = mb;
    if ((double)nb * (double)mb > (double)(1ll << 32))
        return fail(OT_ERR_UNSUPPORTED, "block mask of %lld x %lld pairs is too large (use a larger block)",
                    (long long)nb, (long long)mb);
    if (nb > 65535ll * 32 || (mb + 63) / 64 > 65535)
        return fail(OT_ERR_UNSUPPORTED, "too many blocks for the screen's grid");
    if (o.sparse_mask_out) {
        if (o.sparse_mask_len < nb * mb)
            return fail(OT_ERR_INVALID_ARG, "sparse_mask_len %lld < %lld block pairs",
                        (long long)o.sparse_mask_len, (long long)(nb * mb));
        p->mask_out = o.sparse_mask_out;
    }
    p->sp_delta = o.sparse_delta > 0.0 ? o.sparse_delta : tol / (4.0 * (double)std::max(nb, mb));
    p->sp_frac = o.sparse_dense_frac;
    p->sp_verify = o.sparse_verify;
    p->sp_bound = (double)mb * p->sp_delta * p->asum;
    const int bps = sparse_blocks_per_sm(0, d, p->sp_rpt);
    const int vbps = sparse_blocks_per_sm(1, d, p->sp_rpt);
    if (bps <= 0 || vbps <= 0) return fail(OT_ERR_CUDA, "block-sparse kernels cannot be made resident");
    const int64_t cap = (int64_t)bps * p->sm_count;
    for (int side = 0; side < 2; ++side) {
        // side 1 (the g-update) with items of about 1/8 of a wave, so the launch's
        // tail is short (measured: 3.57 -> 3.40 ms at n = m = 1e6, 0.77 -> 0.71 ms
        // at 2^18 against 1/2 of a wave); side 0 only serves the fallback launch,
        // whose items mostly return at once
        const int64_t tiles = side == 0 ? nb : mb;
        const int64_t per = side == 0 ? 2 : 8;
        const int64_t sp = std::min<int64_t>(std::max<int64_t>((per * cap + tiles - 1) / tiles, 1), 32);
        p->sp_splits[side] = (int)sp;
        p->sp_grid[side] = (int)std::min<int64_t>(tiles * sp, cap);
    }
    p->sp_vgrid = (int)std::min<int64_t>(nb * kVerifySegs, (int64_t)vbps * p->sm_count);
    const int64_t n2x = next_pow2(n), n2y = next_pow2(m);
    const int64_t part = std::max({(int64_t)p->sp_splits[0] * nb, (int64_t)kVerifySegs * nb,
                                   (int64_t)p->sp_splits[1] * mb}) * B;
    float *xs = nullptr, *ys = nullptr, *as = nullptr, *bs = nullptr;
    for (int pass = 0; pass < 2; ++pass) {
        Carver cv{pass ? p->ws_sp : nullptr};
        xs = cv.take<float>(n * d);
        ys = cv.take<float>(m * d);
        as = cv.take<float>(n);
        bs = cv.take<float>(m);
        p->sf[0] = cv.take<float>(n);
        p->sf[1] = cv.take<float>(n);
        p->sg = cv.take<float>(m);
        p->perm_x = cv.take<int64_t>(n);
        p->perm_y = cv.take<int64_t>(m);
        p->keys = cv.take<unsigned long long>(std::max(n2x, n2y));
        p->bsx = cv.take<BlockSum>(nb);
        p->bsy = cv.take<BlockSum>(mb);
        p->mask = cv.take<uint8_t>(nb * mb);
        p->mask_t = cv.take<uint8_t>(nb * mb);
        p->cnt = cv.take<int64_t>(nb);
        p->cnt_t = cv.take<int64_t>(mb);
        p->ptr = cv.take<int64_t>(nb + 1);
        p->ptr_t = cv.take<int64_t>(mb + 1);
        p->sp_scan = cv.take<int64_t>(scan_tmp_count(std::max(nb, mb)));
        p->lst = cv.take<int>(nb * mb);
        p->lst_t = cv.take<int>(nb * mb);
        p->sp_part = cv.take<float2>(part);
        p->sp_tcnt = cv.take<unsigned>(std::max(nb, mb));
        p->sp_tres = cv.take<double>(std::max(nb, mb));
        p->sc = cv.take<SparseCtr>(1);
        if (pass == 0) OT_CU(pool_device_alloc(reinterpret_cast<void **>(&p->ws_sp), cv.off, &p->ws_sp_bytes));
    }
    cudaStream_t s = p->s_int;
    OT_CU(cudaMemsetAsync(p->sp_tcnt, 0, sizeof(unsigned) * std::max(nb, mb), s));
    OT_CU(cudaMemsetAsync(p->sc, 0, sizeof(SparseCtr), s));
    OT_CU(cudaMemsetAsync(p->sc->lohi, 0xff, sizeof(unsigned) * 3, s));
    OT_CU(launch_box(p->x, n, d, p->sc->lohi, s));
    OT_CU(launch_box(p->y, m, d, p->sc->lohi, s));
    OT_CU(cudaMemcpyAsync(&p->hs->sc, p->sc, sizeof(SparseCtr), cudaMemcpyDeviceToHost, s));
    OT_CU(cudaStreamSynchronize(s));
    MortonArgs M{};
    M.d = d;
    M.bits = 30 / d;
    const double cells = (double)(1ll << M.bits);
    for (int k = 0; k < 3; ++k) {
        if (k >= d) continue;
        const double lo = (double)float_from_order(p->hs->sc.lohi[k]);
        const double hi = (double)float_from_order(p->hs->sc.lohi[3 + k]);
        M.lo[k] = lo;
        M.s[k] = hi > lo ? cells / (hi - lo) : 0.0;
    }
    OT_CU(launch_morton_sort(p->x, n, n2x, M, p->keys, s));
    OT_CU(launch_gather(p->keys, n, d, p->x, p->a, warm ? p->f : nullptr, p->perm_x, xs, as,
                        p->sf[0], s));
    OT_CU(launch_morton_sort(p->y, m, n2y, M, p->keys, s));
    OT_CU(launch_gather(p->keys, m, d, p->y, p->b, warm ? p->g : nullptr, p->perm_y, ys, bs, p->sg, s));
    if (!warm) {
        OT_CU(cudaMemsetAsync(p->sf[0], 0, sizeof(float) * n, s));
        OT_CU(cudaMemsetAsync(p->sg, 0, sizeof(float) * m, s));
    }
    OT_CU(launch_block_static(xs, as, n, d, B, p->bsx, s));
    OT_CU(launch_block_static(ys, bs, m, d, B, p->bsy, s));
    p->sx_pts = xs;
    p->sy_pts = ys;
    p->sa = as;
    p->sb = bs;
    return OT_OK;
}

HalfStep make_sparse_step(const ot_plan *p, int side, int parity) {
    HalfStep A = make_step(p, side, parity);
    const bool f = side == 0;
    A.splits = p->sp_splits[side];
    A.tiles = (int)(f ? p->sp_nb : p->sp_mb);
    A.tile_rows = p->sp_B;
    A.part = p->sp_part;
    A.tile_cnt = p->sp_tcnt;
    A.tile_resid = p->sp_tres;
    A.sp_ptr = f ? p->ptr : p->ptr_t;
    A.sp_idx = f ? p->lst : p->lst_t;
    A.sp_coltiles = (int)(f ? p->sp_mb : p->sp_nb);
    return A;
}

// One block-sparse iteration from the state at f-buffer parity `par`: the
// mask at (f, g), then the f-update (f_only: the update that measures the
// final residual) and the g-update on it. Nothing is read back: a kernel after
// the screen chooses dense or sparse updates on the device (the candidate count
// against sparse_dense_frac of all block pairs), and the launches of both kinds
// are gated on that choice; once the stop test has passed every launch returns
// at once, so the host only reads the state every check_every iterations.
int sparse_iteration(ot_plan *p, int par, bool f_only, double eps) {
    cudaStream_t s = p->s_int;
    const int64_t nb = p->sp_nb, mb = p->sp_mb;
    const int B = p->sp_B, d = p->d, rpt = p->sp_rpt;
    OT_CU(launch_block_max(p->sf[par], p->n, B, kLog2e / eps, p->bsx, s));
    OT_CU(launch_block_max(p->sg, p->m, B, kLog2e / eps, p->bsy, s));
    OT_CU(launch_sparse_prep(p->cnt, nb, p->cnt_t, mb, &p->sc->cand, 3, p->st, s));
    ScreenArgs S{};
    S.st = p->st;
    S.rs = p->bsx;
    S.cs = p->bsy;
    S.nb = nb;
    S.mb = mb;
    S.d = d;
    S.c = p->c;
    S.eps = eps;
    S.ln_delta = std::log(p->sp_delta);
    S.mask = p->mask;
    S.cnt = p->cnt;
    S.cnt_t = p->cnt_t;
    S.total = &p->sc->cand;
    OT_CU(launch_screen(S, s));
    OT_CU(launch_decide(&p->sc->cand, p->sp_frac * (double)nb * (double)mb, p->st, p->sc->mode,
                        p->sc->n_mode, f_only ? 0 : 1, s));
    p->launches += 5;
    auto gated = [&](HalfStep A, int val) {
        A.gate = p->sc->mode;
        A.gate_val = val;
        return A;
    };
    // dense f-update (when the candidates are too many)
    OT_CU(launch_halfstep(p->kind, p->dim, p->sx.rpt, gated(make_step(p, 0, par), kModeDense),
                          p->sx.grid, s));
    p->launches += 1;
    if (p->sp_verify) {
        // the candidates as compressed rows, then admitted counts from zero
        OT_CU(launch_row_ptr_scan(p->cnt, nb, p->ptr, p->sp_scan, s));
        OT_CU(launch_mask_list(p->mask, nb, mb, p->ptr, p->lst, s));
        OT_CU(cudaMemsetAsync(p->cnt, 0, sizeof(int64_t) * nb, s));
        VerifyArgs V{};
        V.coltab = reinterpret_cast<const float4 *>(p->sy.coltab);
        V.rowtab = p->sx.rowtab;
        V.pot = p->sf[par];
        V.pts = p->sx_pts;
        V.prm = p->prm;
        V.rs = p->bsx;
        V.cs = p->bsy;
        V.rows = p->n;
        V.cols_pad = p->sy.pad;
        V.nb = nb;
        V.mb = mb;
        V.l2_delta = std::log2(p->sp_delta);
        V.mask = p->mask;
        V.cptr = p->ptr;
        V.clist = p->lst;
        V.segs = kVerifySegs;
        V.cnt = p->cnt;
        V.cnt_t = p->cnt_t;
        V.total = &p->sc->adm;
        V.exact = &p->sc->exact;
        // the verification and the f-update over the admitted tiles in one launch
        HalfStep A = gated(make_sparse_step(p, 0, par), kModeSparse);
        A.splits = kVerifySegs;
        OT_CU(mark_in(p, p->tm_verify));
        OT_CU(launch_verify(d, rpt, A, V, p->sp_vgrid, s));
        OT_CU(mark_in(p, p->tm_verify));
        // row blocks left without an admitted tile: f-update over every column
        OT_CU(cudaMemsetAsync(&p->st->work[0], 0, sizeof(unsigned), s));
        HalfStep Af = gated(make_sparse_step(p, 0, par), kModeSparse);
        Af.sp_ptr = nullptr;
        Af.sp_idx = nullptr;
        Af.sp_fallback = p->cnt;
        OT_CU(launch_halfstep_sparse(d, rpt, Af, p->sp_grid[0], s));
        p->launches += 6;
    } else {
        OT_CU(launch_row_ptr_scan(p->cnt, nb, p->ptr, p->sp_scan, s));
        OT_CU(launch_mask_list(p->mask, nb, mb, p->ptr, p->lst, s));
        OT_CU(mark_in(p, p->tm_hs));
        OT_CU(launch_halfstep_sparse(d, rpt, gated(make_sparse_step(p, 0, par), kModeSparse),
                                     p->sp_grid[0], s));
        OT_CU(mark_in(p, p->tm_hs));
        p->launches += 5;
    }
    if (p->mask_out) {  // the solve's first mask (at the starting potentials), on request
        OT_CU(cudaMemcpyAsync(p->mask_out, p->mask, (size_t)(nb * mb), cudaMemcpyDeviceToDevice, s));
        p->mask_out = nullptr;
    }
    if (!f_only) {
        OT_CU(launch_transpose_bytes(p->mask, nb, mb, p->mask_t, s));
        OT_CU(launch_row_ptr_scan(p->cnt_t, mb, p->ptr_t, p->sp_scan, s));
        OT_CU(launch_mask_list(p->mask_t, mb, nb, p->ptr_t, p->lst_t, s));
        OT_CU(launch_halfstep(p->kind, p->dim, p->sy.rpt, gated(make_step(p, 1, par), kModeDense),
                              p->sy.grid, s));
        OT_CU(mark_in(p, p->tm_hs));
        OT_CU(launch_halfstep_sparse(d, rpt, gated(make_sparse_step(p, 1, par), kModeSparse),
                                     p->sp_grid[1], s));
        OT_CU(mark_in(p, p->tm_hs));
        p->launches += 7;
    }
    return OT_OK;
}

// `iters` block-sparse iterations from global parity `parity0`; the state is
// read every `check` iterations, and the loop ends once the stop test has passed.
int run_sparse(ot_plan *p, int parity0, int iters, double eps, int check) {
    for (int i = 0; i < iters; ++i) {
        OT_CU(mark(p));
        int rc = sparse_iteration(p, (parity0 + i) & 1, false, eps);
        OT_CU(mark(p));
        if (rc != OT_OK) return rc;
        if ((i + 1) % check == 0 && i + 1 < iters) {
            if ((rc = read_state(p)) != OT_OK) return rc;
            if (p->hs->st.stop) break;
        }
    }
    return OT_OK;
}

// Runs `iters` iterations starting at global parity `parity0`, in chunks of
// graph_len (replayed graphs when enabled). With `check`, the stop flag is
// read after every chunk. Returns OT status.
// Device-resident path: chunks of up to kLoopChunk iterations per cooperative launch.
constexpr int kLoopChunk = 256;

int run_loop(ot_plan *p, int parity0, int iters, bool check) {
    LoopArgs L{};
    L.f[0] = make_step(p, 0, 0);
    L.f[1] = make_step(p, 0, 1);
    L.g[0] = L.g[1] = make_step(p, 1, 0);
    L.bar_count = p->bar;
    L.bar_gen = p->bar + 1;
    L.blk_resid = p->blk_resid;
    const bool fault = g_wait_fault.load() == 1;
    L.wait_ns = fault ? 2000000ull : 10000000000ull;  // 2 ms under the failure test, else 10 s
    L.withhold_block = fault ? 0 : -1;
    int i = 0;
    while (i < iters) {
        const int len = std::min(kLoopChunk, iters - i);
        L.iters = len;
        L.parity0 = (parity0 + i) & 1;
        OT_CU(cudaMemsetAsync(p->bar, 0, sizeof(unsigned), p->s_int));  // arrivals
        OT_CU(mark(p));
        OT_CU(launch_loop(p->d, p->loop_rpt, L, p->loop_grid, p->s_int));
        OT_CU(mark(p));
        p->launches += 1;
        i += len;
        if (check || i < iters) {
            int rc = read_state(p);
            if (rc != OT_OK) return rc;
            if (p->hs->st.stop || p->hs->st.wait_timeout) break;
        }
    }
    return OT_OK;
}

int run_iterations(ot_plan *p, int parity0, int iters, bool check, bool use_graphs) {
    if (p->use_loop) return run_loop(p, parity0, iters, check);
    int i = 0;
    while (i < iters) {
        const int len = std::min(p->graph_len, iters - i);
        const int par = (parity0 + i) & 1;
        OT_CU(mark(p));
        if (use_graphs && len == p->graph_len) {
            if (!p->graph[par]) {
                cudaGraph_t gr = nullptr;
                OT_CU(cudaStreamBeginCapture(p->s_int, cudaStreamCaptureModeThreadLocal));
                cudaError_t le = cudaSuccess;
                for (int k = 0; k < len && le == cudaSuccess; ++k)
                    le = launch_iteration(p, (par + k) & 1);
                cudaError_t ce = cudaStreamEndCapture(p->s_int, &gr);
                if (le != cudaSuccess || ce != cudaSuccess) {
                    if (gr) cudaGraphDestroy(gr);
                    return fail(OT_ERR_CUDA, "graph capture failed: %s",
                                cudaGetErrorString(le != cudaSuccess ? le : ce));
                }
                cudaError_t ie = cudaGraphInstantiate(&p->graph[par], gr, 0);
                cudaGraphDestroy(gr);
                if (ie != cudaSuccess)
                    return fail(OT_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(ie));
            }
            OT_CU(cudaGraphLaunch(p->graph[par], p->s_int));
        } else {
            for (int k = 0; k < len; ++k) OT_CU(launch_iteration(p, (par + k) & 1));
        }
        OT_CU(mark(p));
        p->launches += 2 * len;
        i += len;
        if (check) {
            int rc = read_state(p);
            if (rc != OT_OK) return rc;
            if (p->hs->st.stop) break;
        }
    }
    return OT_OK;
}

// The current device must be sm_100; its SM count is cached per device (two
// attribute queries the first time: a full property query costs milliseconds,
// which every call would otherwise spend before its first launch).
int check_device(int *dev, int *sms) {
    static std::atomic<int> cached_sms[64];  // 0: not queried yet
    OT_CU(cudaGetDevice(dev));
    if (*dev >= 0 && *dev < 64) {
        const int c = cached_sms[*dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *sms = c;
            return OT_OK;
        }
    }
    int major = 0, minor = 0, count = 0;
    OT_CU(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev));
    OT_CU(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev));
    if (major != 10)
        return fail(OT_ERR_CUDA, "device %d is sm_%d%d; this library is built for sm_100a", *dev, major,
                    minor);
    OT_CU(cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, *dev));
    if (*dev >= 0 && *dev < 64) cached_sms[*dev].store(count, std::memory_order_relaxed);
    *sms = count;
    return OT_OK;
}

}  // namespace

extern "C" {

int ot_version(void) { return OT_ABI_VERSION; }

const char *ot_last_error_string(void) { return g_err; }

void ot_options_default(ot_options *opt) {
    if (!opt) return;
    std::memset(opt, 0, sizeof *opt);
    opt->warm_start = 0;
    opt->check_every = 16;
    opt->use_graphs = 1;
    opt->iters_per_stage = 20;
    opt->scale_value = 1.0;
    opt->eps_init = 0.0;
    opt->eps_decay = 0.7;
    opt->timing = 0;
    opt->col_splits = 0;
    opt->rows_per_thread = 0;
    opt->tensor_cores = 1;
    opt->device_loop = -1;
    opt->block_sparse = 0;
    opt->sparse_block = 0;
    opt->sparse_verify = 1;
    opt->sparse_delta = 0.0;
    opt->sparse_dense_frac = 0.5;
    opt->resid_history = nullptr;
    opt->resid_history_len = 0;
    opt->sparse_mask_out = nullptr;
    opt->sparse_mask_len = 0;
}

void ot_plan_destroy(ot_plan *plan) {
    NvtxRange nvtx_range("ot_plan_destroy");
    plan_free(plan);
}

void ot_testing_wait_fault(int mode) { g_wait_fault.store(mode == 1 || mode == 2 ? mode : 0); }

}  // extern "C"

namespace {

// Allocates the plan's solve workspace and chooses launch shapes.
int plan_setup(ot_plan *p, const ot_options &o) {
    if (p->d <= 3) {
        p->kind = 0;
        p->dim = p->d;
        p->dp = 4;
    } else if (p->d >= 16 && o.tensor_cores) {
        p->kind = 2;
        p->dim = p->d;
        p->dp = (int)round_up(p->d, 4);
        p->kp = 64 * tc_slabs(p->d);
    } else {
        p->kind = 1;
        p->dim = p->d <= 8 ? 8 : p->d <= 16 ? 16 : p->d <= 32 ? 32 : 64;
        p->dp = p->dim;
    }
    const int64_t colw = p->kind == 0 ? 4 : p->kind == 1 ? p->dp + 4 : 0;
    const int64_t padq = p->kind == 2 ? 128 : kColPad;
    p->sx.cnt = p->n;
    p->sy.cnt = p->m;
    p->sx.pad = round_up(p->n, padq);
    p->sy.pad = round_up(p->m, padq);
    p->sx.lo = p->shard ? p->range[0][0] : 0;
    p->sx.rows = p->shard ? p->range[0][1] - p->range[0][0] : p->n;
    p->sy.lo = p->shard ? p->range[1][0] : 0;
    p->sy.rows = p->shard ? p->range[1][1] - p->range[1][0] : p->m;
    if (!p->shard && p->kind == 0 && o.device_loop != 0 &&
        (o.device_loop == 1 || (double)p->n * (double)p->m <= (double)(1ll << 28))) {
        // rows per thread (1 or 2, both half-steps) with the smaller estimate;
        // measured: 1 row runs ~6 % slower per pair, but balances better on some sizes
        double best = 1e300;
        for (int rpt : {2, 1}) {
            if (o.rows_per_thread > 0 && rpt != o.rows_per_thread) continue;
            const int bps = loop_blocks_per_sm(p->d, rpt);
            if (bps <= 0) continue;
            Side sx = p->sx, sy = p->sy;
            const double t = (choose_splits(p->n, p->sy.pad, rpt, kHsThreads * rpt, bps * p->sm_count, sx,
                                            o.col_splits, kColPad, p->sm_count) +
                              choose_splits(p->m, p->sx.pad, rpt, kHsThreads * rpt, bps * p->sm_count, sy,
                                            o.col_splits, kColPad, p->sm_count)) /
                             (rpt == 1 ? 0.94 : 1.0);
            if (t < best) {
                best = t;
                p->use_loop = true;
                p->loop_rpt = rpt;
                p->loop_grid = bps * p->sm_count;
                p->sx = sx;
                p->sy = sy;
            }
        }
        if (p->use_loop) {
            // no more blocks than there is work for: every block arrives at every barrier
            const int64_t work = std::max({(int64_t)p->sx.tiles * p->sx.splits,
                                           (int64_t)p->sy.tiles * p->sy.splits,
                                           (std::max(p->n, p->m) + kHsThreads - 1) / kHsThreads,
                                           (int64_t)1});
            p->loop_grid = (int)std::min<int64_t>(p->loop_grid, work);
        }
    }
    int rc = OT_OK;
    if (!p->use_loop)
        rc = choose_shape(p->kind, p->dim, p->sm_count, std::max<int64_t>(p->sx.rows, 1), p->sy.pad, p->sx,
                          o.col_splits, o.rows_per_thread);
    if (rc != OT_OK) return rc;
    if (!p->use_loop && (rc = choose_shape(p->kind, p->dim, p->sm_count, std::max<int64_t>(p->sy.rows, 1),
                                           p->sx.pad, p->sy, o.col_splits, o.rows_per_thread)) != OT_OK)
        return rc;
    const int64_t part_cnt = std::max((int64_t)p->sx.splits * p->sx.tiles * p->sx.tile,
                                      (int64_t)p->sy.splits * p->sy.tiles * p->sy.tile);
    const int64_t tiles = std::max(p->sx.tiles, p->sy.tiles);

    for (int pass = 0; pass < 2; ++pass) {
        Carver cv{pass ? p->ws : nullptr};
        p->prm = cv.take<Params>(1);
        p->st = cv.take<State>(1);
        p->o = cv.take<double>(kMaxD);
        p->ds = cv.take<DevScalars>(1);
        p->part1 = cv.take<double>((int64_t)kMaxD * 1024);
        p->part2 = cv.take<double>((int64_t)kMaxD * 1024);
        p->fspare = cv.take<float>(p->n);
        p->sx.rowtab = cv.take<float>(p->sx.pad * p->dp);
        p->sy.rowtab = cv.take<float>(p->sy.pad * p->dp);
        p->sx.coltab = cv.take<float>(p->sx.pad * colw);
        p->sy.coltab = cv.take<float>(p->sy.pad * colw);
        p->sx.arow = cv.take<uint16_t>(p->sx.pad * p->kp);
        p->sx.bcol = cv.take<uint16_t>(p->sx.pad * p->kp);
        p->sy.arow = cv.take<uint16_t>(p->sy.pad * p->kp);
        p->sy.bcol = cv.take<uint16_t>(p->sy.pad * p->kp);
        p->part = cv.take<float2>(part_cnt);
        p->tile_cnt = cv.take<unsigned>(tiles);
        p->tile_resid = cv.take<double>(tiles);
        p->bar = cv.take<unsigned>(2);
        p->blk_resid = cv.take<double>(std::max(p->loop_grid, 1));
        if (pass == 0) OT_CU(pool_device_alloc(reinterpret_cast<void **>(&p->ws), cv.off, &p->ws_bytes));
    }
    if (p->kind == 2) {
        OT_CU(tc_setup(p->d));
        int e = make_operand_map(&p->tm_arow_x, p->sx.arow, p->sx.pad, p->kp);
        if (!e) e = make_operand_map(&p->tm_bcol_y, p->sy.bcol, p->sy.pad, p->kp);
        if (!e) e = make_operand_map(&p->tm_arow_y, p->sy.arow, p->sy.pad, p->kp);
        if (!e) e = make_operand_map(&p->tm_bcol_x, p->sx.bcol, p->sx.pad, p->kp);
        if (e) return fail(OT_ERR_CUDA, "tensor map encoding failed (%d)", e);
    }
    OT_CU(cudaMemsetAsync(p->tile_cnt, 0, sizeof(unsigned) * tiles, p->s_int));
    OT_CU(cudaMemsetAsync(p->bar, 0, sizeof(unsigned) * 2, p->s_int));
    OT_CU(cudaMemsetAsync(p->st, 0, sizeof(State), p->s_int));
    OT_CU(cudaMemsetAsync(p->ds, 0, sizeof(DevScalars), p->s_int));
    return OT_OK;
}

// Input statistics, validation and the coordinate shift o (the midpoint of the
// clouds' means, used by every table); fills p->hs->s with the sums.
int coord_shift(ot_plan *p) {
    DevScalars *ds = p->ds;
    OT_CU(launch_coord_stats(p->x, p->n, p->d, p->part1, p->part2, ds->sums[0], ds->sums[1],
                             &ds->flags[0], nullptr, p->s_int));
    OT_CU(launch_coord_stats(p->y, p->m, p->d, p->part1, p->part2, ds->sums[2], ds->sums[3],
                             &ds->flags[1], nullptr, p->s_int));
    const bool weights = p->a && p->b;  // ot_max_sqdist has none
    if (weights) {
        OT_CU(launch_coord_stats(p->a, p->n, 1, p->part1, p->part2, &ds->wsum[0], &ds->wsum[1],
                                 &ds->flags[2], &ds->zeros[0], p->s_int));
        OT_CU(launch_coord_stats(p->b, p->m, 1, p->part1, p->part2, &ds->wsum[2], &ds->wsum[3],
                                 &ds->flags[3], &ds->zeros[1], p->s_int));
    }
    p->launches += weights ? 8 : 4;
    int rc = read_scalars(p);
    if (rc != OT_OK) return rc;
    const DevScalars &h = p->hs->s;
    if ((h.flags[0] | h.flags[1]) & 1) return fail(OT_ERR_NONFINITE, "x or y holds a NaN or inf");
    if (weights) {
        if ((h.flags[2] | h.flags[3]) & 1) return fail(OT_ERR_NONFINITE, "a or b holds a NaN or inf");
        if ((h.flags[2] | h.flags[3]) & 2) return fail(OT_ERR_INVALID_ARG, "negative weight in a or b");
        if (!(h.wsum[0] > 0.0) || !(h.wsum[2] > 0.0))
            return fail(OT_ERR_INVALID_ARG, "a and b must have positive sums");
    }
    p->n_massless_rows = (int64_t)h.zeros[0];
    p->n_massless_cols = (int64_t)h.zeros[1];
    double dot = 0.0, sxx = 0.0, syy = 0.0;
    for (int k = 0; k < p->d; ++k) {
        const double mx = h.sums[0][k] / (double)p->n, my = h.sums[2][k] / (double)p->m;
        p->hs->o[k] = 0.5 * (mx + my);
        dot += mx * my;
        sxx += h.sums[1][k];
        syy += h.sums[3][k];
    }
    for (int k = p->d; k < kMaxD; ++k) p->hs->o[k] = 0.0;
    OT_CU(cudaMemcpyAsync(p->o, p->hs->o, sizeof(double) * kMaxD, cudaMemcpyHostToDevice, p->s_int));
    p->mean_sq = sxx / (double)p->n + syy / (double)p->m - 2.0 * dot;
    // the stream must not leave before the pinned o[] has been copied
    OT_CU(cudaStreamSynchronize(p->s_int));
    return OT_OK;
}

// The captured scale (after coord_shift): 1, the closed-form mean, the
// all-pairs max_cost pass, or the caller's value.
int resolve_scale(ot_plan *p, ot_scale scale, double scale_value) {
    int rc = coord_shift(p);
    if (rc != OT_OK) return rc;
    DevScalars *ds = p->ds;
    double c = 1.0;
    if (scale == OT_SCALE_MEAN) {
        c = 1.0 / p->mean_sq;
    } else if (scale == OT_SCALE_MAX_COST) {
        OT_CU(launch_max_cost(p->x, p->y, p->n, p->m, p->d, p->o, &ds->max_bits, p->s_int));
        p->launches += 1;
        rc = read_scalars(p);
        if (rc != OT_OK) return rc;
        float mx;
        std::memcpy(&mx, &p->hs->s.max_bits, sizeof mx);
        c = 1.0 / (double)mx;
    } else if (scale == OT_SCALE_VALUE) {
        c = 1.0 / scale_value;
    }
    if (!std::isfinite(c) || !(c > 0.0))
        return fail(OT_ERR_INVALID_ARG, "cost scale is zero or not finite (all points equal?)");
    p->c = c;
    return OT_OK;
}

int validate(const float *x, const float *y, const float *a, const float *b, int64_t n,
             int64_t m, int32_t d, double eps, ot_scale scale, int32_t n_iters, float *f,
             float *g, const ot_options &o) {
    if (!x || !y || !a || !b || !f || !g) return fail(OT_ERR_INVALID_ARG, "null array pointer");
    if (n < 1 || m < 1) return fail(OT_ERR_INVALID_ARG, "n and m must be >= 1 (n=%lld m=%lld)",
                                    (long long)n, (long long)m);
    if (n > INT32_MAX || m > INT32_MAX)
        return fail(OT_ERR_OVERFLOW, "n and m must be < 2^31 (n=%lld m=%lld)", (long long)n,
                    (long long)m);
    if (d < 1 || d > kMaxD) return fail(d < 1 ? OT_ERR_INVALID_ARG : OT_ERR_UNSUPPORTED,
                                        "d=%d outside 1..%d", d, kMaxD);
    if (!(eps > 0.0) || !std::isfinite(eps)) return fail(OT_ERR_INVALID_ARG, "eps must be > 0 and finite");
    if (scale < OT_SCALE_NONE || scale > OT_SCALE_VALUE) return fail(OT_ERR_INVALID_ARG, "bad scale_cost");
    if (scale == OT_SCALE_VALUE && !(o.scale_value > 0.0 && std::isfinite(o.scale_value)))
        return fail(OT_ERR_INVALID_ARG, "scale_value must be > 0 and finite");
    if (n_iters < 0) return fail(OT_ERR_INVALID_ARG, "n_iters must be >= 0");
    if (n_iters == 0 && !o.warm_start)
        return fail(OT_ERR_INVALID_ARG, "n_iters == 0 needs warm_start (a plan at given f, g)");
    if (o.check_every < 1) return fail(OT_ERR_INVALID_ARG, "check_every must be >= 1");
    if (o.resid_history_len < 0 || (o.resid_history_len > 0 && !o.resid_history))
        return fail(OT_ERR_INVALID_ARG, "resid_history_len must be >= 0, with a non-NULL resid_history");
    if (o.sparse_mask_out && !o.block_sparse)
        return fail(OT_ERR_INVALID_ARG, "sparse_mask_out needs block_sparse");
    if (o.col_splits < 0) return fail(OT_ERR_INVALID_ARG, "col_splits must be >= 0");
    if (o.rows_per_thread != 0 && o.rows_per_thread != 1 && o.rows_per_thread != 2 &&
        o.rows_per_thread != 4 && o.rows_per_thread != 8)
        return fail(OT_ERR_INVALID_ARG, "rows_per_thread must be 0, 1, 2, 4 or 8");
    if (o.eps_init > 0.0) {
        if (!(o.eps_decay > 0.0 && o.eps_decay < 1.0)) return fail(OT_ERR_INVALID_ARG, "eps_decay must be in (0,1)");
        if (o.iters_per_stage < 1) return fail(OT_ERR_INVALID_ARG, "iters_per_stage must be >= 1");
    }
    return OT_OK;
}

}  // namespace

extern "C" int ot_sinkhorn_pointcloud(const float *x, const float *y, const float *a,
                                      const float *b, int64_t n, int64_t m, int32_t d, double eps,
                                      ot_scale scale_cost, int32_t n_iters, double tol, float *f,
                                      float *g, void *stream, const ot_options *opt,
                                      ot_plan **plan_out, ot_info *info) {
    NvtxRange nvtx_range("ot_sinkhorn_pointcloud");
    if (plan_out) *plan_out = nullptr;
    ot_options o;
    ot_options_default(&o);
    if (opt) o = *opt;
    int rc = validate(x, y, a, b, n, m, d, eps, scale_cost, n_iters, f, g, o);
    if (rc != OT_OK) return rc;
    const bool sparse = o.block_sparse != 0;
    if (sparse) {
        if (d > 3) return fail(OT_ERR_UNSUPPORTED, "block-sparse iterations need d <= 3");
        if (o.sparse_block != 0 && o.sparse_block != 128 && o.sparse_block != 256)
            return fail(OT_ERR_INVALID_ARG, "sparse_block must be 0, 128 or 256");
        if (!(o.sparse_delta >= 0.0) || !std::isfinite(o.sparse_delta))
            return fail(OT_ERR_INVALID_ARG, "sparse_delta must be >= 0 and finite");
        if (o.sparse_delta == 0.0 && !(tol > 0.0))
            return fail(OT_ERR_INVALID_ARG, "sparse_delta = 0 takes delta from tol, which must be > 0");
        if (!(o.sparse_dense_frac >= 0.0 && o.sparse_dense_frac <= 1.0))
            return fail(OT_ERR_INVALID_ARG, "sparse_dense_frac must be in [0, 1]");
        o.device_loop = 0;  // the mask is rebuilt between every two iterations
    }
    ot_plan *p = new (std::nothrow) ot_plan();
    if (!p) return fail(OT_ERR_OOM, "host allocation failed");
    struct Guard {
        ot_plan *p;
        bool keep = false;
        ~Guard() {
            if (!keep) plan_free(p);
        }
    } guard{p};
    rc = check_device(&p->device, &p->sm_count);
    if (rc != OT_OK) return rc;
    p->x = x; p->y = y; p->a = a; p->b = b; p->f = f; p->g = g;
    p->n = n; p->m = m; p->d = d;
    cudaStream_t us = (cudaStream_t)stream;
    OT_CU(pool_stream(&p->s_int));
    OT_CU(cudaEventCreateWithFlags(&p->ev_in, cudaEventDisableTiming));
    OT_CU(cudaEventCreateWithFlags(&p->ev_out, cudaEventDisableTiming));
    OT_CU(pool_host_alloc(reinterpret_cast<void **>(&p->hs), sizeof(HostScalars)));
    OT_CU(cudaEventRecord(p->ev_in, us));
    OT_CU(cudaStreamWaitEvent(p->s_int, p->ev_in, 0));
    if ((rc = plan_setup(p, o)) != OT_OK) return rc;
    if ((rc = resolve_scale(p, scale_cost, o.scale_value)) != OT_OK) return rc;
    p->sx_pts = x; p->sy_pts = y; p->sa = a; p->sb = b;
    p->sf[0] = f; p->sf[1] = p->fspare; p->sg = g;
    p->asum = p->hs->s.wsum[0];
    p->sparse = sparse;
    if (sparse) {
        if ((rc = sparse_setup(p, o, tol, o.warm_start != 0)) != OT_OK) return rc;
    } else if (!o.warm_start) {
        OT_CU(cudaMemsetAsync(f, 0, sizeof(float) * n, p->s_int));
        OT_CU(cudaMemsetAsync(g, 0, sizeof(float) * m, p->s_int));
    }
    if (o.resid_history_len > 0)  // every entry no f-update measures stays NaN
        OT_CU(cudaMemsetAsync(o.resid_history, 0xff, sizeof(double) * (size_t)o.resid_history_len,
                              p->s_int));
    p->graph_len = std::max(2, (o.check_every + 1) / 2 * 2);
    p->timing = o.timing != 0;

    // eps stages: FlashSinkhorn 2 (sections 3.1, C.3) anneals eps and continues
    // at the target; here stage k runs at max(eps, eps_init * decay^k)
    std::vector<double> stage_eps;
    if (o.eps_init > 0.0) {
        for (int k = 0;; ++k) {
            const double ek = std::max(eps, o.eps_init * std::pow(o.eps_decay, (double)k));
            stage_eps.push_back(ek);
            if (ek == eps || k > 100000) break;
        }
    } else {
        stage_eps.push_back(eps);
    }
    float *const *fb = p->sf;
    const int layout = p->kind == 0 ? 0 : 1;  // CUDA-core paths' column-table layout
    int t = 0, converged = 0;
    int64_t half_steps = 0;
    double resid = NAN;
    for (size_t si = 0; si < stage_eps.size(); ++si) {
        const bool last = si + 1 == stage_eps.size();
        // block-sparse: the admitted plan's residual must leave room for the
        // mass the mask omits (at most sp_bound), so the full residual is <= tol
        const double tol_s = (last && tol > 0.0) ? (sparse ? tol - p->sp_bound : tol) : 0.0;
        const int iters = last ? n_iters : o.iters_per_stage;
        OT_CU(launch_set_params(p->prm, stage_eps[si], p->c, tol_s, o.resid_history, (int64_t)t,
                                o.resid_history_len, p->s_int));
        OT_CU(launch_reset_state(p->st, p->s_int));
        if (p->kind == 2) {
            OT_CU(launch_tc_tables(x, fb[t & 1], n, p->sx.pad, d, p->dp, p->kp, p->o, p->prm,
                                   p->sx.rowtab, p->sx.arow, p->sx.bcol, p->s_int));
            OT_CU(launch_tc_tables(y, g, m, p->sy.pad, d, p->dp, p->kp, p->o, p->prm,
                                   p->sy.rowtab, p->sy.arow, p->sy.bcol, p->s_int));
        } else {
            OT_CU(launch_tables(p->sx_pts, fb[t & 1], n, p->sx.pad, d, p->dp, p->o, p->prm,
                                p->sx.rowtab, p->sx.coltab, layout, p->s_int));
            OT_CU(launch_tables(p->sy_pts, p->sg, m, p->sy.pad, d, p->dp, p->o, p->prm,
                                p->sy.rowtab, p->sy.coltab, layout, p->s_int));
        }
        p->launches += 4;
        rc = sparse ? run_sparse(p, t & 1, iters, stage_eps[si], tol_s > 0.0 ? o.check_every : iters)
                    : run_iterations(p, t & 1, iters, tol_s > 0.0, o.use_graphs != 0);
        if (rc != OT_OK) return rc;
        if ((rc = read_state(p)) != OT_OK) return rc;
        if (p->hs->st.wait_timeout)
            return fail(OT_ERR_CUDA, "a bounded device wait (grid barrier or tensor-core pipeline) "
                                     "timed out; results invalid");
        const int done = p->hs->st.stop ? p->hs->st.conv_iter : iters;
        t += done;
        half_steps += 2 * (int64_t)done + (p->hs->st.stop ? 1 : 0);
        if (last) {
            if (p->hs->st.stop) {
                converged = 1;
                resid = p->hs->st.resid[0];
            } else if (iters > 0) {
                // one more f-update measures ||T1 - a||_1 of the final state
                OT_CU(mark(p));
                if (sparse) {
                    if ((rc = sparse_iteration(p, t & 1, true, stage_eps[si])) != OT_OK) return rc;
                } else {
                    OT_CU(launch_side(p, 0, t & 1));
                    p->launches += 1;
                }
                OT_CU(mark(p));
                half_steps += 1;
                if ((rc = read_state(p)) != OT_OK) return rc;
                resid = p->hs->st.resid[0];
                converged = p->hs->st.stop;
            }
        }
    }
    int64_t sp_it = 0, dn_it = 0;
    if (sparse) {
        OT_CU(cudaMemcpyAsync(&p->hs->sc, p->sc, sizeof(SparseCtr), cudaMemcpyDeviceToHost, p->s_int));
        OT_CU(cudaStreamSynchronize(p->s_int));
        const SparseCtr &sc = p->hs->sc;
        // the counters hold the last screened mask: of the last iteration that ran
        const int kindm = sc.mode[0] == kModeStopped ? sc.mode[1] : sc.mode[0];
        p->last_cand = (int64_t)sc.cand;
        p->last_adm = (kindm == kModeDense || !p->sp_verify) ? (int64_t)sc.cand : (int64_t)sc.adm;
        p->last_exact = kindm == kModeDense ? 0 : (int64_t)sc.exact;
        // iterations of the returned state: the one whose f-update met the stop test
        // was counted but not completed
        sp_it = (int64_t)sc.n_mode[kModeSparse];
        dn_it = (int64_t)sc.n_mode[kModeDense];
        const int64_t excess = sp_it + dn_it - (int64_t)t;
        if (excess > 0) (sc.mode[1] == kModeDense ? dn_it : sp_it) -= excess;
    }
    if (sparse) {  // back to the caller's order
        OT_CU(launch_scatter(p->sf[t & 1], p->perm_x, n, p->f, p->s_int));
        OT_CU(launch_scatter(p->sg, p->perm_y, m, p->g, p->s_int));
        p->launches += 2;
    } else if (t & 1) {
        OT_CU(cudaMemcpyAsync(p->f, p->fspare, sizeof(float) * n, cudaMemcpyDeviceToDevice, p->s_int));
    }
    if ((rc = read_state(p)) != OT_OK) return rc;
    if (p->hs->st.wait_timeout)
        return fail(OT_ERR_CUDA, "a bounded device wait (grid barrier or tensor-core pipeline) "
                                 "timed out; results invalid");
    if (p->hs->st.nonfinite)
        return fail(OT_ERR_NONFINITE, "a potential left the finite range (eps too small for float32?)");
    p->eps = stage_eps.back();
    double loop_ms = 0.0;
    for (size_t e = 0; e + 1 < p->tev_used; e += 2) {
        float ms = 0.0f;
        OT_CU(cudaEventElapsedTime(&ms, p->tev[e], p->tev[e + 1]));
        loop_ms += ms;
    }
    OT_CU(cudaEventRecord(p->ev_out, p->s_int));
    OT_CU(cudaStreamWaitEvent(us, p->ev_out, 0));
    if (info) {
        info->iterations = t;
        info->converged = converged;
        info->stages = (int32_t)stage_eps.size();
        info->col_splits = p->sx.splits;
        info->residual = resid;
        info->inv_scale_cost = p->c;
        info->eps = p->eps;
        info->n_massless_rows = p->n_massless_rows;
        info->n_massless_cols = p->n_massless_cols;
        info->half_steps = half_steps;
        info->kernel_launches = p->launches;
        info->loop_ms = loop_ms;
        info->sparse_iterations = sp_it;
        info->dense_iterations = dn_it;
        info->tiles_candidate = p->last_cand;
        info->tiles_admitted = p->last_adm;
        info->tiles_exact = p->last_exact;
        info->tiles_total = sparse ? p->sp_nb * p->sp_mb : 0;
        info->omitted_bound = sparse ? p->sp_bound : 0.0;
        if ((rc = sum_marks(p->tm_verify, &info->verify_ms)) != OT_OK) return rc;
        if ((rc = sum_marks(p->tm_hs, &info->sparse_hs_ms)) != OT_OK) return rc;
        info->sparse_hs_launches = (int64_t)(p->tm_hs.used / 2);
    }
    if (plan_out) {
        *plan_out = p;
        guard.keep = true;
    }
    if (p->n_massless_rows > 0) {
        fail(OT_WARN_MASSLESS_ROWS, "%lld rows carry no mass", (long long)p->n_massless_rows);
        return OT_WARN_MASSLESS_ROWS;
    }
    return OT_OK;
}

extern "C" int ot_sinkhorn_pointcloud_host(const float *x, const float *y, const float *a,
                                           const float *b, int64_t n, int64_t m, int32_t d,
                                           double eps, ot_scale scale_cost, int32_t n_iters,
                                           double tol, float *f, float *g, void *stream,
                                           const ot_options *opt, ot_plan **plan_out,
                                           ot_info *info) {
    NvtxRange nvtx_range("ot_sinkhorn_pointcloud_host");
    if (plan_out) *plan_out = nullptr;
    if (!x || !y || !a || !b || !f || !g) return fail(OT_ERR_INVALID_ARG, "null array pointer");
    if (n < 1 || m < 1 || n > INT32_MAX || m > INT32_MAX || d < 1 || d > kMaxD)
        return fail(n > INT32_MAX || m > INT32_MAX ? OT_ERR_OVERFLOW
                    : d > kMaxD                    ? OT_ERR_UNSUPPORTED
                                                   : OT_ERR_INVALID_ARG,
                    "bad sizes (n=%lld m=%lld d=%d)", (long long)n, (long long)m, d);
    int dev = 0, sms = 0;
    int rc = check_device(&dev, &sms);
    if (rc != OT_OK) return rc;
    const bool warm = opt && opt->warm_start;
    cudaStream_t s = (cudaStream_t)stream;
    // device copies of x, y, a, b, f, g in one pooled buffer
    float *dx = nullptr, *dy = nullptr, *da = nullptr, *db = nullptr, *df = nullptr, *dg = nullptr;
    char *buf = nullptr;
    size_t got = 0;
    for (int pass = 0; pass < 2; ++pass) {
        Carver cv{pass ? buf : nullptr};
        dx = cv.take<float>(n * d);
        dy = cv.take<float>(m * d);
        da = cv.take<float>(n);
        db = cv.take<float>(m);
        df = cv.take<float>(n);
        dg = cv.take<float>(m);
        if (pass == 0) OT_CU(pool_device_alloc(reinterpret_cast<void **>(&buf), cv.off, &got));
    }
    struct Release {
        char *buf;
        size_t got;
        int dev;
        cudaStream_t s;
        ~Release() {
            if (buf) {
                cudaStreamSynchronize(s);  // no copy may still use it
                pool_device_free(buf, got, dev);
            }
        }
    } rel{buf, got, dev, s};
    cudaError_t e = cudaSuccess;
    const struct { void *dst; const void *src; size_t bytes; } in[] = {
        {dx, x, sizeof(float) * (size_t)(n * d)}, {dy, y, sizeof(float) * (size_t)(m * d)},
        {da, a, sizeof(float) * (size_t)n},       {db, b, sizeof(float) * (size_t)m},
        {df, f, warm ? sizeof(float) * (size_t)n : 0}, {dg, g, warm ? sizeof(float) * (size_t)m : 0}};
    for (const auto &c : in)
        if (e == cudaSuccess && c.bytes) e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return fail(OT_ERR_CUDA, "host-to-device copy failed: %s", cudaGetErrorString(e));
    ot_plan *plan = nullptr;
    rc = ot_sinkhorn_pointcloud(dx, dy, da, db, n, m, d, eps, scale_cost, n_iters, tol, df, dg, stream,
                                opt, &plan, info);
    if (rc < 0) return rc;
    e = cudaMemcpyAsync(f, df, sizeof(float) * (size_t)n, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(g, dg, sizeof(float) * (size_t)m, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        plan_free(plan);
        return fail(OT_ERR_CUDA, "device-to-host copy failed: %s", cudaGetErrorString(e));
    }
    if (plan_out) {  // the plan keeps the device copies it reads
        plan->ws_in = buf;
        plan->ws_in_bytes = got;
        rel.buf = nullptr;
        *plan_out = plan;
    } else {
        plan_free(plan);
    }
    if (rc == OT_WARN_MASSLESS_ROWS) fail(OT_WARN_MASSLESS_ROWS, "some rows carry no mass");
    return rc;
}

// ------------------------------------------------------------ sharded solve
// The solve split by rows across ranks (FlashSinkhorn 2, section 5: problems
// beyond one GPU's memory run on several): every rank holds both clouds in
// full and updates a contiguous range of x's rows in the f-update and of y's in
// the g-update; the caller exchanges the updated potential ranges between the
// half-steps (an all-gather) and sums the residual partials (an all-reduce).

extern "C" int ot_max_sqdist(const float *x, const float *y, int64_t n, int64_t m, int32_t d,
                             int64_t x_lo, int64_t x_hi, float *out, void *stream) {
    NvtxRange nvtx_range("ot_max_sqdist");
    if (!x || !y || !out) return fail(OT_ERR_INVALID_ARG, "null pointer");
    if (n < 1 || m < 1 || d < 1 || d > kMaxD)
        return fail(d > kMaxD ? OT_ERR_UNSUPPORTED : OT_ERR_INVALID_ARG, "bad sizes");
    if (n > INT32_MAX || m > INT32_MAX) return fail(OT_ERR_OVERFLOW, "n and m must be < 2^31");
    if (x_lo < 0 || x_hi > n || x_lo > x_hi) return fail(OT_ERR_INVALID_ARG, "bad row range");
    // a plan without iterations supplies the shift o (the same as every solve's)
    // and the pass's scratch; its own scale resolution is skipped
    ot_options o;
    ot_options_default(&o);
    o.device_loop = 0;
    ot_plan *p = new (std::nothrow) ot_plan();
    if (!p) return fail(OT_ERR_OOM, "host allocation failed");
    struct Guard {
        ot_plan *p;
        ~Guard() { plan_free(p); }
    } guard{p};
    int rc = check_device(&p->device, &p->sm_count);
    if (rc != OT_OK) return rc;
    p->x = x; p->y = y; p->n = n; p->m = m; p->d = d;
    p->shard = true;  // no half-step shapes are needed: an empty range
    cudaStream_t us = (cudaStream_t)stream;
    OT_CU(pool_stream(&p->s_int));
    OT_CU(cudaEventCreateWithFlags(&p->ev_in, cudaEventDisableTiming));
    OT_CU(cudaEventCreateWithFlags(&p->ev_out, cudaEventDisableTiming));
    OT_CU(pool_host_alloc(reinterpret_cast<void **>(&p->hs), sizeof(HostScalars)));
    OT_CU(cudaEventRecord(p->ev_in, us));
    OT_CU(cudaStreamWaitEvent(p->s_int, p->ev_in, 0));
    if ((rc = plan_setup(p, o)) != OT_OK) return rc;
    if ((rc = coord_shift(p)) != OT_OK) return rc;
    unsigned bits = 0;
    if (x_hi > x_lo) {
        OT_CU(cudaMemsetAsync(&p->ds->max_bits, 0, sizeof(unsigned), p->s_int));
        OT_CU(launch_max_cost(x + x_lo * d, y, x_hi - x_lo, m, d, p->o, &p->ds->max_bits, p->s_int));
        if ((rc = read_scalars(p)) != OT_OK) return rc;
        bits = p->hs->s.max_bits;
    }
    std::memcpy(out, &bits, sizeof bits);
    OT_CU(cudaEventRecord(p->ev_out, p->s_int));
    OT_CU(cudaStreamWaitEvent(us, p->ev_out, 0));
    return OT_OK;
}

extern "C" int ot_shard_plan_create(const float *x, const float *y, const float *a, const float *b,
                                    int64_t n, int64_t m, int32_t d, double eps, ot_scale scale_cost,
                                    int64_t x_lo, int64_t x_hi, int64_t y_lo, int64_t y_hi,
                                    void *stream, const ot_options *opt, ot_plan **plan_out,
                                    ot_info *info) {
    NvtxRange nvtx_range("ot_shard_plan_create");
    if (!plan_out) return fail(OT_ERR_INVALID_ARG, "plan_out must not be NULL");
    *plan_out = nullptr;
    ot_options o;
    ot_options_default(&o);
    if (opt) o = *opt;
    o.device_loop = 0;
    o.warm_start = 1;
    float dummy = 0.0f;
    int rc = validate(x, y, a, b, n, m, d, eps, scale_cost, 1, &dummy, &dummy, o);
    if (rc != OT_OK) return rc;
    if (o.block_sparse) return fail(OT_ERR_UNSUPPORTED, "a sharded plan runs dense half-steps");
    if (x_lo < 0 || x_hi > n || x_lo > x_hi || y_lo < 0 || y_hi > m || y_lo > y_hi)
        return fail(OT_ERR_INVALID_ARG, "row ranges must satisfy 0 <= lo <= hi <= n (m)");
    if ((x_lo | y_lo) & (kColPad - 1))
        return fail(OT_ERR_INVALID_ARG, "x_lo and y_lo must be multiples of %d", kColPad);
    ot_plan *p = new (std::nothrow) ot_plan();
    if (!p) return fail(OT_ERR_OOM, "host allocation failed");
    struct Guard {
        ot_plan *p;
        bool keep = false;
        ~Guard() {
            if (!keep) plan_free(p);
        }
    } guard{p};
    rc = check_device(&p->device, &p->sm_count);
    if (rc != OT_OK) return rc;
    p->x = x; p->y = y; p->a = a; p->b = b;
    p->n = n; p->m = m; p->d = d;
    p->shard = true;
    p->range[0][0] = x_lo; p->range[0][1] = x_hi;
    p->range[1][0] = y_lo; p->range[1][1] = y_hi;
    cudaStream_t us = (cudaStream_t)stream;
    OT_CU(pool_stream(&p->s_int));
    OT_CU(cudaEventCreateWithFlags(&p->ev_in, cudaEventDisableTiming));
    OT_CU(cudaEventCreateWithFlags(&p->ev_out, cudaEventDisableTiming));
    OT_CU(pool_host_alloc(reinterpret_cast<void **>(&p->hs), sizeof(HostScalars)));
    OT_CU(cudaEventRecord(p->ev_in, us));
    OT_CU(cudaStreamWaitEvent(p->s_int, p->ev_in, 0));
    if ((rc = plan_setup(p, o)) != OT_OK) return rc;
    if ((rc = resolve_scale(p, scale_cost, o.scale_value)) != OT_OK) return rc;
    p->sx_pts = x; p->sy_pts = y; p->sa = a; p->sb = b;
    p->eps = eps;
    // no tol: the caller decides when to stop from the summed residual
    OT_CU(launch_set_params(p->prm, eps, p->c, 0.0, nullptr, 0, 0, p->s_int));
    OT_CU(launch_reset_state(p->st, p->s_int));
    // both clouds' row tables (the coordinates); each half-step rebuilds the other
    // cloud's column terms from its potential (the weights stand in until then)
    if (p->kind == 2) {
        OT_CU(launch_tc_tables(x, a, n, p->sx.pad, d, p->dp, p->kp, p->o, p->prm, p->sx.rowtab, p->sx.arow,
                               p->sx.bcol, p->s_int));
        OT_CU(launch_tc_tables(y, b, m, p->sy.pad, d, p->dp, p->kp, p->o, p->prm, p->sy.rowtab, p->sy.arow,
                               p->sy.bcol, p->s_int));
    } else {
        const int layout = p->kind == 0 ? 0 : 1;
        OT_CU(launch_tables(x, a, n, p->sx.pad, d, p->dp, p->o, p->prm, p->sx.rowtab, p->sx.coltab, layout,
                            p->s_int));
        OT_CU(launch_tables(y, b, m, p->sy.pad, d, p->dp, p->o, p->prm, p->sy.rowtab, p->sy.coltab, layout,
                            p->s_int));
    }
    OT_CU(cudaEventRecord(p->ev_out, p->s_int));
    OT_CU(cudaStreamWaitEvent(us, p->ev_out, 0));
    OT_CU(cudaStreamSynchronize(p->s_int));
    if (info) {
        std::memset(info, 0, sizeof *info);
        info->col_splits = p->sx.splits;
        info->inv_scale_cost = p->c;
        info->eps = eps;
        info->n_massless_rows = p->n_massless_rows;
        info->n_massless_cols = p->n_massless_cols;
    }
    guard.keep = true;
    *plan_out = p;
    return OT_OK;
}

extern "C" int ot_shard_half_step(ot_plan *p, int32_t side, const float *other, const float *cur,
                                  float *out, double *resid, void *stream) {
    NvtxRange nvtx_range("ot_shard_half_step");
    if (!p || !p->shard || !p->prm) return fail(OT_ERR_INVALID_ARG, "not a sharded plan");
    if (side != 0 && side != 1) return fail(OT_ERR_INVALID_ARG, "side must be 0 (f) or 1 (g)");
    if (!other || !cur || !out) return fail(OT_ERR_INVALID_ARG, "null potential pointer");
    int dev = -1;
    OT_CU(cudaGetDevice(&dev));
    if (dev != p->device) return fail(OT_ERR_INVALID_ARG, "plan belongs to device %d, current is %d", p->device, dev);
    cudaStream_t us = (cudaStream_t)stream;
    OT_CU(cudaEventRecord(p->ev_in, us));
    OT_CU(cudaStreamWaitEvent(p->s_int, p->ev_in, 0));
    // the other cloud's column table from its whole potential (all ranks' rows)
    const bool f = side == 0;
    Side &cols = f ? p->sy : p->sx;
    const float *cpts = f ? p->y : p->x;
    if (p->kind == 2) {
        OT_CU(launch_tc_tables(cpts, other, cols.cnt, cols.pad, p->d, p->dp, p->kp, p->o, p->prm,
                               cols.rowtab, cols.arow, cols.bcol, p->s_int));
    } else {
        OT_CU(launch_tables(cpts, other, cols.cnt, cols.pad, p->d, p->dp, p->o, p->prm, cols.rowtab,
                            cols.coltab, p->kind == 0 ? 0 : 1, p->s_int));
    }
    const Side &rows = f ? p->sx : p->sy;
    if (rows.rows > 0) {
        // the half-step over this plan's rows: old potential `cur`, new one into `out`
        float *save[3] = {p->sf[0], p->sf[1], p->sg};
        p->sf[0] = const_cast<float *>(cur);
        p->sf[1] = out;
        p->sg = out;  // g-update: pot_old and pot_new both come from sg
        HalfStep A = make_step(p, side, 0);
        if (!f) A.pot_old = cur + rows.lo;
        p->sf[0] = save[0]; p->sf[1] = save[1]; p->sg = save[2];
        cudaError_t e = p->kind == 2
            ? launch_halfstep_tc(p->d, A, f ? &p->tm_arow_x : &p->tm_arow_y, f ? &p->tm_bcol_y : &p->tm_bcol_x,
                                 rows.grid, p->s_int)
            : launch_halfstep(p->kind, p->dim, rows.rpt, A, rows.grid, p->s_int);
        if (e != cudaSuccess) return fail(OT_ERR_CUDA, "half-step launch failed: %s", cudaGetErrorString(e));
    }
    OT_CU(cudaEventRecord(p->ev_out, p->s_int));
    OT_CU(cudaStreamWaitEvent(us, p->ev_out, 0));
    if (resid || rows.rows > 0) {
        int rc = read_state(p);
        if (rc != OT_OK) return rc;
        if (p->hs->st.wait_timeout)
            return fail(OT_ERR_CUDA, "a bounded device wait timed out; results invalid");
        if (p->hs->st.nonfinite) return fail(OT_ERR_NONFINITE, "a potential left the finite range");
        if (resid) *resid = rows.rows > 0 ? p->hs->st.resid[side] : 0.0;
    }
    return OT_OK;
}

namespace {

int plan_check(const ot_plan *p) {
    if (!p) return fail(OT_ERR_INVALID_ARG, "null plan");
    if (p->shard) return fail(OT_ERR_INVALID_ARG, "a sharded plan serves ot_shard_half_step only");
    int dev = -1;
    OT_CU(cudaGetDevice(&dev));
    if (dev != p->device) return fail(OT_ERR_INVALID_ARG, "plan belongs to device %d, current is %d", p->device, dev);
    return OT_OK;
}

// Workspace of the row kernels, allocated on first use and kept by the plan.
int ensure_rows_ws(ot_plan *p) {
    if (p->ws_rows) return OT_OK;
    const int64_t big = std::max(p->n, p->m);
    for (int pass = 0; pass < 2; ++pass) {
        Carver cv{pass ? p->ws_rows : nullptr};
        p->dcol = cv.take<double>(big * (p->d + 1));
        p->rpart = cv.take<double>(rowpass_blocks(big, p->d));
        p->rowmax = cv.take<float>(p->n);
        p->counts = cv.take<int64_t>(p->n);
        p->scan = cv.take<int64_t>(scan_tmp_count(p->n));
        if (p->d <= 3) {
            p->mperm[0] = cv.take<int64_t>(p->n);
            p->mperm[1] = cv.take<int64_t>(p->m);
            p->rperm = cv.take<int64_t>(big);
            p->rkeys = cv.take<unsigned long long>(next_pow2(big));
            p->csum = cv.take<double>(7 * chunk_count(big));
            p->rlohi = cv.take<unsigned>(6);
        }
        if (pass == 0)
            OT_CU(pool_device_alloc(reinterpret_cast<void **>(&p->ws_rows), cv.off, &p->ws_rows_bytes));
    }
    return OT_OK;
}

// Rows one launch of a row pass covers: the caller's block (0 = all rows), but
// never fewer than sixteen waves of the row-pass blocks (3 per SM) -- a block
// of rows changes no result (every row is reduced within one thread block), so
// a small block would only add launch tails: with the tile screen the blocks'
// work varies with where their rows lie (measured at workload 5, blocks of
// 4096 rows: min_row 1.72 s with launches of four waves, 1.56 s in one launch).
int64_t launch_rows(const ot_plan *p, int64_t block_rows) {
    const int64_t min_rows = rowpass_rows_per_block(p->d) * 3 * 16 * std::max(p->sm_count, 1);
    if (block_rows == 0 || block_rows > p->n) return p->n;
    return std::min(p->n, std::max(block_rows, min_rows));
}

int sync_read(ot_plan *p, cudaStream_t s) {
    OT_CU(cudaMemcpyAsync(&p->hs->s, p->ds, sizeof(DevScalars), cudaMemcpyDeviceToHost, s));
    OT_CU(cudaStreamSynchronize(s));
    p->screen_visited = (int64_t)p->hs->s.visited;
    return OT_OK;
}

RowPassArgs row_args(const ot_plan *p) {
    RowPassArgs R{};
    R.pts = p->x; R.pot = p->f; R.w = p->a; R.dcol = p->dcol; R.o = p->o; R.prm = p->prm;
    R.cols = p->m; R.d = p->d; R.rowmax = p->rowmax; R.counts = p->counts; R.part = p->rpart;
    R.visited = p->d <= 3 ? &p->ds->visited : nullptr;
    return R;
}

// Start of a row call: zero its chunk statistics.
int screen_reset(ot_plan *p, cudaStream_t s) {
    OT_CU(cudaMemsetAsync(&p->ds->visited, 0, sizeof(unsigned long long), s));
    p->screen_total = 0;
    return OT_OK;
}

// Chunks a full visit of positions [p0, p1) against `cols` columns evaluates.
void screen_count(ot_plan *p, int64_t p0, int64_t p1, int64_t cols) {
    if (p->d <= 3 && p1 > p0) p->screen_total += rowpass_blocks(p1 - p0, p->d) * chunk_count(cols);
}

// Morton order (30-bit codes over the cloud's own bounding box, the point
// index breaking ties) of points [lo, hi) of cloud `cl` (0: x, 1: y) into perm
// (indices of the cloud).
int morton_order(ot_plan *p, int cl, int64_t lo, int64_t hi, int64_t *perm, cudaStream_t s) {
    const float *pts = cl ? p->y : p->x;
    const int64_t cnt = cl ? p->m : p->n;
    const int d = p->d;
    if (!p->mort_ready[cl]) {
        OT_CU(cudaMemsetAsync(p->rlohi, 0xff, 3 * sizeof(unsigned), s));
        OT_CU(cudaMemsetAsync(p->rlohi + 3, 0, 3 * sizeof(unsigned), s));
        OT_CU(launch_box(pts, cnt, d, p->rlohi, s));
        unsigned h[6];
        OT_CU(cudaMemcpyAsync(h, p->rlohi, sizeof h, cudaMemcpyDeviceToHost, s));
        OT_CU(cudaStreamSynchronize(s));
        MortonArgs &M = p->mort[cl];
        M = MortonArgs{};
        M.d = d;
        M.bits = 30 / d;
        const double cells = (double)(1ll << M.bits);
        for (int k = 0; k < d; ++k) {
            const double blo = (double)float_from_order(h[k]), bhi = (double)float_from_order(h[3 + k]);
            M.lo[k] = blo;
            M.s[k] = bhi > blo ? cells / (bhi - blo) : 0.0;
        }
        p->mort_ready[cl] = true;
    }
    const int64_t k = hi - lo;
    if (k <= 0) return OT_OK;
    OT_CU(launch_morton_sort(pts + lo * d, k, next_pow2(k), p->mort[cl], p->rkeys, s));
    OT_CU(launch_perm_from_keys(p->rkeys, k, lo, perm, s));
    return OT_OK;
}

// The rows a pass visits and the column table it reads. For d <= 3 the
// columns (the other cloud) are put in Morton order with their chunk
// summaries, and rows [lo, hi) of the pass's cloud (`side` 0: x, 1: y) are
// visited in Morton order, positions [0, hi - lo); `screen` lets the kernel
// skip the chunks whose entries all vanish. Otherwise the columns keep their
// order and positions are the rows themselves.
struct PassRows {
    const int64_t *rperm = nullptr;
    const double *csum = nullptr;
    int64_t p0 = 0, p1 = 0;
};

int pass_setup(ot_plan *p, int side, int64_t lo, int64_t hi, bool screen, cudaStream_t s, PassRows &pr) {
    const float *cpts = side ? p->x : p->y, *cpot = side ? p->f : p->g;
    const int64_t ccnt = side ? p->n : p->m, rcnt = side ? p->m : p->n;
    if (p->d > 3) {
        OT_CU(launch_dcol(cpts, cpot, ccnt, p->d, p->o, p->prm, p->dcol, s));
        pr = PassRows{nullptr, nullptr, lo, hi};
        return OT_OK;
    }
    int rc = OT_OK;
    for (int cl = 0; cl < 2; ++cl) {
        if (p->mperm_ready[cl]) continue;
        if ((rc = morton_order(p, cl, 0, cl ? p->m : p->n, p->mperm[cl], s)) != OT_OK) return rc;
        p->mperm_ready[cl] = true;
    }
    OT_CU(launch_dcol(cpts, cpot, ccnt, p->d, p->o, p->prm, p->dcol, s, p->mperm[side ^ 1]));
    OT_CU(launch_chunk_summary(p->dcol, ccnt, p->d, p->prm, p->csum, s));
    const int64_t *rperm = p->mperm[side];
    if (lo != 0 || hi != rcnt) {
        if ((rc = morton_order(p, side, lo, hi, p->rperm, s)) != OT_OK) return rc;
        rperm = p->rperm;
    }
    pr = PassRows{rperm, screen ? p->csum : nullptr, 0, hi - lo};
    return OT_OK;
}

// min_row pass A over rows [lo, hi): max_j T_ij of every row, then the
// minimum over the massful ones (thr, its smallest row index, -1 if none) and
// the number of massless rows. pr from pass_setup(side 0, lo, hi).
int min_row_pass(ot_plan *p, int64_t lo, int64_t hi, const PassRows &pr, int64_t block_rows,
                 cudaStream_t s, float *thr, int64_t *argmin, int64_t *n_massless) {
    RowPassArgs R = row_args(p);
    R.rperm = pr.rperm;
    R.csum = pr.csum;
    for (int64_t r0 = pr.p0; r0 < pr.p1; r0 += block_rows) {
        R.row_begin = r0;
        R.row_end = std::min(pr.p1, r0 + block_rows);
        OT_CU(launch_rowpass(0, R, s));
        screen_count(p, R.row_begin, R.row_end, R.cols);
    }
    OT_CU(launch_min_row_reduce(p->rowmax + lo, p->a + lo, hi - lo, &p->ds->thr, &p->ds->argmin,
                                &p->ds->n_massless, s));
    int rc = sync_read(p, s);
    if (rc != OT_OK) return rc;
    *thr = p->hs->s.thr;
    *argmin = p->hs->s.argmin >= 0 ? p->hs->s.argmin + lo : -1;
    *n_massless = p->hs->s.n_massless;
    return OT_OK;
}

// min_row pass B over rows [lo, hi): counts[i] = #{j : T_ij >= thr} (0 for a
// massless row), indexed by the row, and their sum. The tile screen applies
// only at thr > 0 (below, the vanishing entries count too).
int count_pass(ot_plan *p, int64_t lo, int64_t hi, const PassRows &pr, int64_t block_rows,
               float thr, int64_t *counts, cudaStream_t s, int64_t *nnz) {
    RowPassArgs R = row_args(p);
    R.thr = thr;
    R.counts = counts;
    R.rperm = pr.rperm;
    R.csum = thr > 0.0f ? pr.csum : nullptr;
    for (int64_t r0 = pr.p0; r0 < pr.p1; r0 += block_rows) {
        R.row_begin = r0;
        R.row_end = std::min(pr.p1, r0 + block_rows);
        OT_CU(launch_rowpass(1, R, s));
        screen_count(p, R.row_begin, R.row_end, R.cols);
    }
    OT_CU(launch_sum_i64(counts + lo, hi - lo, &p->ds->nnz, s));
    int rc = sync_read(p, s);
    if (rc != OT_OK) return rc;
    *nnz = p->hs->s.nnz;
    return OT_OK;
}

// One side of the marginal residual over rows [lo, hi) of that side:
// sum_i |sum_j T_ij - w_i| (side 0: rows of x against a; side 1: rows of y
// against b, the pass with the clouds' roles swapped). Rebuilds the column
// table of the other side; the result lands in p->ds->r_sum[side].
int residual_pass(ot_plan *p, int side, int64_t lo, int64_t hi, cudaStream_t s) {
    PassRows pr;
    int rc = pass_setup(p, side, lo, hi, true, s, pr);
    if (rc != OT_OK) return rc;
    RowPassArgs R = row_args(p);
    if (side == 1) {
        R.pts = p->y; R.pot = p->g; R.w = p->b; R.cols = p->n;
    }
    R.rperm = pr.rperm;
    R.csum = pr.csum;
    R.row_begin = pr.p0;
    R.row_end = pr.p1;
    OT_CU(launch_rowpass(2, R, s));
    screen_count(p, R.row_begin, R.row_end, R.cols);
    OT_CU(launch_sum_f64(p->rpart, rowpass_blocks(hi - lo, p->d), &p->ds->r_sum[side], s));
    return OT_OK;
}

int range_check(int64_t lo, int64_t hi, int64_t count, const char *what) {
    if (lo < 0 || hi < lo || hi > count)
        return fail(OT_ERR_INVALID_ARG, "%s range [%lld, %lld) is not inside [0, %lld)", what,
                    (long long)lo, (long long)hi, (long long)count);
    return OT_OK;
}

}  // namespace

extern "C" int ot_materialize_rows(const ot_plan *cplan, const int64_t *row_idx, int64_t k,
                                   float *out, void *stream) {
    NvtxRange nvtx_range("ot_materialize_rows");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if (k < 0) return fail(OT_ERR_INVALID_ARG, "k must be >= 0");
    if (k == 0) return OT_OK;
    if (!row_idx || !out) return fail(OT_ERR_INVALID_ARG, "null row_idx or out");
    if (k > INT64_MAX / p->m) return fail(OT_ERR_OVERFLOW, "k*m overflows int64");
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    OT_CU(cudaMemsetAsync(&p->ds->bad, 0, sizeof(int), s));
    OT_CU(launch_dcol(p->y, p->g, p->m, p->d, p->o, p->prm, p->dcol, s));
    MatArgs M{};
    M.x = p->x; M.f = p->f; M.dcol = p->dcol; M.o = p->o; M.prm = p->prm;
    M.row_idx = row_idx; M.k = k; M.n = p->n; M.m = p->m; M.d = p->d;
    M.vec = (p->m % 4 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
    M.out = out;
    M.bad = &p->ds->bad;
    OT_CU(launch_materialize(M, s));
    if ((rc = sync_read(p, s)) != OT_OK) return rc;
    if (p->hs->s.bad) return fail(OT_ERR_INVALID_ARG, "a row index is outside [0, n)");
    return OT_OK;
}

namespace {

// The two low-rank row flavours: no plan, the factors are the output's own.
int lowrank_rows(int mode, const float *fa, const float *fb, const float *g, const float *f,
                 const float *gp, int64_t n, int64_t m, int32_t r, double bias, double c, double eps,
                 const int64_t *row_idx, int64_t k, float *out, void *stream) {
    if (n < 1 || m < 1) return fail(OT_ERR_INVALID_ARG, "n and m must be >= 1");
    if (r < 1 || r > kLrMaxRank) return fail(OT_ERR_UNSUPPORTED, "rank r must be in [1, %d]", kLrMaxRank);
    if (k < 0) return fail(OT_ERR_INVALID_ARG, "k must be >= 0");
    if (!fa || !fb || (mode == 0 ? !g : (!f || !gp)))
        return fail(OT_ERR_INVALID_ARG, "null factor or potential pointer");
    if (mode == 1 && (!(eps > 0.0) || !std::isfinite(eps) || !std::isfinite(c) || !std::isfinite(bias)))
        return fail(OT_ERR_INVALID_ARG, "eps must be > 0 and eps, inv_scale_cost, bias finite");
    if (k == 0) return OT_OK;
    if (!row_idx || !out) return fail(OT_ERR_INVALID_ARG, "null row_idx or out");
    if (k > INT64_MAX / m) return fail(OT_ERR_OVERFLOW, "k*m overflows int64");
    int dev = 0, sms = 0;
    int rc = check_device(&dev, &sms);
    if (rc != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    int *flag = nullptr, *hflag = nullptr;
    size_t got = 0;
    OT_CU(pool_device_alloc(reinterpret_cast<void **>(&flag), 256, &got));
    if (pool_host_alloc(reinterpret_cast<void **>(&hflag), sizeof(int)) != cudaSuccess) {
        pool_device_free(flag, got, dev);
        return fail(OT_ERR_OOM, "pinned host allocation failed");
    }
    LrArgs L{};
    L.fa = fa; L.fb = fb; L.g = g; L.f = f; L.gp = gp;
    L.n = n; L.m = m; L.k = k; L.r = r; L.row_idx = row_idx;
    const double kappa = 1.4426950408889634 / eps;  // log2(e) / eps
    L.bias = bias; L.kappa = kappa; L.kc = kappa * c;
    L.out = out;
    L.vec = (m % 4 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
    L.bad = flag;
    cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int), s);
    if (e == cudaSuccess) e = launch_lowrank_rows(mode, L, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(hflag, flag, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    const int bad = e == cudaSuccess ? *hflag : 0;
    pool_host_free(hflag, sizeof(int));
    pool_device_free(flag, got, dev);
    if (e != cudaSuccess) return fail(OT_ERR_CUDA, "low-rank rows: %s", cudaGetErrorString(e));
    if (bad) return fail(OT_ERR_INVALID_ARG, "a row index is outside [0, n)");
    return OT_OK;
}

}  // namespace

extern "C" int ot_materialize_rows_lowrank(const float *Q, const float *R, const float *g, int64_t n,
                                           int64_t m, int32_t r, const int64_t *row_idx, int64_t k,
                                           float *out, void *stream) {
    NvtxRange nvtx_range("ot_materialize_rows_lowrank");
    return lowrank_rows(0, Q, R, g, nullptr, nullptr, n, m, r, 0.0, 1.0, 1.0, row_idx, k, out, stream);
}

extern "C" int ot_materialize_rows_lrcost(const float *cost1, const float *cost2, const float *f,
                                          const float *g, int64_t n, int64_t m, int32_t r,
                                          double bias, double inv_scale_cost, double eps,
                                          const int64_t *row_idx, int64_t k, float *out,
                                          void *stream) {
    NvtxRange nvtx_range("ot_materialize_rows_lrcost");
    return lowrank_rows(1, cost1, cost2, nullptr, f, g, n, m, r, bias, inv_scale_cost, eps, row_idx, k,
                        out, stream);
}

extern "C" int ot_sparsify_min_row(const ot_plan *cplan, int64_t block_rows, float *thr_out,
                                   int64_t *row_counts, int64_t *nnz_out,
                                   int64_t *n_massless_out, int64_t *argmin_out, void *stream) {
    NvtxRange nvtx_range("ot_sparsify_min_row");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if (block_rows < 0) return fail(OT_ERR_INVALID_ARG, "block_rows must be >= 0");
    block_rows = launch_rows(p, block_rows);
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    PassRows pr;
    if ((rc = pass_setup(p, 0, 0, p->n, true, s, pr)) != OT_OK) return rc;
    float thr = 0.0f;
    int64_t argmin = -1, nm = 0, nnz = 0;
    if ((rc = min_row_pass(p, 0, p->n, pr, block_rows, s, &thr, &argmin, &nm)) != OT_OK) return rc;
    rc = count_pass(p, 0, p->n, pr, block_rows, thr, row_counts ? row_counts : p->counts, s, &nnz);
    if (rc != OT_OK) return rc;
    if (thr_out) *thr_out = thr;
    if (nnz_out) *nnz_out = nnz;
    if (n_massless_out) *n_massless_out = nm;
    if (argmin_out) *argmin_out = argmin;
    if (nm > 0) {
        fail(OT_WARN_MASSLESS_ROWS, "%lld rows carry no mass", (long long)nm);
        return OT_WARN_MASSLESS_ROWS;
    }
    return OT_OK;
}

extern "C" int ot_min_row_range(const ot_plan *cplan, int64_t row_lo, int64_t row_hi,
                                int64_t block_rows, float *thr_out, int64_t *argmin_out,
                                int64_t *n_massless_out, void *stream) {
    NvtxRange nvtx_range("ot_min_row_range");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if ((rc = range_check(row_lo, row_hi, p->n, "row")) != OT_OK) return rc;
    if (block_rows < 0) return fail(OT_ERR_INVALID_ARG, "block_rows must be >= 0");
    block_rows = launch_rows(p, block_rows);
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    PassRows pr;
    if ((rc = pass_setup(p, 0, row_lo, row_hi, true, s, pr)) != OT_OK) return rc;
    float thr = 0.0f;
    int64_t argmin = -1, nm = 0;
    if ((rc = min_row_pass(p, row_lo, row_hi, pr, block_rows, s, &thr, &argmin, &nm)) != OT_OK) return rc;
    if (thr_out) *thr_out = thr;
    if (argmin_out) *argmin_out = argmin;
    if (n_massless_out) *n_massless_out = nm;
    return OT_OK;
}

extern "C" int ot_kept_counts_range(const ot_plan *cplan, int64_t row_lo, int64_t row_hi,
                                    int64_t block_rows, float thr, int64_t *row_counts,
                                    int64_t *nnz_out, void *stream) {
    NvtxRange nvtx_range("ot_kept_counts_range");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if ((rc = range_check(row_lo, row_hi, p->n, "row")) != OT_OK) return rc;
    if (block_rows < 0) return fail(OT_ERR_INVALID_ARG, "block_rows must be >= 0");
    if (std::isnan(thr)) return fail(OT_ERR_INVALID_ARG, "thr must not be NaN");
    block_rows = launch_rows(p, block_rows);
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    PassRows pr;
    if ((rc = pass_setup(p, 0, row_lo, row_hi, true, s, pr)) != OT_OK) return rc;
    int64_t nnz = 0;
    if ((rc = count_pass(p, row_lo, row_hi, pr, block_rows, thr, p->counts, s, &nnz)) != OT_OK) return rc;
    if (row_counts && row_hi > row_lo) {
        OT_CU(cudaMemcpyAsync(row_counts, p->counts + row_lo, (size_t)(row_hi - row_lo) * sizeof(int64_t),
                              cudaMemcpyDeviceToDevice, s));
        OT_CU(cudaStreamSynchronize(s));
    }
    if (nnz_out) *nnz_out = nnz;
    return OT_OK;
}

extern "C" int ot_sparsify_csr(const ot_plan *cplan, int64_t block_rows, float thr, int64_t *row_ptr,
                               int64_t *col_idx, float *vals, int64_t capacity, int64_t *nnz_out,
                               void *stream) {
    NvtxRange nvtx_range("ot_sparsify_csr");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if (block_rows < 0) return fail(OT_ERR_INVALID_ARG, "block_rows must be >= 0");
    if (!row_ptr) return fail(OT_ERR_INVALID_ARG, "row_ptr must not be NULL");
    if (capacity < 0) return fail(OT_ERR_INVALID_ARG, "capacity must be >= 0");
    if (capacity > 0 && (!col_idx || !vals))
        return fail(OT_ERR_INVALID_ARG, "col_idx and vals must not be NULL when capacity > 0");
    if (std::isnan(thr)) return fail(OT_ERR_INVALID_ARG, "thr must not be NaN");
    block_rows = launch_rows(p, block_rows);
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    // pass 1: kept entries per row (the count pass of ot_sparsify_min_row)
    PassRows pr;
    if ((rc = pass_setup(p, 0, 0, p->n, true, s, pr)) != OT_OK) return rc;
    int64_t counted = 0;
    if ((rc = count_pass(p, 0, p->n, pr, block_rows, thr, p->counts, s, &counted)) != OT_OK) return rc;
    // the write pass reads the columns in their own order
    if (p->d <= 3) OT_CU(launch_dcol(p->y, p->g, p->m, p->d, p->o, p->prm, p->dcol, s));
    // row pointers, and nnz = row_ptr[n]
    OT_CU(launch_row_ptr_scan(p->counts, p->n, row_ptr, p->scan, s));
    OT_CU(cudaMemcpyAsync(&p->ds->nnz, row_ptr + p->n, sizeof(int64_t), cudaMemcpyDeviceToDevice, s));
    OT_CU(cudaMemsetAsync(&p->ds->bad, 0, sizeof(int), s));
    if ((rc = sync_read(p, s)) != OT_OK) return rc;
    const int64_t nnz = p->hs->s.nnz;
    if (nnz_out) *nnz_out = nnz;
    if (nnz > capacity)
        return fail(OT_ERR_OVERFLOW, "%lld entries are kept, capacity is %lld", (long long)nnz,
                    (long long)capacity);
    // pass 2: the entries, in row order and increasing columns
    CsrArgs C{};
    C.pts = p->x; C.pot = p->f; C.w = p->a; C.dcol = p->dcol; C.o = p->o; C.prm = p->prm;
    C.cols = p->m; C.d = p->d; C.thr = thr; C.row_ptr = row_ptr; C.col_idx = col_idx; C.vals = vals;
    C.bad = &p->ds->bad;
    for (int64_t r0 = 0; r0 < p->n; r0 += block_rows) {
        C.row_begin = r0;
        C.row_end = std::min(p->n, r0 + block_rows);
        OT_CU(launch_csr_write(C, s));
    }
    if ((rc = sync_read(p, s)) != OT_OK) return rc;
    if (p->hs->s.bad) return fail(OT_ERR_CUDA, "the count and write passes kept different entries");
    return OT_OK;
}

extern "C" int ot_marginal_residual(const ot_plan *cplan, double *row_l1, double *col_l1,
                                    void *stream) {
    NvtxRange nvtx_range("ot_marginal_residual");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    if ((rc = residual_pass(p, 0, 0, p->n, s)) != OT_OK) return rc;
    if ((rc = residual_pass(p, 1, 0, p->m, s)) != OT_OK) return rc;
    if ((rc = sync_read(p, s)) != OT_OK) return rc;
    if (row_l1) *row_l1 = p->hs->s.r_sum[0];
    if (col_l1) *col_l1 = p->hs->s.r_sum[1];
    return OT_OK;
}

extern "C" int ot_row_pass_stats(const ot_plan *plan, int64_t *chunks_visited, int64_t *chunks_total) {
    if (!plan) return fail(OT_ERR_INVALID_ARG, "null plan");
    if (chunks_visited) *chunks_visited = plan->d <= 3 ? plan->screen_visited : 0;
    if (chunks_total) *chunks_total = plan->d <= 3 ? plan->screen_total : 0;
    return OT_OK;
}

extern "C" int ot_marginal_residual_range(const ot_plan *cplan, int64_t row_lo, int64_t row_hi,
                                          int64_t col_lo, int64_t col_hi, double *row_part,
                                          double *col_part, void *stream) {
    NvtxRange nvtx_range("ot_marginal_residual_range");
    ot_plan *p = const_cast<ot_plan *>(cplan);
    int rc = plan_check(p);
    if (rc != OT_OK) return rc;
    if ((rc = range_check(row_lo, row_hi, p->n, "row")) != OT_OK) return rc;
    if ((rc = range_check(col_lo, col_hi, p->m, "column")) != OT_OK) return rc;
    if ((rc = ensure_rows_ws(p)) != OT_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    if ((rc = screen_reset(p, s)) != OT_OK) return rc;
    if ((rc = residual_pass(p, 0, row_lo, row_hi, s)) != OT_OK) return rc;
    if ((rc = residual_pass(p, 1, col_lo, col_hi, s)) != OT_OK) return rc;
    if ((rc = sync_read(p, s)) != OT_OK) return rc;
    if (row_part) *row_part = p->hs->s.r_sum[0];
    if (col_part) *col_part = p->hs->s.r_sum[1];
    return OT_OK;
}
