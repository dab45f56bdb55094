"""The Sinkhorn solve split by rows across ranks (one process per GPU).

"FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section 5: at
10^10 points one measure no longer fits one GPU, so the solve runs on several.
Here every rank holds both clouds in full (2e6 points in 3-D are 24 MB) and
owns one contiguous, tile-aligned range of x's rows and one of y's. One
iteration is

    f-update of the rank's x rows  (ot_shard_half_step, side 0)
    all-gather of f                (the updated ranges of every rank)
    g-update of the rank's y rows  (side 1)
    all-gather of g

and, for a stopping test, an all-reduce (sum) of the ranks' residual parts,
which the f-update of the next iteration measures at the state before it,
exactly as the single-GPU solve does. Every rank takes the same collective
steps in the same order. The half-steps run in the library's kernels; this
module only orders the calls and the collectives (torch.distributed: NCCL for
CUDA tensors, gloo for the CPU tests, whose ranks use the float64 oracle's
half-step as a stand-in backend).

The row calls split the same way (ShardedRows): each rank reduces its own
rows of the plan at the gathered potentials -- the marginal residual's parts
(one all-reduce, sum), the min_row threshold's candidates (all-reduce, min),
then the kept counts at that threshold (all-reduce, sum) -- and materializes
its own share of a row list, which needs no exchange at all.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass
class Ranges:
    """Rank r owns rows [lo(r), hi(r)) of a cloud of `count` points; every rank's
    share is padded to `shard` rows (a multiple of `align`), so potentials are
    exchanged as equal chunks of a buffer of world * shard entries."""
    count: int
    world: int
    align: int = 1024

    @property
    def shard(self) -> int:
        per = -(-self.count // self.world)
        return max(self.align, -(-per // self.align) * self.align)

    def lo(self, rank: int) -> int:
        lo = rank * self.shard
        return lo if lo < self.count else 0

    def hi(self, rank: int) -> int:
        lo = rank * self.shard
        return min(lo + self.shard, self.count) if lo < self.count else 0

    @property
    def padded(self) -> int:
        return self.world * self.shard


class CudaShard:
    """The library's half-step over one rank's rows (C ABI, device buffers)."""

    def __init__(self, x, y, a, b, eps, scale, xr: Ranges, yr: Ranges, rank, stream=None, **opts):
        import torch
        from . import _binding as B
        self.B = B
        self.stream = (torch.cuda.current_stream() if stream is None else stream).cuda_stream
        n, d = x.shape
        m = y.shape[0]
        opt = B.ot_options_default()
        for k, v in opts.items():
            setattr(opt, k, v)
        if isinstance(scale, str):
            sc = {"none": B.OT_SCALE_NONE, "mean": B.OT_SCALE_MEAN, "max_cost": B.OT_SCALE_MAX_COST}[scale]
        else:
            sc = B.OT_SCALE_VALUE
            opt.scale_value = float(scale)
        self.plan, self.info = B.ot_shard_plan_create(
            x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), n, m, d, float(eps), sc,
            xr.lo(rank), xr.hi(rank), yr.lo(rank), yr.hi(rank), self.stream, opt)
        self._keep = (x, y, a, b)

    def half_step(self, side, other, cur, out, want_resid):
        return self.B.ot_shard_half_step(self.plan, side, other.data_ptr(), cur.data_ptr(), out.data_ptr(),
                                         self.stream, want_resid)

    def close(self):
        if self.plan:
            self.B.ot_plan_destroy(self.plan)
            self.plan = None


def max_cost_value(x, y, xr: Ranges, rank, group=None):
    """The all-pairs max of ||x_i - y_j||^2 as the single-GPU max_cost pass finds
    it: each rank takes its x rows, an all-reduce (max) combines them."""
    import torch
    import torch.distributed as dist
    from . import _binding as B
    n, d = x.shape
    v = B.ot_max_sqdist(x.data_ptr(), y.data_ptr(), n, y.shape[0], d, xr.lo(rank), xr.hi(rank),
                        torch.cuda.current_stream().cuda_stream)
    t = torch.tensor([v], dtype=torch.float32, device=x.device)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


class ShardedSinkhorn:
    """Alternating updates with the rows split across the ranks of `group`.

    backend: an object with half_step(side, other, cur, out, want_resid) ->
    residual part (or None) that updates `out` on this rank's rows; the
    potentials are 1-D tensors of Ranges.padded entries (x side) and (y side).
    """

    def __init__(self, backend, xr: Ranges, yr: Ranges, rank, world, group=None, like=None):
        import torch
        self.backend, self.xr, self.yr = backend, xr, yr
        self.rank, self.world, self.group = rank, world, group
        kw = dict(dtype=like.dtype, device=like.device) if like is not None else dict(dtype=torch.float32)
        self.f = [torch.zeros(xr.padded, **kw), torch.zeros(xr.padded, **kw)]
        self.g = torch.zeros(yr.padded, **kw)
        self.k = 0  # self.f[self.k] holds the current state

    # ---- collectives (the same sequence on every rank)
    def _gather(self, buf, r: Ranges):
        import torch.distributed as dist
        if self.world == 1:
            return
        mine = buf[self.rank * r.shard:(self.rank + 1) * r.shard].clone()
        if buf.is_cuda:
            dist.all_gather_into_tensor(buf, mine, group=self.group)
        else:
            dist.all_gather(list(buf.split(r.shard)), mine, group=self.group)

    def _sum(self, v):
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return float(v)
        dev = self.f[0].device
        t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, group=self.group)
        return float(t.item())

    # ---- the two half-steps
    def f_update(self, want_resid):
        cur, out = self.f[self.k], self.f[self.k ^ 1]
        r = self.backend.half_step(0, self.g, cur, out, want_resid)
        self._gather(out, self.xr)
        return r

    def g_update(self):
        self.backend.half_step(1, self.f[self.k ^ 1], self.g, self.g, False)
        self._gather(self.g, self.yr)
        self.k ^= 1

    def solve(self, n_iters, tol=0.0, measure_final=True):
        """Runs up to n_iters iterations; with tol > 0 stops after the first
        iteration whose ||T1 - a||_1 <= tol. Returns (iterations, residual or
        None); the state is in self.potentials()."""
        done, resid = 0, None
        for it in range(n_iters):
            check = tol > 0.0 and done >= 1
            r = self.f_update(check)
            if check:
                resid = self._sum(r)
                if resid <= tol:
                    return done, resid  # the state before this f-update
            self.g_update()
            done += 1
        if measure_final and done > 0:
            resid = self._sum(self.f_update(True))  # the final state's residual; f[k] unchanged
        return done, resid

    def potentials(self):
        return self.f[self.k][:self.xr.count], self.g[:self.yr.count]


class CudaRows:
    """The library's row calls over one rank's rows: a plan of
    ot_sinkhorn_pointcloud at the given (gathered) potentials, no iteration.
    scale: the resolved value the solve used (a string re-resolves it, which
    for "max_cost" is a full pass over all pairs)."""

    def __init__(self, x, y, a, b, f, g, eps, scale, stream=None):
        import torch
        from . import _binding as B
        from . import sinkhorn
        self.B = B
        self.stream = (torch.cuda.current_stream() if stream is None else stream)
        self.plan = sinkhorn(x, y, a, b, eps=eps, scale=scale, n_iters=0, warm_start=True,
                             f=f.clone(), g=g.clone(), stream=self.stream)
        self.n = x.shape[0]

    def residual(self, row_lo, row_hi, col_lo, col_hi):
        return self.B.ot_marginal_residual_range(self.plan.handle, row_lo, row_hi, col_lo, col_hi,
                                                 self.stream.cuda_stream)

    def row_max(self, lo, hi, block_rows):
        return self.B.ot_min_row_range(self.plan.handle, lo, hi, block_rows, self.stream.cuda_stream)

    def row_count(self, lo, hi, thr, block_rows):
        import torch
        counts = torch.empty(max(hi - lo, 0), dtype=torch.int64, device=self.plan.f.device)
        nnz = self.B.ot_kept_counts_range(self.plan.handle, lo, hi, block_rows, float(thr),
                                          counts.data_ptr() if hi > lo else 0, self.stream.cuda_stream)
        return counts, nnz

    def materialize(self, row_idx, out=None):
        return self.plan.materialize_rows(row_idx, out=out, stream=self.stream)

    def close(self):
        self.plan.close()


def share(count: int, rank: int, world: int):
    """Positions [lo, hi) of a list of `count` items that rank `rank` takes
    (contiguous, sizes differing by at most one)."""
    lo = count * rank // world
    return lo, count * (rank + 1) // world


class ShardedRows:
    """Row calls with the rows split across the ranks of `group` (the same
    Ranges as the solve). backend: residual(row_lo, row_hi, col_lo, col_hi) ->
    (row_part, col_part); row_max(lo, hi, block_rows) -> (thr, argmin,
    n_massless); row_count(lo, hi, thr, block_rows) -> (counts of the range,
    nnz). device: where the collectives' buffers live (CUDA for NCCL)."""

    _NONE = 1 << 62

    def __init__(self, backend, xr: Ranges, yr: Ranges, rank, world, group=None, device=None):
        self.backend, self.xr, self.yr = backend, xr, yr
        self.rank, self.world, self.group, self.device = rank, world, group, device

    def _reduce(self, vals, dtype, op):
        import torch
        import torch.distributed as dist
        t = torch.tensor(vals, dtype=dtype, device=self.device)
        if self.world > 1:
            dist.all_reduce(t, op=op, group=self.group)
        return t.tolist()

    def marginal_residual(self):
        """(||T1 - a||_1, ||T^T 1 - b||_1): this rank's rows of x and of y."""
        import torch
        import torch.distributed as dist
        r, c = self.backend.residual(self.xr.lo(self.rank), self.xr.hi(self.rank),
                                     self.yr.lo(self.rank), self.yr.hi(self.rank))
        return tuple(self._reduce([r, c], torch.float64, dist.ReduceOp.SUM))

    def min_row(self, block_rows=0):
        """The min_row threshold of the whole plan (thr, argmin, n_massless,
        nnz) and this rank's kept counts (rows [xr.lo(rank), xr.hi(rank)))."""
        import torch
        import torch.distributed as dist
        lo, hi = self.xr.lo(self.rank), self.xr.hi(self.rank)
        thr_l, arg_l, nm_l = self.backend.row_max(lo, hi, block_rows)
        thr = self._reduce([thr_l], torch.float64, dist.ReduceOp.MIN)[0]
        cand = arg_l if (arg_l >= 0 and thr_l == thr) else self._NONE
        arg = self._reduce([cand], torch.int64, dist.ReduceOp.MIN)[0]
        nm = self._reduce([nm_l], torch.int64, dist.ReduceOp.SUM)[0]
        counts, nnz_l = self.backend.row_count(lo, hi, thr, block_rows)
        nnz = self._reduce([nnz_l], torch.int64, dist.ReduceOp.SUM)[0]
        return dict(thr=thr, argmin=-1 if arg == self._NONE else arg, n_massless=nm, nnz=nnz,
                    counts=counts)
