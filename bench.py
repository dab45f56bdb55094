"""Benchmark of the online log-domain Sinkhorn hot path on B200.

The bench line runs workload 5, the largest configuration that fits one GPU:
n = m = 2e6 points in 3-D (two interleaved spirals), scale "max_cost",
eps 1e-3, uniform weights. One step is one call of the public entry point
ot_sinkhorn_pointcloud continuing the solve from the previous step's
potentials (warm start): the per-point tables, one iteration (the f- and the
g-half-step, fused streaming log-sum-exp over on-the-fly costs) and the f-update
that measures ||T1 - a||_1 of the new state (the fused residual and stop test),
i.e. 3 half-steps of n*m pair-updates each. The scale is resolved by the first
(warm-up) call's all-pairs max_cost pass and passed as a value afterwards (the
captured scale is never re-derived). Inputs are resident in HBM before the
timed region; the column tables (32 MB) fit in L2, so L2 is flushed (512 MiB
write) before every step. `value` = pair-updates per second of device time.
`e2e` repeats the step through ot_sinkhorn_pointcloud_host, the C-ABI call
that takes HOST arrays (pinned here): x, y, a, b, f, g copied in and f, g copied
out inside the timed region.

Side objects, timed once after the steps on the same problem: `scale_pass` (the
max_cost pass), `rows` (the row kernels at the solved state: one 4096-row
materializer block of the workload's 65,536 rows, 4096 x 2e6 entries = 32.8 GB,
the float64-assembled marginal residual and the exact min_row threshold with
counts, both over all 4e12 entries) and `block_sparse` (block-sparse fine iterations against dense ones at
n = m = 2^18); --no-side skips them.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload w5]

Under torchrun (N > 1) the same problem is split by rows across the ranks
(strong scaling): each rank updates its range of rows, NCCL all-gathers the
potentials after every half-step and all-reduces the residual; rank 0 prints
the JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Sinkhorn pair-updates/s (n·m per half-step) and % of ex2/MUFU roofline"
UNIT = "pair-updates/s"
# MUFU ex2 peak: 148 SMs x 16 ex2 per clock per SM x the maximum SM clock
SMS, EX2_PER_CLK = 148, 16


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="w5", choices=["w1", "w2", "w3", "w4", "w5"])
    ap.add_argument("--n", type=int, default=None, help="replica size of the workload (rows)")
    ap.add_argument("--m", type=int, default=None, help="replica size of the workload (columns)")
    ap.add_argument("--iters-per-step", type=int, default=1,
                    help="Sinkhorn iterations per step (one call continuing the solve)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lowrank", type=int, default=0, metavar="R",
                    help="instead of the step: time the two low-rank row materializers at rank R "
                         "(4096 rows x 100000 columns) and print their own JSON line")
    ap.add_argument("--sparse", type=int, default=0, metavar="N",
                    help="instead of the step: block-sparse against dense fine iterations on the "
                         "uniform-vs-64-clusters workload at n = m = N (its eps rule), from a "
                         "state annealed by block-sparse iterations; prints its own JSON line")
    ap.add_argument("--configs", action="store_true",
                    help="instead of the step: one JSON line per workload (w1..w5) with the GPU's "
                         "time per half-step and pair-updates/s (measured; totals of the long "
                         "configurations extrapolated and marked) and the oracle's rate on the "
                         "host cores")
    ap.add_argument("--full-run", default=None, choices=["w3", "w4", "w5"],
                    help="instead of the step: the configuration end to end as it is stated (its "
                         "iterations or anneal, then the residual, min_row and, for w5, every block "
                         "of its 65,536 rows), each part timed with CUDA events; prints its own "
                         "JSON line")
    ap.add_argument("--block-sparse", action="store_true",
                    help="--full-run: solve with block-sparse iterations (delta = 5e-3 / (4 max(NB, "
                         "MB)), blocks of 128; dense iterations where the candidates exceed half "
                         "of all block pairs)")
    ap.add_argument("--sparse-workload", default="w4", choices=["w4", "w5"],
                    help="--sparse: uniform-vs-64-clusters (w4) or interleaved spirals (w5)")
    ap.add_argument("--sparse-block", type=int, default=0, choices=[0, 128, 256],
                    help="--sparse: block size B (0 = the library's choice)")
    ap.add_argument("--rows", action="store_true",
                    help="instead of the step: the row kernels (one materializer block of the workload, the "
                         "marginal residual, min_row) at the state after 5 iterations of the workload "
                         "(or its --n/--m replica); prints its own JSON line")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (scale pass, row kernels, block-sparse)")
    ap.add_argument("--clock-ms", type=int, default=200,
                    help="nvidia-smi sampling period during the timed region")
    return ap.parse_args()


def _workload(name, n=None, m=None):
    """The named workload, or a same-recipe replica with n rows / m columns."""
    from log_domain_sinkhorn_online_b200 import workloads
    kw = {}
    if n is not None:
        kw["n"] = n
    if m is not None:
        kw["m"] = m
    return workloads.ALL[name](**kw)


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_ms=200):
        self.index, self.proc, self.path, self.period = index, None, None, period_ms

    def start(self):
        import tempfile
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows if len(r) >= 9 for k in range(4)
                          if r[5 + k].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def _dist_init(n_gpus):
    import torch
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import datetime
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    return rank, world, dist


def _max_over_ranks(v, dist, device="cuda"):
    """The max of v over all ranks (the job's time is its slowest rank's)."""
    import torch
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, max_ms_per_step):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (max_ms_per_step / 1e3)


def _barrier(dist):
    if dist is not None:
        dist.barrier()


class Step:
    """One step: a call of ot_sinkhorn_pointcloud that continues the solve for
    `iters` iterations from the current potentials (warm start), on device
    buffers that stay resident. The first call resolves the cost scale (the
    all-pairs pass of "max_cost", or the closed form of "mean"); later calls
    pass that captured value, so the scale is never re-derived."""

    def __init__(self, ot, w, dev, iters=1):
        import torch
        self.ot, self.w, self.dev, self.iters = ot, w, dev, iters
        self.x, self.y, self.a, self.b = (torch.from_numpy(np.ascontiguousarray(v)).to(dev)
                                          for v in (w.x, w.y, w.a, w.b))
        self.f = torch.zeros(w.n, dtype=torch.float32, device=dev)
        self.g = torch.zeros(w.m, dtype=torch.float32, device=dev)
        self.scale = w.scale  # becomes the captured value after the first call
        self.iterations = 0

    def kwargs(self, timing=False):
        return dict(eps=self.w.eps, scale=self.scale, n_iters=self.iters, warm_start=True,
                    timing=timing)

    def capture(self, info):
        if isinstance(self.scale, str) and self.scale != "none":
            # the float32 max (or mean) the library resolved, exactly: c = 1 / value
            self.scale = float(np.float32(1.0 / info.inv_scale_cost)) if self.scale == "max_cost" \
                else 1.0 / info.inv_scale_cost
        self.iterations += int(info.iterations)

    def __call__(self, timing=False):
        plan = self.ot.sinkhorn(self.x, self.y, self.a, self.b, f=self.f, g=self.g, **self.kwargs(timing))
        info = plan.info
        plan.close()
        self.capture(info)
        return info


def _flush_l2(buf):
    buf.zero_()


def _cpu_baseline(w, target_s=10.0):
    """The float64 oracle (as it stands) on a bounded sample of the f-half-step:
    a row sample, repeated until about target_s seconds of CPU work."""
    import oracle
    oracle.build()
    c = 1.0  # the arithmetic per pair does not depend on the scale value
    g = np.zeros(w.m)
    probe = min(w.n, 256)
    oracle.f_step(w.x, w.y, w.a, g, c, w.eps, rows=np.arange(probe))  # warm the thread pool
    t0 = time.perf_counter()
    oracle.f_step(w.x, w.y, w.a, g, c, w.eps, rows=np.arange(probe))
    rate = probe * w.m / max(time.perf_counter() - t0, 1e-6)
    rows = int(max(probe, min(w.n, rate * target_s / w.m)))
    reps = max(1, int(round(target_s / max(rows * w.m / rate, 1e-6))))
    idx = np.linspace(0, w.n - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.f_step(w.x, w.y, w.a, g, c, w.eps, rows=idx)
    dt = time.perf_counter() - t0
    return {"value": reps * rows * w.m / dt, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{reps} f-half-step(s) on {rows} of {w.n} rows x all {w.m} columns "
                      f"(float64 C, OpenMP), {dt:.1f} s"}


def _config(w, world, iters_per_step):
    """The workload as the bench line names it (the same for both arms)."""
    cfg = {"workload": w.name, "n": w.n, "m": w.m, "d": w.d, "eps": w.eps, "scale": w.scale,
           "weights": "uniform" if float(w.a.min()) == float(w.a.max()) else "non-uniform",
           "step": f"ot_sinkhorn_pointcloud continuing the solve: {iters_per_step} iteration(s) "
                   f"+ the residual f-update",
           "half_steps_per_step": 2 * iters_per_step + 1,
           "l2": "flushed (512 MiB write) before every step",
           "parallelism": "replicas" if world > 1 else "single-gpu"}
    if w.anneal:
        cfg["anneal"] = w.anneal
    return cfg


def run_reference(args):
    """The oracle, as it stands, on the host cores: bounded row samples of one
    f-half-step of the same workload, at the same metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = _workload(args.workload, args.n, args.m)
    times = []
    for it in range(args.warmup + args.steps):
        cb = _cpu_baseline(w, target_s=8.0)
        if it >= args.warmup:
            times.append(cb)
    value = statistics.mean(t["value"] for t in times)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": _config(w, 1, args.iters_per_step),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": times[0]["cores"], "kind": "oracle",
                             "sample": times[0]["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# DRAM traffic per launch of the dominant kernel comes from ncu captures
# recorded in profiles/dram_traffic.json, each with a digest of the kernel's
# source files at capture time: a kernel changed since then reports null.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def kernel_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(workload, kernel):
    try:
        with open(TRAFFIC_FILE) as fh:
            rec = json.load(fh).get(f"{workload}/{kernel}")
    except (OSError, ValueError):
        return None, "no capture recorded"
    if not rec:
        return None, "no capture recorded for this workload and kernel"
    if kernel_digest(rec["sources"]) != rec["digest"]:
        return None, "kernel source changed since the capture"
    return float(rec["bytes_per_launch"]), rec.get("note", "")


def run_lowrank(args, k=4096, m=100_000, n=20_000, reps=5):
    """Write bandwidth of the low-rank row materializers (coupling rows and
    entropic rows on a low-rank cost), k rows x m columns at rank args.lowrank,
    seeded nonnegative factors; CUDA events over `reps` calls after a warm-up."""
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    dev = torch.device("cuda", 0)
    r = args.lowrank
    gen = torch.Generator(device=dev).manual_seed(7)
    Q = torch.rand(n, r, device=dev, generator=gen)
    R = torch.rand(m, r, device=dev, generator=gen)
    g = torch.rand(r, device=dev, generator=gen) + 0.5
    f = torch.rand(n, device=dev, generator=gen) * 0.01
    gp = torch.rand(m, device=dev, generator=gen) * 0.01
    rows = torch.randint(0, n, (k,), device=dev, generator=gen)
    out = torch.empty((k, m), dtype=torch.float32, device=dev)
    peaks, kind = _peaks()
    line = {"metric": "low-rank row materializer write bandwidth", "unit": "GB/s", "rank": r,
            "config": {"rows": k, "cols": m, "n": n, "factors": "seeded uniform [0, 1)"},
            "peak_gbs": float(peaks["hbm_gbs"]), "peak_note": f"{kind} copy bandwidth"}
    for name, call in (("coupling", lambda: ot.lowrank_rows(Q, R, g, rows, out=out)),
                       ("cost", lambda: ot.lrcost_rows(Q, R, f, gp, rows, eps=0.05, bias=0.1, out=out))):
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            call()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        gbs = k * m * 4 / (ms / 1e3) / 1e9
        line[name] = {"ms": ms, "gbs": gbs, "frac": gbs / float(peaks["hbm_gbs"])}
    print(json.dumps(line), flush=True)


def run_configs(args):
    """Per workload: the GPU solve as the configuration states it where that takes
    seconds (w1, w2), else a short run of the same shape (w3: 20 of its 500
    iterations; w4: 2 iterations at its final eps; w5: 2 of its 100 iterations)
    whose time per half-step (CUDA events around the iteration loop) gives the
    configuration's total by its half-step count (marked "extrapolated"); and the
    oracle's pair-update rate on a bounded row sample on the host cores."""
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    from log_domain_sinkhorn_online_b200 import workloads as W
    dev = torch.device("cuda", 0)
    mufu = SMS * EX2_PER_CLK * 1.965e9
    for name in ("w1", "w2", "w3", "w4", "w5"):
        w = W.ALL[name]()
        x, y, a, b = (torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (w.x, w.y, w.a, w.b))
        if name in ("w1", "w2"):
            iters, full_half_steps = w.n_iters, None
        elif name == "w3":
            iters, full_half_steps = 20, 2 * w.n_iters + 1
        elif name == "w4":
            stages = 1
            while max(w.eps, w.anneal["eps_init"] * w.anneal["decay"] ** (stages - 1)) > w.eps:
                stages += 1
            iters, full_half_steps = 2, 2 * (stages * w.anneal["iters_per_stage"]) + 1
        else:
            iters, full_half_steps = 2, 2 * w.n_iters + 1
        kw = dict(tol=w.tol) if name == "w2" else {}
        plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=iters, timing=True, **kw)
        torch.cuda.synchronize()
        plan.close()  # warm: the timed call below reuses the cached workspace
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=iters, timing=True, **kw)
        e1.record()
        torch.cuda.synchronize()
        info = plan.info
        plan.close()
        per_hs_ms = info.loop_ms / max(info.half_steps, 1)
        rate = float(w.n) * float(w.m) / (per_hs_ms / 1e3)
        gpu = {"iterations": int(info.iterations), "half_steps": int(info.half_steps),
               "call_ms": e0.elapsed_time(e1), "ms_per_half_step": per_hs_ms,
               "pair_updates_per_s": rate, "frac_of_mufu": rate / mufu}
        if full_half_steps:
            gpu["total_s_extrapolated"] = per_hs_ms * full_half_steps / 1e3
            gpu["total_half_steps"] = full_half_steps
        cb = _cpu_baseline(w, target_s=5.0)
        line = {"metric": METRIC, "unit": UNIT, "config": {"workload": w.name, "n": w.n, "m": w.m,
                                                           "d": w.d, "eps": w.eps, "scale": w.scale},
                "gpu": gpu, "oracle": {"pair_updates_per_s": cb["value"], "cores": cb["cores"],
                                       "sample": cb["sample"],
                                       "ms_per_half_step_extrapolated": float(w.n) * w.m / cb["value"] * 1e3}}
        print(json.dumps(line), flush=True)


def run_full(args):
    """One configuration end to end (measured, nothing extrapolated): the solve as the
    configuration states it (w3: 500 iterations; w4: the anneal from eps 1.0 by 0.7
    per stage of 20 iterations down to its eps; w5: 100 iterations with the max_cost
    scale), then at the solved state the marginal residual, min_row with the
    workload's row blocks and, where it lists rows (w5), their materialization block
    by block into one reused buffer."""
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    dev = torch.device("cuda", 0)
    w = _workload(args.full_run)
    x, y, a, b = (torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (w.x, w.y, w.a, w.b))
    kw = dict(eps=w.eps, scale=w.scale, n_iters=w.n_iters, timing=True)
    if w.anneal:
        kw.update(n_iters=w.anneal["iters_per_stage"], eps_init=w.anneal["eps_init"],
                  eps_decay=w.anneal["decay"], iters_per_stage=w.anneal["iters_per_stage"])
    if args.block_sparse:
        nb = (max(w.n, w.m) + 127) // 128
        kw.update(block_sparse=True, sparse_block=128, sparse_delta=5e-3 / (4 * nb))
    stream = torch.cuda.current_stream()
    clocks = Clocks(torch.cuda.current_device(), args.clock_ms)
    clocks.start()
    plan, solve_ms = _timed(lambda: ot.sinkhorn(x, y, a, b, **kw), stream)
    info = plan.info
    (r, c), res_ms = _timed(plan.marginal_residual, stream)
    mr, mr_ms = _timed(lambda: plan.sparsify_min_row(block_rows=w.block_rows or 0), stream)
    visited, total = plan.row_pass_stats()
    out = {"metric": "configuration end to end", "config": {"workload": w.name, "n": w.n, "m": w.m, "d": w.d,
                                                            "eps": w.eps, "scale": w.scale},
           "solve": {"ms": solve_ms, "iterations": int(info.iterations), "stages": int(info.stages),
                     "half_steps": int(info.half_steps), "loop_ms": info.loop_ms,
                     "pair_updates_per_s": float(w.n) * w.m * info.half_steps / (info.loop_ms / 1e3),
                     "final_residual": info.residual,
                     "mode": "block-sparse" if args.block_sparse else "dense"},
           "marginal_residual": {"ms": res_ms, "row_l1": r, "col_l1": c},
           "min_row": {"ms": mr_ms, "thr": mr["thr"], "nnz": mr["nnz"], "evaluated_share": visited / total
                       if total else 1.0}}
    total_ms = solve_ms + res_ms + mr_ms
    if w.rows is not None:
        k = w.block_rows or 4096
        buf = torch.empty((k, w.m), dtype=torch.float32, device=dev)
        rows = torch.from_numpy(np.ascontiguousarray(w.rows)).to(dev)
        plan.materialize_rows(rows[:k], out=buf)  # load the kernel once, untimed

        def blocks():
            for s0 in range(0, rows.numel(), k):
                r_ = rows[s0:s0 + k]
                plan.materialize_rows(r_, out=buf[:r_.numel()])
        _, rows_ms = _timed(blocks, stream)
        out["materialize"] = {"rows": int(rows.numel()), "block_rows": k, "ms": rows_ms,
                              "gb_written": rows.numel() * w.m * 4 / 1e9,
                              "gb_per_s": rows.numel() * w.m * 4 / (rows_ms / 1e3) / 1e9}
        total_ms += rows_ms
        del buf
    if args.block_sparse:
        out["solve"].update(sparse_iterations=int(info.sparse_iterations),
                            dense_iterations=int(info.dense_iterations),
                            omitted_bound=info.omitted_bound,
                            note="pair_updates_per_s is dense-equivalent (n*m per half-step)")
    out["clocks"] = clocks.stop()
    out["total_s"] = total_ms / 1e3
    plan.close()
    print(json.dumps(out), flush=True)


def run_sparse(args, reps=10, dense_reps=2, tau=5e-3, emit=True):
    """Fine iterations at the target eps on the uniform-vs-64-clusters workload
    (n = m = args.sparse, eps = (2 x mean nearest-neighbour spacing)^2): block-
    sparse ("FlashSinkhorn 2", section 3.2; delta = tau / (4 max(NB, MB)),
    tau = 5e-3) against dense, both from the same state. The state comes from an
    untimed annealed block-sparse solve from 16 eps (x0.7 per stage, 20
    iterations each). Times are the library's CUDA events around every
    iteration (the sparse ones include the mask build and its host read-back)."""
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    from log_domain_sinkhorn_online_b200 import workloads as W
    dev = torch.device("cuda", 0)
    gen = W.w5 if (emit and args.sparse_workload == "w5") else W.w4
    w = gen(n=args.sparse if emit else 262144)
    x, y, a, b = (torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (w.x, w.y, w.a, w.b))
    blk = args.sparse_block if emit and args.sparse_block else (
        128 if (-(-w.n // 128)) * (-(-w.m // 128)) <= (1 << 27) else 256)
    delta = tau / (4.0 * max(-(-w.n // blk), -(-w.m // blk)))
    kw = dict(eps=w.eps, scale=w.scale, block_sparse=True, sparse_delta=delta, sparse_block=blk)
    t0 = time.time()
    warm = ot.sinkhorn(x, y, a, b, n_iters=20, eps_init=16.0 * w.eps, eps_decay=0.7,
                       iters_per_stage=20, **kw)
    torch.cuda.synchronize()
    warm_s = time.time() - t0
    f0, g0 = warm.f.clone(), warm.g.clone()
    warm.close()
    mufu = SMS * EX2_PER_CLK * 1.965e9
    res = {}
    for mode, k in (("sparse", reps), ("dense", dense_reps)):
        extra = kw if mode == "sparse" else dict(eps=w.eps, scale=w.scale)
        plan = ot.sinkhorn(x, y, a, b, n_iters=k, f=f0.clone(), g=g0.clone(), warm_start=True,
                           timing=True, **extra)
        torch.cuda.synchronize()
        info = plan.info
        ms_it = info.loop_ms / max(info.iterations, 1)
        res[mode] = {"ms_per_iteration": ms_it,
                     "pair_updates_per_s": 2.0 * w.n * w.m / (ms_it / 1e3),
                     "iterations": int(info.iterations), "residual": float(info.residual)}
        if mode == "sparse":
            res[mode].update(tiles_total=int(info.tiles_total), tiles_candidate=int(info.tiles_candidate),
                             tiles_admitted=int(info.tiles_admitted), tiles_exact=int(info.tiles_exact),
                             sparse_iterations=int(info.sparse_iterations),
                             omitted_bound=float(info.omitted_bound))
            full_row, full_col = plan.marginal_residual()
            res[mode]["full_row_residual"] = float(full_row)
            # the block-sparse half-step against the MUFU ex2 rate: one ex2 per
            # entry of every admitted tile (the last mask's count; the masks of
            # the timed iterations differ by a few tiles)
            pairs = float(info.tiles_admitted) * blk * blk * info.sparse_hs_launches
            hs_s = info.sparse_hs_ms / 1e3
            res[mode]["roofline"] = {
                "bound": "mufu", "kernel": "hs_sparse_kernel (block-sparse g half-step)",
                "achieved": pairs / hs_s / 1e12, "peak": mufu / 1e12, "unit": "Tex2/s",
                "frac": pairs / hs_s / mufu, "traffic": None,
                "per_launch_us": info.sparse_hs_ms * 1e3 / max(info.sparse_hs_launches, 1)}
            # the verification fused with the f-update (hs_verify_kernel): one ex2
            # per entry of every tile whose exact mass is evaluated
            vx = float(info.tiles_exact) * blk * blk * (info.sparse_iterations + 1)
            res[mode]["verify_and_f"] = {"kernel": "hs_verify_kernel (tile verification + f-update)",
                                         "ms_per_iteration": info.verify_ms / (info.sparse_iterations + 1),
                                         "exact_tiles": int(info.tiles_exact),
                                         "ex2_per_s": vx / (info.verify_ms / 1e3),
                                         "frac": vx / (info.verify_ms / 1e3) / mufu}
        plan.close()
    line = {"metric": "Sinkhorn pair-updates/s (n*m per half-step, dense equivalent)",
            "unit": "pair-updates/s", "value": res["sparse"]["pair_updates_per_s"],
            "dense_value": res["dense"]["pair_updates_per_s"],
            "speedup_vs_dense": res["dense"]["ms_per_iteration"] / res["sparse"]["ms_per_iteration"],
            "config": {"workload": f"{'spirals' if gen is W.w5 else 'uniform_vs_64clusters'}_{w.n}",
                       "n": w.n, "m": w.m, "d": 3,
                       "eps": w.eps, "scale": w.scale, "block": blk, "delta": delta, "tau": tau,
                       "state": f"annealed block-sparse from 16 eps, {warm_s:.1f} s untimed"},
            "sparse": res["sparse"], "dense": res["dense"], "mufu_peak_ex2_per_s": mufu}
    if not emit:
        return line
    print(json.dumps(line), flush=True)


CSRC = "log_domain_sinkhorn_online_b200/csrc/"
# the dominant kernel of a workload's step and the sources that define it
KERNELS = {
    "hs_loop_kernel": [CSRC + f for f in ("loop.cu", "lowd.cuh", "finish.cuh", "common.cuh")],
    "hs_lowd_kernel": [CSRC + f for f in ("halfstep.cu", "lowd.cuh", "finish.cuh", "common.cuh")],
    "hs_tc_kernel": [CSRC + f for f in ("halfstep_tc.cu", "finish.cuh", "common.cuh")],
    "hs_generic_kernel": [CSRC + f for f in ("halfstep.cu", "finish.cuh", "common.cuh")],
}


def _dominant_kernel(w):
    if w.d <= 3:
        return "hs_loop_kernel" if float(w.n) * w.m <= 2.0 ** 28 else "hs_lowd_kernel"
    return "hs_tc_kernel" if w.d >= 16 else "hs_generic_kernel"


def _timed(fn, stream):
    """Runs fn once between CUDA events on `stream`; returns (result, ms)."""
    import torch
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    r = fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return r, e0.elapsed_time(e1)


def _side(ot, step, w, stream, peak_ex2, hbm_gbs):
    """Side measurements on the solved problem (each call timed once, warm)."""
    import torch
    out = {}
    # a1: the all-pairs max_cost pass (a plan built with no iteration)
    if w.scale == "max_cost":
        kw = dict(eps=w.eps, n_iters=0, warm_start=True, f=step.f.clone(), g=step.g.clone())
        ot.sinkhorn(step.x, step.y, step.a, step.b, scale="max_cost", **kw).close()
        _, ms = _timed(lambda: ot.sinkhorn(step.x, step.y, step.a, step.b, scale="max_cost", **kw).close(),
                       stream)
        out["scale_pass"] = {"what": "plan set-up with the all-pairs max_cost pass (max_cost_lowd_kernel)",
                             "ms": ms, "pairs_per_s": float(w.n) * w.m / (ms / 1e3)}
    # a8-a10 at the solved state, through one plan; the row kernels are loaded first on a
    # small problem of the same d (their first launch would otherwise load the module)
    xs, ys = step.x[:256].contiguous(), step.y[:256].contiguous()
    ws = torch.full((256,), 1.0 / 256, device=step.dev)
    small = ot.sinkhorn(xs, ys, ws, ws, eps=w.eps, scale=step.scale, n_iters=2)
    small.materialize_rows(torch.arange(8, device=step.dev))
    small.marginal_residual()
    small.sparsify_min_row()
    small.close()
    plan = ot.sinkhorn(step.x, step.y, step.a, step.b, eps=w.eps, scale=step.scale, n_iters=0,
                       warm_start=True, f=step.f.clone(), g=step.g.clone())
    k = w.block_rows or 1024  # one block of the workload's row materialization
    rows = torch.from_numpy(np.ascontiguousarray(w.rows[:k] if w.rows is not None
                                                 else np.arange(min(k, w.n), dtype=np.int64))).to(step.dev)
    buf = torch.empty((rows.numel(), w.m), dtype=torch.float32, device=step.dev)
    plan.materialize_rows(rows, out=buf)
    _, ms = _timed(lambda: plan.materialize_rows(rows, out=buf), stream)
    gbs = rows.numel() * w.m * 4 / (ms / 1e3) / 1e9
    out["materialize"] = {"kernel": "materialize_kernel", "rows": int(rows.numel()), "cols": w.m, "ms": ms,
                          "gb_per_s": gbs, "frac_of_hbm": gbs / hbm_gbs}
    # a8, a10: two passes over the plan's entries each; the tile screen skips tiles whose
    # entries all vanish, so the rate over all entries and the MUFU fraction over the
    # entries actually evaluated are both given
    ent = 2.0 * w.n * w.m

    def _rows(ms):
        visited, total = plan.row_pass_stats()
        share = visited / total if total else 1.0
        return {"ms": ms, "entries_per_s": ent / (ms / 1e3), "evaluated_share": share,
                "frac_of_mufu": ent * share / (ms / 1e3) / peak_ex2,
                "note": "entries_per_s counts every entry of both passes; frac_of_mufu the evaluated ones"}
    (r, c), ms = _timed(plan.marginal_residual, stream)
    out["marginal_residual"] = dict(kernel="rowpass_kernel (sum)", row_l1=r, col_l1=c, **_rows(ms))
    mr, ms = _timed(lambda: plan.sparsify_min_row(block_rows=w.block_rows or 0), stream)
    out["min_row"] = dict(kernel="rowpass_kernel (max, count)", thr=mr["thr"], nnz=mr["nnz"], **_rows(ms))
    plan.close()
    del buf
    return out


def run_sharded(args, rank, world, dist, w, dev):
    """N > 1: the solve split by rows across the ranks (log_domain_sinkhorn_online_b200.sharded):
    per step one iteration and the residual f-update, each half-step followed by an NCCL
    all-gather of the updated potential ranges, the residual summed by an all-reduce.
    Strong scaling: the whole problem's pair-updates over the slowest rank's time."""
    import torch
    from log_domain_sinkhorn_online_b200 import sharded as S
    x, y, a, b = (torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (w.x, w.y, w.a, w.b))
    xr, yr = S.Ranges(w.n, world), S.Ranges(w.m, world)
    scale = w.scale
    if scale == "max_cost":
        scale = S.max_cost_value(x, y, xr, rank)
    backend = S.CudaShard(x, y, a, b, w.eps, scale, xr, yr, rank)
    solver = S.ShardedSinkhorn(backend, xr, yr, rank, world, like=x)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        solver.solve(args.iters_per_step)
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device(), args.clock_ms)
    _barrier(dist)
    clocks.start()
    total_ms, resid = 0.0, None
    for _ in range(args.steps):
        _flush_l2(flush)
        (_, resid), ms = _timed(lambda: solver.solve(args.iters_per_step), stream)
        total_ms += ms
    clk = clocks.stop()
    _barrier(dist)
    total_ms = _max_over_ranks(total_ms, dist)
    half_steps = 2 * args.iters_per_step + 1
    units = float(w.n) * float(w.m) * half_steps  # the whole problem's pair-updates per step
    value = units / (total_ms / args.steps / 1e3)
    # e2e: every rank's inputs and the potentials from and to pinned host memory
    host = [t.cpu().pin_memory() for t in (x, y, a, b)]
    fh = torch.zeros(w.n, dtype=torch.float32).pin_memory()
    gh = torch.zeros(w.m, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    e2e_ms = 0.0

    def e2e_step():
        for dst, src in zip((x, y, a, b), host):
            dst.copy_(src, non_blocking=True)
        solver.f[solver.k][:w.n].copy_(fh, non_blocking=True)
        solver.g[:w.m].copy_(gh, non_blocking=True)
        solver.solve(args.iters_per_step)
        f, g = solver.potentials()
        fh.copy_(f, non_blocking=True)
        gh.copy_(g, non_blocking=True)

    _barrier(dist)
    for _ in range(e2e_steps):
        _flush_l2(flush)
        _, ms = _timed(e2e_step, stream)
        e2e_ms += ms
    e2e_ms = _max_over_ranks(e2e_ms, dist)
    backend.close()
    if rank == 0:
        peaks, kind = _peaks()
        sm_max = float(peaks.get("sm_max_mhz", 1965.0))
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded point clouds; recipe in log_domain_sinkhorn_online_b200/workloads.py)",
                "config": dict(_config(w, world, args.iters_per_step), parallelism=f"rows split over {world} GPUs"),
                "clocks": clk,
                "e2e": {"value": units * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                        "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host) + 4 * (w.n + w.m),
                        "d2h_bytes_per_step": 4 * (w.n + w.m), "steps": e2e_steps,
                        "call": "ot_shard_half_step per rank, NCCL all-gathers (pinned host arrays)"},
                "gpu_launches": 2 * half_steps * args.steps,
                "roofline": {"bound": "mufu", "kernel": _dominant_kernel(w) + " (fused f/g half-step, row range)",
                             "achieved": units / world / (total_ms / args.steps / 1e3) / 1e12,
                             "peak": SMS * EX2_PER_CLK * sm_max * 1e6 / 1e12, "unit": "Tex2/s per GPU",
                             "frac": units / world / (total_ms / args.steps / 1e3) / (SMS * EX2_PER_CLK * sm_max * 1e6),
                             "traffic": None, "traffic_note": "not captured for the split solve",
                             "note": "per GPU, whole step time (collectives included)"},
                "run": {"last_residual": resid}}
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()


def run_ours(args):
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    from log_domain_sinkhorn_online_b200 import _binding as B
    rank, world, dist = _dist_init(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = _workload(args.workload, args.n, args.m)
    if world > 1:
        return run_sharded(args, rank, world, dist, w, dev)
    step = Step(ot, w, dev, args.iters_per_step)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-resident timed region
    clocks = Clocks(torch.cuda.current_device(), args.clock_ms)
    _barrier(dist)
    clocks.start()
    total_ms, loop_ms, half_steps, launches = 0.0, 0.0, 0, 0
    for _ in range(args.steps):
        _flush_l2(flush)
        info, ms = _timed(lambda: step(timing=True), stream)
        total_ms += ms
        loop_ms += info.loop_ms
        half_steps += info.half_steps
        launches += info.kernel_launches
    clk = clocks.stop()
    _barrier(dist)
    total_ms = _max_over_ranks(total_ms, dist)
    units = float(w.n) * float(w.m) * half_steps / args.steps  # pair-updates per step (this rank)
    value = weak_scaling_value(units, world, total_ms / args.steps)

    # ---- end to end through the C-ABI call that takes host arrays (pinned)
    host = [t.cpu().pin_memory() for t in (step.x, step.y, step.a, step.b, step.f, step.g)]
    opt = B.ot_options_default()
    opt.warm_start = 1
    sc = B.OT_SCALE_VALUE if not isinstance(step.scale, str) else B.OT_SCALE_NONE
    if sc == B.OT_SCALE_VALUE:
        opt.scale_value = float(step.scale)
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = (w.n + w.m) * 4
    e2e_steps = max(1, min(args.steps, 5))
    e2e_ms, e2e_units = 0.0, 0.0
    _barrier(dist)
    for _ in range(e2e_steps):
        _flush_l2(flush)
        (_, _, inf), ms = _timed(lambda: B.ot_sinkhorn_pointcloud_host(
            *(t.data_ptr() for t in host[:4]), w.n, w.m, w.d, float(w.eps), sc, args.iters_per_step, 0.0,
            host[4].data_ptr(), host[5].data_ptr(), stream.cuda_stream, opt), stream)
        e2e_ms += ms
        e2e_units += float(w.n) * float(w.m) * inf.half_steps
    e2e_ms = _max_over_ranks(e2e_ms, dist)
    e2e_value = e2e_units * world / (e2e_ms / 1e3)

    if rank == 0:
        peaks, kind = _peaks()
        sm_max = float(peaks.get("sm_max_mhz", 1965.0))
        peak_ex2 = SMS * EX2_PER_CLK * sm_max * 1e6
        side = _side(ot, step, w, stream, peak_ex2, float(peaks["hbm_gbs"])) if not args.no_side else None
        sparse_line = run_sparse(args, emit=False) if (not args.no_side and w.d <= 3) else None
        per_launch_ms = loop_ms / max(half_steps, 1)
        achieved = float(w.n) * float(w.m) / (per_launch_ms / 1e3)
        kname = _dominant_kernel(w)
        traffic, tnote = _traffic(w.name if (args.n, args.m) == (None, None) else None, kname)
        roof = {"bound": "mufu", "kernel": kname + " (fused f/g half-step)",
                "achieved": achieved / 1e12, "peak": peak_ex2 / 1e12, "unit": "Tex2/s",
                "frac": achieved / peak_ex2, "traffic": traffic, "traffic_note": tnote,
                "per_launch_us": per_launch_ms * 1e3,
                "peak_note": f"derived: 148 SMs x 16 MUFU ex2/clk x {sm_max:.0f} MHz ({kind} sm_max); "
                             "one ex2 per pair-update"}
        if clk.get("sm_mhz"):
            roof["frac_at_sampled_clock"] = achieved / (SMS * EX2_PER_CLK * clk["sm_mhz"] * 1e6)
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": warmup, "ms_per_step": total_ms / args.steps,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded point clouds; recipe in log_domain_sinkhorn_online_b200/workloads.py)",
                "config": _config(w, world, args.iters_per_step),
                "roofline": roof, "clocks": clk,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                        "call": "ot_sinkhorn_pointcloud_host (pinned host arrays)"},
                "gpu_launches": launches,
                "run": {"iterations_done": step.iterations, "half_steps_timed": half_steps,
                        "last_residual": float(info.residual), "col_splits": int(info.col_splits)}}
        if side:
            line.update(side)
        if sparse_line is not None:
            sp = sparse_line["sparse"]
            line["block_sparse"] = {
                "workload": sparse_line["config"]["workload"], "eps": sparse_line["config"]["eps"],
                "ms_per_fine_iteration": sp["ms_per_iteration"],
                "dense_ms_per_iteration": sparse_line["dense"]["ms_per_iteration"],
                "speedup_vs_dense": sparse_line["speedup_vs_dense"],
                "pair_updates_per_s_dense_equivalent": sparse_line["value"],
                "tiles_admitted": sp["tiles_admitted"], "tiles_total": sp["tiles_total"],
                "residual_certified": sp["residual"], "residual_full": sp["full_row_residual"],
                "hs_verify_frac": sp["verify_and_f"]["frac"], "hs_sparse_frac": sp["roofline"]["frac"]}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = _cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_rows(args):
    """The row kernels alone on a solved state of the workload (one materializer
    block of the workload's block size)."""
    import torch
    import log_domain_sinkhorn_online_b200 as ot
    dev = torch.device("cuda", 0)
    w = _workload(args.workload, args.n, args.m)
    step = Step(ot, w, dev, iters=5)
    step()
    peaks, kind = _peaks()
    peak_ex2 = SMS * EX2_PER_CLK * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    side = _side(ot, step, w, torch.cuda.current_stream(), peak_ex2, float(peaks["hbm_gbs"]))
    side.pop("scale_pass", None)
    print(json.dumps({"metric": "row kernels", "config": {"workload": w.name, "n": w.n, "m": w.m, "d": w.d},
                      "peak_ex2_per_s": peak_ex2, "hbm_gbs": float(peaks["hbm_gbs"]), "peaks": kind,
                      **side}), flush=True)


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    elif args.rows:
        run_rows(args)
    elif args.full_run:
        run_full(args)
    elif args.lowrank:
        run_lowrank(args)
    elif args.sparse:
        run_sparse(args)
    elif args.configs:
        run_configs(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
