"""Writes the float64 oracle's Sinkhorn trajectories that the GPU parity tests
compare against (``tests/golden/traj_<case>.npz``).

Only ``oracle/`` computes here; the inputs come from the seeded recipes of
``log_domain_sinkhorn_online_b200/workloads.py`` (which hold none of the
method's arithmetic). Nothing is read from the CUDA path. Each case is a
benchmark workload, at its full size where the oracle finishes in minutes and
otherwise as a same-recipe replica:

=====================  =======================================================
case                   what the oracle runs
=====================  =======================================================
w2_8000                workload 2 in full: 8000 x 8000, d = 3, scale "mean",
                       eps 0.01, from f = g = 0 until ||T1 - a||_1 <= 1e-3
                       (cap 2000); the row residual after every iteration is
                       kept for the rounding rule on the stopping iteration
w3_4000x5000           workload 3's recipe at 4000 x 5000 (d = 50, scale
                       "mean", eps 0.005, non-uniform weights): 500 iterations
w4_20000_own_eps       workload 4's recipe at n = m = 20000 with its own eps
                       rule, (2 x mean nearest-neighbour spacing of this x)^2,
                       annealed from 1.0 by x0.7 per stage, 20 iterations per
                       stage including the last
w4_20000_eps_1e6       the same replica at the eps of the 10^6-point workload
                       (about 1.24e-4, 27 stages, 540 iterations)
w5_20000               workload 5's recipe at n = m = 20000: spirals, scale
                       "max_cost", eps 1e-3, 100 iterations
=====================  =======================================================

Updates are those of "FlashSinkhorn 2: Block-Sparse Entropic Optimal
Transport", section 2.1 (f then g, streaming log-sum-exp); annealing follows
sections 3.1 and C.3 (decreasing eps, continuation at the target).

    python tests/golden/make_trajectories.py [case ...]
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from log_domain_sinkhorn_online_b200 import workloads as W  # noqa: E402


def _w4_eps_1e6() -> float:
    """eps of the 10^6-point workload 4 (its own nearest-neighbour rule)."""
    return W.w4().eps


CASES = {
    "w2_8000": dict(gen="w2", kw={}),
    "w3_4000x5000": dict(gen="w3", kw=dict(n=4000, m=5000)),
    "w4_20000_own_eps": dict(gen="w4", kw=dict(n=20000)),
    "w4_20000_eps_1e6": dict(gen="w4", kw=dict(n=20000), eps=_w4_eps_1e6),
    "w5_20000": dict(gen="w5", kw=dict(n=20000)),
}


def path(case: str) -> str:
    return os.path.join(HERE, f"traj_{case}.npz")


def run(case: str) -> dict:
    spec = CASES[case]
    w = W.ALL[spec["gen"]](**spec["kw"])
    eps = float(np.float32(spec["eps"]())) if "eps" in spec else float(w.eps)
    c = oracle.inv_scale_cost(w.x, w.y, w.scale)
    t0 = time.time()
    out = dict(n=w.n, m=w.m, d=w.d, eps=eps, c=c, scale=w.scale)
    if w.anneal:
        an = w.anneal
        f, g, stages, r = oracle.sinkhorn_anneal(w.x, w.y, w.a, w.b, c, eps, an["eps_init"], an["decay"],
                                                 an["iters_per_stage"])
        out.update(f=f, g=g, iterations=stages * an["iters_per_stage"], stages=stages, residual=r,
                   eps_init=an["eps_init"], eps_decay=an["decay"], iters_per_stage=an["iters_per_stage"])
    elif w.tol > 0.0:
        # one iteration per call, so the row residual of every state is kept
        f, g = np.zeros(w.n), np.zeros(w.m)
        hist = []
        for _ in range(w.n_iters):
            f, g, _, r = oracle.sinkhorn(w.x, w.y, w.a, w.b, c, eps, 1, f0=f, g0=g)
            hist.append(r)
            if r <= w.tol:
                break
        out.update(f=f, g=g, iterations=len(hist), residual=hist[-1], resid_hist=np.array(hist),
                   tol=w.tol, cap=w.n_iters)
    else:
        f, g, it, r = oracle.sinkhorn(w.x, w.y, w.a, w.b, c, eps, w.n_iters)
        out.update(f=f, g=g, iterations=it, residual=r)
    out["oracle_seconds"] = time.time() - t0
    out["oracle_threads"] = oracle.num_threads()
    return out


def main(argv):
    oracle.build()
    for case in (argv or list(CASES)):
        res = run(case)
        np.savez(path(case), **{k: np.asarray(v) for k, v in res.items()})
        print(f"{case}: {res['iterations']} iterations, residual {float(res['residual']):.6e}, "
              f"{res['oracle_seconds']:.0f} s on {res['oracle_threads']} threads", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
