"""Seeded synthetic point-cloud workloads (inputs only -- none of the method's arithmetic).

Both the CUDA path and the float64 oracle are fed from here; nothing in this
module evaluates a cost, a potential or a plan. Every generator uses NumPy's
PCG64 (``default_rng``): coordinates from ``seed``, weights and row indices
from ``seed + 100``. Coordinates are drawn in float64 and cast to float32 once.

The five recipes are the workloads this library is measured on:

=====  ==========================================================================
name   recipe
=====  ==========================================================================
w1     n=m=512, d=2, x,y i.i.d. U[0,1]^2; a=b=1/n; unscaled; eps=0.05; 200 iters
w2     n=m=8000, d=3, 8-component isotropic Gaussian mixture (sigma=0.05, centres
       U[0,1]^3); y: a fresh sample of the same mixture shifted by +0.1 per axis;
       uniform weights; scale "mean"; eps=0.01; tol 1e-3 on ||T1-a||_1, cap 2000;
       min_row sparsify in row blocks of 1024
w3     n=40000, m=50000, d=50, x ~ N(0, diag(1/k)), y ~ N(mu, diag(1/k)) with
       mu = 0.3 on the first 5 axes; a,b ~ Exp(1) normalised; scale "mean";
       eps=0.005; 500 iters
w4     n=m=1e6, d=3, x U[0,1]^3, y a 64-cluster mixture (sigma=0.02, centres
       U[0,1]^3, equal weights, clipped to the cube); unscaled;
       eps=(2 * mean nearest-neighbour spacing of x)^2; eps annealed from 1.0 by
       x0.7 per stage, 20 iters per stage
w5     n=m=2e6, d=3, two interleaved spirals (radius noise 0.01) in [0,1]^3;
       scale "max_cost"; eps=1e-3; 100 iters; 65,536 random rows materialized in
       blocks of 4096
=====  ==========================================================================

Every generator accepts smaller ``n``/``m`` to build a replica of the same
distribution for tests that the oracle must finish in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass
class Workload:
    name: str
    x: np.ndarray            # [n, d] float32
    y: np.ndarray            # [m, d] float32
    a: np.ndarray            # [n] float32
    b: np.ndarray            # [m] float32
    eps: float
    scale: str               # "none" | "mean" | "max_cost"
    n_iters: int
    tol: float = 0.0
    anneal: dict | None = None           # eps_init, decay, iters_per_stage
    block_rows: int = 0
    rows: np.ndarray | None = None       # int64 row indices to materialize
    extra: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return self.x.shape[0]

    @property
    def m(self) -> int:
        return self.y.shape[0]

    @property
    def d(self) -> int:
        return self.x.shape[1]


def _uniform_weights(k: int) -> np.ndarray:
    return np.full(k, 1.0 / k, dtype=np.float64).astype(np.float32)


def _mixture(rng, k, centres, sigma):
    lab = rng.integers(0, centres.shape[0], size=k)
    return centres[lab] + sigma * rng.standard_normal((k, centres.shape[1]))


def w1(n: int = 512, m: int | None = None, seed: int = 0) -> Workload:
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    x = rng.random((n, 2))
    y = rng.random((m, 2))
    return Workload("w1_uniform2d_512", x.astype(np.float32), y.astype(np.float32),
                    _uniform_weights(n), _uniform_weights(m), eps=0.05, scale="none",
                    n_iters=200, block_rows=0, rows=np.arange(n, dtype=np.int64))


def w2(n: int = 8000, m: int | None = None, seed: int = 1) -> Workload:
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    centres = rng.random((8, 3))
    x = _mixture(rng, n, centres, 0.05)
    y = _mixture(rng, m, centres, 0.05) + 0.1
    return Workload("w2_gmm3d_8000", x.astype(np.float32), y.astype(np.float32),
                    _uniform_weights(n), _uniform_weights(m), eps=0.01, scale="mean",
                    n_iters=2000, tol=1e-3, block_rows=1024)


def w3(n: int = 40000, m: int = 50000, seed: int = 2) -> Workload:
    rng = np.random.default_rng(seed)
    d = 50
    std = 1.0 / np.sqrt(np.arange(1, d + 1, dtype=np.float64))
    x = rng.standard_normal((n, d)) * std
    mu = np.zeros(d)
    mu[:5] = 0.3
    y = rng.standard_normal((m, d)) * std + mu
    wr = np.random.default_rng(seed + 100)
    a = wr.exponential(1.0, n)
    b = wr.exponential(1.0, m)
    a = (a / a.sum()).astype(np.float32)
    b = (b / b.sum()).astype(np.float32)
    return Workload("w3_embed50d_40000x50000", x.astype(np.float32), y.astype(np.float32), a, b,
                    eps=0.005, scale="mean", n_iters=500)


def mean_nn_spacing(x: np.ndarray) -> float:
    """Mean over points of the distance to the nearest other point (float64, exact kd-tree)."""
    from scipy.spatial import cKDTree
    xd = np.asarray(x, dtype=np.float64)
    dist, _ = cKDTree(xd).query(xd, k=2)
    return float(dist[:, 1].mean())


def w4(n: int = 1_000_000, m: int | None = None, seed: int = 3) -> Workload:
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    x = rng.random((n, 3))
    centres = rng.random((64, 3))
    y = np.clip(_mixture(rng, m, centres, 0.02), 0.0, 1.0)
    x32 = x.astype(np.float32)
    eps = float(np.float32((2.0 * mean_nn_spacing(x32)) ** 2))
    return Workload("w4_uniform_vs_clusters_1e6", x32, y.astype(np.float32),
                    _uniform_weights(n), _uniform_weights(m), eps=eps, scale="none",
                    n_iters=20, anneal=dict(eps_init=1.0, decay=0.7, iters_per_stage=20))


def _spiral(rng, k, phase):
    t = rng.random(k)
    theta = 6.0 * np.pi * t + phase
    r = 0.45 * t + 0.01 * rng.standard_normal(k)
    p = np.stack([0.5 + r * np.cos(theta), 0.5 + r * np.sin(theta), t], axis=1)
    return np.clip(p, 0.0, 1.0)


def w5(n: int = 2_000_000, m: int | None = None, seed: int = 4, n_rows: int = 65536,
       block_rows: int = 4096) -> Workload:
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    x = _spiral(rng, n, 0.0)
    y = _spiral(rng, m, np.pi)
    wr = np.random.default_rng(seed + 100)
    rows = np.sort(wr.choice(n, size=min(n_rows, n), replace=False)).astype(np.int64)
    return Workload("w5_spirals_2e6", x.astype(np.float32), y.astype(np.float32),
                    _uniform_weights(n), _uniform_weights(m), eps=1e-3, scale="max_cost",
                    n_iters=100, block_rows=block_rows, rows=rows)


ALL = {"w1": w1, "w2": w2, "w3": w3, "w4": w4, "w5": w5}
