"""Seeded synthetic inputs for the exact-budget LapSum soft top-k.

This module only draws numbers: it holds none of the operator's arithmetic,
so both the CUDA path and the fp64 oracle can take their inputs from it.

Every generator uses numpy's PCG64 (``numpy.random.default_rng``), draws in
fp64 and casts to fp32, so the oracle and the GPU read identical fp32 buffers.
Scores use seed 0 and the upstream gradient ``g`` uses seed 1 unless a caller
asks otherwise.

The five workloads (rows x n, distribution, k, alpha):

=====  ===============  ======================================================  =========  =====
name   shape            scores                                                  k          alpha
=====  ===============  ======================================================  =========  =====
c1     1 x 4096         i.i.d. N(0,1)                                           64         1.0
c2     1 x 1e6          i.i.d. N(0,1)                                           1e4        0.1
c3     1 x 1e7          mixture: 99% N(0,1), 1% N(4, sd 0.5)                    1e5        0.05
c4     1 x 1e8          i.i.d. Uniform[0,1)                                     1e6        1e-3
c5     2048 x 16384     N(0,1); rows with row % 4 == 3 quantised to the 16      256        0.5
                        levels -2 + 4j/15 after clipping to [-2, 2]
=====  ===============  ======================================================  =========  =====

The sizes are those the Fast LapSum abstract times (1e6, 1e7, 1e8 scores) plus
a small single row and a tied batch that exercises wide bands.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_scores", "make_grad", "workload"]


@dataclass(frozen=True)
class Workload:
    name: str
    rows: int
    n: int
    dist: str
    k: float
    alpha: float

    @property
    def shape(self):
        return (self.rows, self.n)

    def scaled(self, n: int | None = None, rows: int | None = None) -> "Workload":
        """Same distribution at another size; k keeps its ratio to n."""
        n2 = self.n if n is None else int(n)
        r2 = self.rows if rows is None else int(rows)
        k2 = self.k * n2 / self.n
        return Workload(self.name, r2, n2, self.dist, k2, self.alpha)


WORKLOADS = {
    "c1": Workload("c1", 1, 4096, "normal", 64.0, 1.0),
    "c2": Workload("c2", 1, 1_000_000, "normal", 10_000.0, 0.1),
    "c3": Workload("c3", 1, 10_000_000, "mixture", 100_000.0, 0.05),
    "c4": Workload("c4", 1, 100_000_000, "uniform", 1_000_000.0, 1e-3),
    "c5": Workload("c5", 2048, 16384, "tied_batch", 256.0, 0.5),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _quantise_rows(x: np.ndarray) -> np.ndarray:
    """Clip to [-2, 2] and snap to the nearest of 16 equally spaced levels."""
    q = np.clip(x, -2.0, 2.0)
    idx = np.rint((q + 2.0) * (15.0 / 4.0))
    return -2.0 + idx * (4.0 / 15.0)


def make_scores(dist: str | Workload, rows: int = 1, n: int = 0, seed: int = 0) -> np.ndarray:
    """fp32 array of shape (rows, n) drawn from the named distribution."""
    if isinstance(dist, Workload):
        rows, n, dist = dist.rows, dist.n, dist.dist
    rng = np.random.default_rng(seed)
    shape = (rows, n)
    if dist == "normal":
        x = rng.standard_normal(shape)
    elif dist == "uniform":
        x = rng.random(shape)
    elif dist == "mixture":
        z = rng.standard_normal(shape)
        u = rng.random(shape)
        x = np.where(u < 0.01, 4.0 + 0.5 * z, z)
    elif dist == "tied_batch":
        x = rng.standard_normal(shape)
        tied = (np.arange(rows) % 4) == 3
        x[tied] = _quantise_rows(x[tied])
    elif dist == "all_tied":
        x = np.full(shape, 0.25)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return np.ascontiguousarray(x.astype(np.float32))


def make_grad(rows: int, n: int, seed: int = 1) -> np.ndarray:
    """Upstream gradient g ~ N(0,1), fp32, shape (rows, n)."""
    rng = np.random.default_rng(seed)
    return np.ascontiguousarray(rng.standard_normal((rows, n)).astype(np.float32))
