"""Seeded synthetic inputs for the hash-grid encoding: tables, points, upstream gradients.

This module is shared by the tests, the benchmark and the smoke check. It holds none of
the encoding's arithmetic (no resolution, hash, interpolation or gradient): only the
workload descriptions and numpy draws, in one fixed order per workload, so that the CUDA
path and the CPU oracle are fed identical bytes.

Workloads (the pages' encoder hyper-parameters; NeRF ray samples as the point source):
  tiny_L4F2T10        L=4  F=2 T=2^10 N 2->16,   4096 uniform points, fwd + bwd
  grid_L16F2T19       L=16 F=2 T=2^19 N 16->512, 2^18 uniform points, fwd only
  rays_L16F2T19       same grid, 2^14 rays x 64 stratified samples (2^20 points), fwd + bwd
  half_L16F2T19       same grid, fp16 table, 2^22 uniform points, fwd + bwd
  large_L16F4T22      L=16 F=4 T=2^22 N 16->4096 (1 GiB fp32 table), 2^16 rays x 64, fwd + bwd

Draw order for one workload, all from ``numpy.random.default_rng(seed)``:
  1. table: U[0,1) fp32 draws mapped to (2u - 1) * 1e-4 in fp32 (so values lie in
     [-1e-4, 1e-4)); an fp16 table is that fp32 array rounded to nearest-even fp16;
  2. points: uniform -> U[0,1)^3 fp32 draws; rays -> see ``ray_points``;
  3. upstream gradients (fwd + bwd workloads): standard normal fp32 [N, L*F].
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    L: int
    F: int
    log2T: int
    N_min: int
    N_max: int
    dtype: str          # "f32" or "f16" table storage
    points: str         # "uniform" or "rays"
    n_points: int
    samples_per_ray: int = 64
    backward: bool = True

    @property
    def T(self) -> int:
        return 1 << self.log2T

    @property
    def n_rays(self) -> int:
        assert self.points == "rays"
        return self.n_points // self.samples_per_ray

    def describe(self) -> str:
        pts = (f"{self.n_points} uniform points" if self.points == "uniform" else
               f"{self.n_rays} rays x {self.samples_per_ray} samples")
        return (f"L={self.L} F={self.F} T=2^{self.log2T} N_min={self.N_min} N_max={self.N_max} "
                f"{self.dtype} table; {pts}; {'fwd+bwd' if self.backward else 'fwd'}")


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_L4F2T10", 4, 2, 10, 2, 16, "f32", "uniform", 4096),
        Workload("grid_L16F2T19", 16, 2, 19, 16, 512, "f32", "uniform", 1 << 18, backward=False),
        Workload("rays_L16F2T19", 16, 2, 19, 16, 512, "f32", "rays", 1 << 20),
        Workload("half_L16F2T19", 16, 2, 19, 16, 512, "f16", "uniform", 1 << 22),
        Workload("large_L16F4T22", 16, 4, 22, 16, 4096, "f32", "rays", 1 << 22),
    ]
}


def table_values(rng: np.random.Generator, L: int, T: int, F: int, dtype: str = "f32") -> np.ndarray:
    """[L, T, F] table in [-1e-4, 1e-4): fp32, or those values rounded to fp16."""
    u = rng.random(L * T * F, dtype=np.float32)
    t = (u * np.float32(2.0) - np.float32(1.0)) * np.float32(1e-4)
    t = t.reshape(L, T, F)
    if dtype == "f16":
        return t.astype(np.float16)
    return t


def uniform_points(rng: np.random.Generator, n: int) -> np.ndarray:
    """[n, 3] fp32 points, uniform in [0, 1)^3."""
    return rng.random((n, 3), dtype=np.float32)


def ray_points(rng: np.random.Generator, n_rays: int, samples: int = 64) -> np.ndarray:
    """[n_rays * samples, 3] fp32 samples along random rays through the unit cube.

    Origin o = (0.5, 0.5, 0.5) + 1.5 u with u uniform on the unit sphere (a normalised
    standard-normal draw); the ray aims at q ~ U[0.25, 0.75]^3, direction d = q - o. The
    ray's interval [t_in, t_out] inside [0, 1]^3 comes from the slab test, and sample k
    sits at t_in + (k + u_k)/samples * (t_out - t_in), u_k ~ U[0, 1) (stratified). Samples
    are clamped per axis to [0, 1 - 2^-24] and stored ray-major (index r*samples + k).
    """
    u = rng.standard_normal((n_rays, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    o = 0.5 + 1.5 * u
    q = rng.uniform(0.25, 0.75, size=(n_rays, 3))
    d = q - o
    d = np.where(np.abs(d) < 1e-12, 1e-12, d)
    t0 = (0.0 - o) / d
    t1 = (1.0 - o) / d
    t_in = np.max(np.minimum(t0, t1), axis=1)
    t_out = np.min(np.maximum(t0, t1), axis=1)
    uk = rng.random((n_rays, samples))
    k = np.arange(samples, dtype=np.float64)[None, :]
    t = t_in[:, None] + (k + uk) / samples * (t_out - t_in)[:, None]
    p = o[:, None, :] + t[:, :, None] * d[:, None, :]
    p = np.clip(p, 0.0, 1.0 - 2.0 ** -24)
    return p.reshape(-1, 3).astype(np.float32)


def upstream_grads(rng: np.random.Generator, n: int, width: int) -> np.ndarray:
    """[n, width] fp32 standard-normal upstream gradients."""
    return rng.standard_normal((n, width), dtype=np.float32)


@dataclass
class Inputs:
    table: np.ndarray          # [L, T, F] float32 or float16
    x: np.ndarray              # [N, 3] float32
    g: np.ndarray | None       # [N, L*F] float32 or None


def make_inputs(w: Workload, seed: int = 0, n_points: int | None = None,
                grads: bool | None = None) -> Inputs:
    """All inputs of workload ``w`` in the fixed draw order. ``n_points`` overrides the
    point count (for rays: rounded up to whole rays); ``grads`` overrides whether the
    upstream gradients are drawn (default: the workload's own ``backward`` flag)."""
    rng = np.random.default_rng(seed)
    table = table_values(rng, w.L, w.T, w.F, w.dtype)
    n = w.n_points if n_points is None else n_points
    if w.points == "uniform":
        x = uniform_points(rng, n)
    else:
        n_rays = -(-n // w.samples_per_ray)
        x = ray_points(rng, n_rays, w.samples_per_ray)[:n]
    want_g = w.backward if grads is None else grads
    g = upstream_grads(rng, x.shape[0], w.L * w.F) if want_g else None
    return Inputs(table, np.ascontiguousarray(x), g)
