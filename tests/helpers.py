"""Shared test helpers: small geometries and independent reference formulas.

Nothing here calls the CUDA library or reuses the oracle's arithmetic; the
brute-force integrator and the ellipsoid chord are written independently of
both so they can pin the oracle.
"""
from __future__ import annotations

import math

import numpy as np

from ray_forward_back_b200 import workloads as W


def brute_force_line_integral(vol, origin, spacing, a, b, n_samples=1_000_000):
    """Midpoint-rule integral of the piecewise-constant volume along a -> b.

    Each sample point is assigned to the voxel containing it (floor), so the
    only error comes from samples that straddle a voxel boundary: at most one
    sample per boundary crossing.  Returns (value, error bound).
    """
    vol = np.asarray(vol, dtype=np.float64)
    nz, ny, nx = vol.shape
    a = np.asarray(a, dtype=np.float64)
    d = np.asarray(b, dtype=np.float64) - a
    L = float(np.linalg.norm(d))
    t = (np.arange(n_samples, dtype=np.float64) + 0.5) / n_samples
    o = np.asarray(origin, dtype=np.float64)
    s = np.asarray(spacing, dtype=np.float64)
    ix = np.floor((a[0] + t * d[0] - o[0]) / s[0]).astype(np.int64)
    iy = np.floor((a[1] + t * d[1] - o[1]) / s[1]).astype(np.int64)
    iz = np.floor((a[2] + t * d[2] - o[2]) / s[2]).astype(np.int64)
    inside = (ix >= 0) & (ix < nx) & (iy >= 0) & (iy < ny) & (iz >= 0) & (iz < nz)
    vals = vol[iz[inside], iy[inside], ix[inside]]
    step = L / n_samples
    value = float(vals.sum()) * step
    # boundaries crossed: changes of voxel id along the samples, plus entry/exit
    vid = np.where(inside, (iz * ny + iy) * nx + ix, -1)
    crossings = int(np.count_nonzero(np.diff(vid))) + 2
    bound = crossings * step * float(np.abs(vol).max() if vol.size else 0.0)
    return value, bound


def ellipsoid_chord(e: W.Ellipsoid, a, b):
    """Length of the segment a -> b inside ellipsoid e (closed form)."""
    a = np.asarray(a, dtype=np.float64)
    d = np.asarray(b, dtype=np.float64) - a
    q0 = e.rotation.T @ (a - e.centre) / e.semi_axes
    qd = e.rotation.T @ d / e.semi_axes
    A = float(qd @ qd)
    B = 2.0 * float(q0 @ qd)
    C = float(q0 @ q0) - 1.0
    disc = B * B - 4 * A * C
    if disc <= 0 or A == 0:
        return 0.0
    r = math.sqrt(disc)
    t1, t2 = (-B - r) / (2 * A), (-B + r) / (2 * A)
    t1, t2 = max(t1, 0.0), min(t2, 1.0)
    return max(t2 - t1, 0.0) * float(np.linalg.norm(d))


def small_geometries():
    """Small geometries of every kind with ragged, unequal sizes and
    anisotropic spacing; none puts a ray inside a voxel-boundary plane."""
    gs = {}
    gs["parallel"] = W.make_parallel(11, 9, 7, 6, 5, 13, pitch_u=0.9, pitch_v=1.1,
                                     spacing=(1.0, 1.2, 0.8), start=0.1)
    g = W.make_cone(10, 12, 9, 5, 7, 11, sid=40.0, sdd=70.0, pitch_u=1.7, pitch_v=1.3,
                    spacing=(1.1, 0.9, 1.0), start=0.3)
    g.det_c = g.det_c + np.array([0.013, -0.021, 0.037])
    gs["cone_flat"] = g
    pu = W.helical_fan_pitch(15, 7.0, 30.0, 55.0)
    g = W.make_cone(12, 10, 8, 7, 6, 15, sid=30.0, sdd=55.0, pitch_u=pu, pitch_v=0.9,
                    spacing=(1.0, 1.05, 0.95), detector=W.DET_CYLINDRICAL,
                    z_start=-3.1, z_end=2.9, start=0.2)
    g.det_c = g.det_c + np.array([0.0, 0.0, 0.37])   # detector centre above the source plane
    gs["helical_cyl"] = g
    return gs
