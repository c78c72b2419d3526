"""Seeded synthetic inputs: acquisition trajectories and voxel phantoms.

This module only builds inputs.  It holds none of the projector's arithmetic
(no pixel-centre expansion, no clipping, no traversal): it writes per-view
vectors and volumes that both the CUDA library and the FP64 oracle consume.

Conventions (diffct "Execution", section "Batch dimensions and axis spacing"):
trajectory coordinates are world (x, y, z); volumes are stored as tensors of
shape (nz, ny, nx), x fastest; sinograms as (n_views, n_rows, n_cols), column
fastest.

Per-view vectors, each float64 of shape (n_views, 3):
  * ``src``   cone beam: source position.  Parallel beam: ray direction.
  * ``det_c`` centre of the detector (between the middle pixels when a count
              is even).
  * ``det_u`` column step; its length is the column pitch (the arc pitch on a
              cylindrical detector).
  * ``det_v`` row step; its length is the row pitch.

The volume's ``origin`` is the world position of the minimum corner of voxel
(0, 0, 0) and ``spacing`` is the per-axis pitch (dx, dy, dz).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BEAM_PARALLEL = 0
BEAM_CONE = 1
DET_FLAT = 0
DET_CYLINDRICAL = 1


@dataclasses.dataclass
class Geometry:
    beam: int
    detector: int
    n_rows: int
    n_cols: int
    src: np.ndarray
    det_c: np.ndarray
    det_u: np.ndarray
    det_v: np.ndarray
    nx: int
    ny: int
    nz: int
    origin: tuple
    spacing: tuple

    @property
    def n_views(self) -> int:
        return int(self.src.shape[0])

    @property
    def vol_shape(self) -> tuple:
        return (self.nz, self.ny, self.nx)

    @property
    def sino_shape(self) -> tuple:
        return (self.n_views, self.n_rows, self.n_cols)

    @property
    def n_rays(self) -> int:
        return self.n_views * self.n_rows * self.n_cols

    @property
    def n_vox(self) -> int:
        return self.nx * self.ny * self.nz

    def subset_views(self, views) -> "Geometry":
        """The same acquisition restricted to the listed view indices."""
        views = np.asarray(views, dtype=np.int64)
        return dataclasses.replace(
            self,
            src=np.ascontiguousarray(self.src[views]),
            det_c=np.ascontiguousarray(self.det_c[views]),
            det_u=np.ascontiguousarray(self.det_u[views]),
            det_v=np.ascontiguousarray(self.det_v[views]),
        )


def centred_origin(nx, ny, nz, spacing=(1.0, 1.0, 1.0)):
    """Origin that puts the volume centre at the world origin."""
    return (-0.5 * nx * spacing[0], -0.5 * ny * spacing[1], -0.5 * nz * spacing[2])


def parallel_trajectory(n_views, arc=math.pi, pitch_u=1.0, pitch_v=1.0, start=0.0):
    """Parallel beam rotating about z: views at start + k*arc/n_views.

    Ray direction (cos t, sin t, 0); detector u = (-sin t, cos t, 0)*pitch_u,
    v = (0, 0, 1)*pitch_v; detector centred on the rotation axis.
    """
    th = start + np.arange(n_views, dtype=np.float64) * (arc / n_views)
    c, s = np.cos(th), np.sin(th)
    z = np.zeros_like(th)
    src = np.stack([c, s, z], axis=1)
    det_c = np.zeros((n_views, 3))
    det_u = np.stack([-s, c, z], axis=1) * pitch_u
    det_v = np.stack([z, z, np.ones_like(th)], axis=1) * pitch_v
    return src, det_c, det_u, det_v


def cone_trajectory(n_views, sid, sdd, pitch_u=1.0, pitch_v=1.0, arc=2 * math.pi,
                    z_start=0.0, z_end=None, start=0.0):
    """Circular (z_end is None) or helical cone-beam source path about z.

    Source s = (sid cos t, sid sin t, z_k); detector centre s - sdd*(cos t, sin t, 0);
    u = (-sin t, cos t, 0)*pitch_u; v = (0, 0, 1)*pitch_v.  For a helix the
    source z runs linearly from z_start (first view) to z_end (last view).
    """
    th = start + np.arange(n_views, dtype=np.float64) * (arc / n_views)
    c, s = np.cos(th), np.sin(th)
    if z_end is None:
        zs = np.full_like(th, z_start)
    else:
        zs = z_start + (z_end - z_start) * np.arange(n_views, dtype=np.float64) / max(n_views - 1, 1)
    zero = np.zeros_like(th)
    src = np.stack([sid * c, sid * s, zs], axis=1)
    det_c = src - sdd * np.stack([c, s, zero], axis=1)
    det_u = np.stack([-s, c, zero], axis=1) * pitch_u
    det_v = np.stack([zero, zero, np.ones_like(th)], axis=1) * pitch_v
    return src, det_c, det_u, det_v


def _random_rotation(rng):
    """Uniform random rotation from a normalised Gaussian quaternion."""
    q = rng.standard_normal(4)
    q /= np.linalg.norm(q)
    w, x, y, z = q
    return np.array([
        [1 - 2 * (y * y + z * z), 2 * (x * y - z * w), 2 * (x * z + y * w)],
        [2 * (x * y + z * w), 1 - 2 * (x * x + z * z), 2 * (y * z - x * w)],
        [2 * (x * z - y * w), 2 * (y * z + x * w), 1 - 2 * (x * x + y * y)],
    ])


@dataclasses.dataclass
class Ellipsoid:
    centre: np.ndarray      # world (x, y, z)
    semi_axes: np.ndarray   # world lengths along the body axes
    rotation: np.ndarray    # columns are the body axes in world coordinates
    density: float


def random_ellipsoids(rng, n, nx, ny, nz, origin, spacing):
    """n ellipsoids: semi-axes in [n_k/16, 5 n_k/16] voxels per axis, densities
    U[0.5, 2], uniform random orientation, centres uniform in the box shrunk by
    the largest semi-axis."""
    dims = np.array([nx, ny, nz], dtype=np.float64)
    sp = np.asarray(spacing, dtype=np.float64)
    lo = np.asarray(origin, dtype=np.float64)
    hi = lo + dims * sp
    out = []
    for _ in range(n):
        semi = rng.uniform(dims / 16.0, 5.0 * dims / 16.0) * sp
        rot = _random_rotation(rng)
        rmax = float(semi.max())
        c_lo = np.minimum(lo + rmax, 0.5 * (lo + hi))
        c_hi = np.maximum(hi - rmax, 0.5 * (lo + hi))
        centre = rng.uniform(c_lo, c_hi)
        dens = float(rng.uniform(0.5, 2.0))
        out.append(Ellipsoid(centre, semi, rot, dens))
    return out


def rasterise_ellipsoids(vol, ellipsoids, origin, spacing):
    """Add each ellipsoid's density to the voxels whose centres lie inside it."""
    nz, ny, nx = vol.shape
    o = np.asarray(origin, dtype=np.float64)
    sp = np.asarray(spacing, dtype=np.float64)
    for e in ellipsoids:
        r = float(e.semi_axes.max())
        lo_idx = np.floor((e.centre - r - o) / sp - 0.5).astype(np.int64)
        hi_idx = np.ceil((e.centre + r - o) / sp - 0.5).astype(np.int64) + 1
        lo_idx = np.clip(lo_idx, 0, [nx, ny, nz])
        hi_idx = np.clip(hi_idx, 0, [nx, ny, nz])
        if np.any(hi_idx <= lo_idx):
            continue
        xs = o[0] + (np.arange(lo_idx[0], hi_idx[0]) + 0.5) * sp[0] - e.centre[0]
        ys = o[1] + (np.arange(lo_idx[1], hi_idx[1]) + 0.5) * sp[1] - e.centre[1]
        zs = o[2] + (np.arange(lo_idx[2], hi_idx[2]) + 0.5) * sp[2] - e.centre[2]
        Z, Y, X = np.meshgrid(zs, ys, xs, indexing="ij")
        # body coordinates: rotation^T * (p - c)
        R = e.rotation
        bx = R[0, 0] * X + R[1, 0] * Y + R[2, 0] * Z
        by = R[0, 1] * X + R[1, 1] * Y + R[2, 1] * Z
        bz = R[0, 2] * X + R[1, 2] * Y + R[2, 2] * Z
        inside = (bx / e.semi_axes[0]) ** 2 + (by / e.semi_axes[1]) ** 2 + (bz / e.semi_axes[2]) ** 2 <= 1.0
        sl = (slice(lo_idx[2], hi_idx[2]), slice(lo_idx[1], hi_idx[1]), slice(lo_idx[0], hi_idx[0]))
        vol[sl] += (inside * e.density).astype(vol.dtype)
    return vol


@dataclasses.dataclass
class Workload:
    name: str
    index: int
    geom: Geometry
    n_ellipsoids: int
    noise: float            # background U[0, noise) (0 = none)
    seed: int

    def phantom(self) -> np.ndarray:
        """The FP32 volume (nz, ny, nx) for this workload, from its seed."""
        g = self.geom
        rng = np.random.Generator(np.random.PCG64(self.seed))
        if self.noise > 0:
            vol = (rng.random((g.nz, g.ny, g.nx), dtype=np.float32) * np.float32(self.noise))
        else:
            vol = np.zeros((g.nz, g.ny, g.nx), dtype=np.float32)
        ells = random_ellipsoids(rng, self.n_ellipsoids, g.nx, g.ny, g.nz, g.origin, g.spacing)
        return rasterise_ellipsoids(vol, ells, g.origin, g.spacing)

    def sinogram(self, seed_offset=7) -> np.ndarray:
        """A seeded FP32 sinogram U[0, 1) of this workload's shape (adjoint input)."""
        rng = np.random.Generator(np.random.PCG64(self.seed + seed_offset))
        return rng.random(self.geom.sino_shape, dtype=np.float32)


def make_parallel(nx, ny, nz, n_views, n_rows, n_cols, pitch_u=1.0, pitch_v=1.0,
                  spacing=(1.0, 1.0, 1.0), arc=math.pi, start=0.0, origin=None):
    src, dc, du, dv = parallel_trajectory(n_views, arc, pitch_u, pitch_v, start)
    if origin is None:
        origin = centred_origin(nx, ny, nz, spacing)
    return Geometry(BEAM_PARALLEL, DET_FLAT, n_rows, n_cols, src, dc, du, dv,
                    nx, ny, nz, tuple(origin), tuple(spacing))


def make_cone(nx, ny, nz, n_views, n_rows, n_cols, sid, sdd, pitch_u=1.0, pitch_v=1.0,
              spacing=(1.0, 1.0, 1.0), arc=2 * math.pi, detector=DET_FLAT,
              z_start=0.0, z_end=None, start=0.0, origin=None):
    src, dc, du, dv = cone_trajectory(n_views, sid, sdd, pitch_u, pitch_v, arc, z_start, z_end, start)
    if origin is None:
        origin = centred_origin(nx, ny, nz, spacing)
    return Geometry(BEAM_CONE, detector, n_rows, n_cols, src, dc, du, dv,
                    nx, ny, nz, tuple(origin), tuple(spacing))


def helical_fan_pitch(n_cols, fov_half_width, radius, sdd):
    """Arc pitch of a cylindrical detector centred on the source whose n_cols
    columns span the fan that just covers a circle of the given half-width."""
    gamma_max = math.asin(fov_half_width / radius)
    return sdd * (2.0 * gamma_max / n_cols)


def workload(index: int) -> Workload:
    """The five seeded workloads (seed = 1000 + index)."""
    seed = 1000 + index
    if index == 0:
        g = make_parallel(64, 64, 64, 64, 64, 64)
        return Workload("parallel 64^3, 64 views, 64x64 detector", 0, g, 4, 1.0, seed)
    if index == 1:
        g = make_cone(64, 64, 64, 16, 128, 128, sid=1000.0, sdd=2000.0)
        return Workload("cone flat 64^3, 16 views, 128x128, sid 1000 sdd 2000", 1, g, 10, 0.0, seed)
    if index == 2:
        g = make_cone(256, 256, 256, 360, 384, 384, sid=500.0, sdd=1000.0)
        return Workload("cone flat 256^3, 360 views, 384x384, sid 500 sdd 1000", 2, g, 30, 0.05, seed)
    if index == 3:
        pu = helical_fan_pitch(736, 256.0, 595.0, 1085.6)
        g = make_cone(512, 512, 96, 1338, 64, 736, sid=595.0, sdd=1085.6, pitch_u=pu, pitch_v=1.0,
                      detector=DET_CYLINDRICAL, z_start=-48.0, z_end=48.0)
        return Workload("helical cone cylindrical 96x512x512, 1338 views, 64x736", 3, g, 40, 0.0, seed)
    if index == 4:
        g = make_parallel(512, 512, 512, 900, 512, 736)
        return Workload("parallel 512^3, 900 views, 512x736 detector", 4, g, 8, 1.0, seed)
    raise ValueError(f"no workload {index}")


N_WORKLOADS = 5
