"""FP64 oracle for the cell-constant Siddon projector pair (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product library.  The C source
(``siddon_oracle.c``) states what is computed and which passage each step
follows; this wrapper only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "siddon_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Geom(ctypes.Structure):
    _fields_ = [
        ("beam", ctypes.c_int32), ("detector", ctypes.c_int32),
        ("n_views", ctypes.c_int64), ("n_rows", ctypes.c_int64), ("n_cols", ctypes.c_int64),
        ("src", ctypes.c_void_p), ("det_c", ctypes.c_void_p),
        ("det_u", ctypes.c_void_p), ("det_v", ctypes.c_void_p),
        ("n", ctypes.c_int64 * 3), ("origin", ctypes.c_double * 3), ("spacing", ctypes.c_double * 3),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(_Geom)
            vp, i64 = ctypes.c_void_p, ctypes.c_int64
            lib.oracle_pixel_centre.argtypes = [P, i64, i64, i64, vp]
            lib.oracle_ray_endpoints.argtypes = [P, i64, i64, i64, vp, vp]
            lib.oracle_forward.argtypes = [P, vp, vp, i64, i64]
            lib.oracle_forward.restype = ctypes.c_int
            lib.oracle_forward_rays.argtypes = [P, vp, i64, vp, vp, vp, vp]
            lib.oracle_forward_rays.restype = ctypes.c_int
            lib.oracle_back.argtypes = [P, vp, vp, i64, i64, ctypes.c_int]
            lib.oracle_back.restype = ctypes.c_int
            lib.oracle_ray_segments.argtypes = [P, i64, i64, i64, vp, vp, i64]
            lib.oracle_ray_segments.restype = i64
            lib.oracle_count_updates.argtypes = [P, i64, i64]
            lib.oracle_count_updates.restype = i64
            _lib = lib
    return _lib


class _Bound:
    """Keeps the geometry arrays alive while the C struct points at them."""

    def __init__(self, geom):
        self.arrays = [np.ascontiguousarray(a, dtype=np.float64) for a in
                       (geom.src, geom.det_c, geom.det_u, geom.det_v)]
        g = _Geom()
        g.beam, g.detector = int(geom.beam), int(geom.detector)
        g.n_views, g.n_rows, g.n_cols = int(geom.n_views), int(geom.n_rows), int(geom.n_cols)
        g.src, g.det_c, g.det_u, g.det_v = [a.ctypes.data for a in self.arrays]
        g.n[:] = [int(geom.nx), int(geom.ny), int(geom.nz)]
        g.origin[:] = [float(x) for x in geom.origin]
        g.spacing[:] = [float(x) for x in geom.spacing]
        self.g = g

    @property
    def ptr(self):
        return ctypes.byref(self.g)


def pixel_centre(geom, v, r, c):
    b = _Bound(geom)
    p = np.zeros(3)
    _load().oracle_pixel_centre(b.ptr, v, r, c, p.ctypes.data)
    return p


def ray_endpoints(geom, v, r, c):
    b = _Bound(geom)
    a, e = np.zeros(3), np.zeros(3)
    _load().oracle_ray_endpoints(b.ptr, v, r, c, a.ctypes.data, e.ctypes.data)
    return a, e


def forward(geom, vol, views=None) -> np.ndarray:
    """y = A x in FP64 for views [v0, v1) (all by default); vol is promoted
    from float32 exactly."""
    v0, v1 = (0, geom.n_views) if views is None else views
    vol = np.ascontiguousarray(vol, dtype=np.float32)
    assert vol.shape == geom.vol_shape
    out = np.zeros((v1 - v0, geom.n_rows, geom.n_cols), dtype=np.float64)
    b = _Bound(geom)
    if _load().oracle_forward(b.ptr, vol.ctypes.data, out.ctypes.data, v0, v1) != 0:
        raise MemoryError("oracle_forward")
    return out


def forward_rays(geom, vol, vs, rs, cs) -> np.ndarray:
    """Forward values of the listed rays (v, r, c)."""
    vol = np.ascontiguousarray(vol, dtype=np.float32)
    vs, rs, cs = [np.ascontiguousarray(x, dtype=np.int64) for x in (vs, rs, cs)]
    out = np.zeros(vs.shape[0], dtype=np.float64)
    b = _Bound(geom)
    if _load().oracle_forward_rays(b.ptr, vol.ctypes.data, vs.shape[0], vs.ctypes.data, rs.ctypes.data,
                                   cs.ctypes.data, out.ctypes.data) != 0:
        raise MemoryError("oracle_forward_rays")
    return out


def back(geom, sino, views=None, power: int = 1) -> np.ndarray:
    """x = A^T y in FP64 (coefficient ** power; power 0 counts segments).
    ``sino`` holds exactly the views [v0, v1)."""
    v0, v1 = (0, geom.n_views) if views is None else views
    sino = np.ascontiguousarray(sino, dtype=np.float32)
    assert sino.shape == (v1 - v0, geom.n_rows, geom.n_cols)
    out = np.zeros(geom.vol_shape, dtype=np.float64)
    b = _Bound(geom)
    if _load().oracle_back(b.ptr, sino.ctypes.data, out.ctypes.data, v0, v1, int(power)) != 0:
        raise MemoryError("oracle_back")
    return out


def ray_segments(geom, v, r, c):
    """(flat voxel indices, physical lengths) of one ray's positive segments."""
    b = _Bound(geom)
    cap = geom.nx + geom.ny + geom.nz + 8
    idx = np.zeros(cap, dtype=np.int64)
    w = np.zeros(cap, dtype=np.float64)
    n = _load().oracle_ray_segments(b.ptr, v, r, c, idx.ctypes.data, w.ctypes.data, cap)
    if n < 0:
        raise MemoryError("oracle_ray_segments")
    return idx[:n].copy(), w[:n].copy()


def count_updates(geom, views=None) -> int:
    """Exact number of positive-length ray-voxel segments (the work count)."""
    v0, v1 = (0, geom.n_views) if views is None else views
    b = _Bound(geom)
    n = _load().oracle_count_updates(b.ptr, v0, v1)
    if n < 0:
        raise MemoryError("oracle_count_updates")
    return int(n)


def dense_matrix(geom) -> np.ndarray:
    """System matrix A (n_rays x n_vox) assembled row by row from ray_segments."""
    A = np.zeros((geom.n_rays, geom.n_vox))
    q = 0
    for v in range(geom.n_views):
        for r in range(geom.n_rows):
            for c in range(geom.n_cols):
                idx, w = ray_segments(geom, v, r, c)
                np.add.at(A[q], idx, w)
                q += 1
    return A
