"""FP64 reference for geometry gradients: central finite differences of the
oracle's forward projection.

TEST INFRASTRUCTURE ONLY (imported by the tests, never by the library).

For an upstream gradient g = dL/dy on the sinogram, the gradient of L with
respect to view v's vectors (src, det_c, det_u, det_v), each a 3-vector, is
sum over the view's rays of g * dy/dtheta (diffct "Execution", section
"Streaming analytical reconstruction": geometry gradients of the
projection).  The Siddon line integral is piecewise linear in the geometry
(its kinks are where a ray meets a voxel edge), so a central difference with
a small step is exact up to rounding away from kinks.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import forward

FIELDS = ("src", "det_c", "det_u", "det_v")


def geometry_gradient_fd(geom, vol, g, h=1e-6):
    """Array [n_views][4][3]: dL/d(src, det_c, det_u, det_v) of every view.

    A step on det_u (det_v) moves pixel column c (row r) by (c - cc) (or
    (r - rc)) times the step, so those steps are divided by the largest such
    factor: no pixel moves by more than h, and a wide detector does not carry
    its outer rays across the kinks of the piecewise-linear line integral."""
    g = np.asarray(g, dtype=np.float64)
    out = np.zeros((geom.n_views, 4, 3))
    lever = {"src": 1.0, "det_c": 1.0,
             "det_u": max(0.5 * (geom.n_cols - 1), 1.0), "det_v": max(0.5 * (geom.n_rows - 1), 1.0)}
    for v in range(geom.n_views):
        one = geom.subset_views([v])
        for f, name in enumerate(FIELDS):
            hf = h / lever[name]
            for k in range(3):
                vals = []
                for sgn in (1.0, -1.0):
                    arr = getattr(one, name).copy()
                    arr[0, k] += sgn * hf
                    pert = dataclasses.replace(one, **{name: arr})
                    vals.append(forward(pert, vol)[0])
                out[v, f, k] = float((g[v] * (vals[0] - vals[1])).sum()) / (2 * hf)
    return out
