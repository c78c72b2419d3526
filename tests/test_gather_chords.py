"""The gather adjoint's reading of the Siddon coefficients, on the CPU.

For parallel rays in z-planes the coefficient of column c's ray and cell
(x, y) is the chord of a line through a rectangle, a trapezoid in the line's
offset from the cell centre (the reading the gather adjoint computes).  Here
that closed form, restated in numpy, with the sinogram summed over the rows
of each slice, reproduces the FP64 oracle's back projection, which merges
plane crossings instead; a slope taken from the wrong combination of the
direction's components does not.  No CUDA is involved."""
import math

import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import workloads as W


def _view(g, v):
    cc, rc = 0.5 * (g.n_cols - 1), 0.5 * (g.n_rows - 1)
    s = g.src[v] / np.linalg.norm(g.src[v])
    p00 = g.det_c[v] - cc * g.det_u[v] - rc * g.det_v[v]
    return s, p00, g.det_u[v], g.det_v[v]


def chord(delta, dx, dy, slope_mistake=False):
    """Chord of a line of direction (dx, dy) (voxel units per unit length)
    through the unit cell whose centre lies at offset delta from the line
    (delta measured along (-dy, dx))."""
    adx, ady = abs(dx), abs(dy)
    w = 0.5 * (adx + ady)
    lmax = min(1.0 / adx if adx else math.inf, 1.0 / ady if ady else math.inf)
    if adx == 0.0 or ady == 0.0:
        return np.where(np.abs(delta) < w, lmax, 0.0)
    slope = (adx + ady) if slope_mistake else adx * ady
    return np.clip((w - np.abs(delta)) / slope, 0.0, lmax)


def back_by_chords(g, sino, slope_mistake=False):
    org, inv = np.array(g.origin), 1.0 / np.array(g.spacing)
    X, Y = np.meshgrid(np.arange(g.nx) + 0.5, np.arange(g.ny) + 0.5)
    cols, rows = np.arange(g.n_cols), np.arange(g.n_rows)
    out = np.zeros(g.vol_shape)
    for v in range(g.n_views):
        s, p00, du, dv = _view(g, v)
        # slice sums: rows whose height falls in slice z, per column
        az = ((rows[:, None] * dv[2] + cols[None, :] * du[2] + p00[2]) - org[2]) * inv[2]
        inside = (az >= 0) & (az < g.nz)
        k = np.clip(np.floor(az).astype(int), 0, g.nz - 1)
        ysum = np.zeros((g.n_cols, g.nz))
        for r in range(g.n_rows):
            m = inside[r]
            np.add.at(ysum, (cols[m], k[r, m]), sino[v, r, m].astype(np.float64))
        Dx, Dy = s[0] * inv[0], s[1] * inv[1]
        for c in range(g.n_cols):
            ax = ((c * du[0] + p00[0]) - org[0]) * inv[0]
            ay = ((c * du[1] + p00[1]) - org[1]) * inv[1]
            delta = -Dy * (X - ax) + Dx * (Y - ay)
            L = chord(delta, Dx, Dy, slope_mistake)
            out += L[None, :, :] * ysum[c][:, None, None]
    return out


def geometries():
    gs = {
        "anisotropic": W.make_parallel(14, 11, 6, 5, 9, 19, pitch_u=1.1, pitch_v=0.9, spacing=(1.0, 1.1, 0.95),
                                       start=0.05),
        "rows_finer_than_slices": W.make_parallel(12, 10, 5, 4, 13, 17, pitch_u=0.8, pitch_v=0.45, start=0.3),
        "axis_views": W.make_parallel(10, 10, 4, 4, 4, 10),
    }
    src, dc, du, dv = W.parallel_trajectory(4, start=0.4)
    du[:, 2] = 0.07  # a row's slice changes along the row
    gs["slanted_rows"] = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, 9, 15, src, dc, du, dv, 12, 9, 7,
                                    W.centred_origin(12, 9, 7), (1.0, 1.0, 1.0))
    return gs


@pytest.mark.parametrize("name", sorted(geometries()))
def test_trapezoid_chords_reproduce_the_oracle_back_projection(name):
    g = geometries()[name]
    sino = np.random.default_rng(3).random(g.sino_shape).astype(np.float32)
    ref = oracle.back(g, sino)
    got = back_by_chords(g, sino)
    assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()


def test_a_wrong_slope_fails():
    g = geometries()["anisotropic"]
    sino = np.random.default_rng(3).random(g.sino_shape).astype(np.float32)
    ref = oracle.back(g, sino)
    bad = back_by_chords(g, sino, slope_mistake=True)
    assert np.abs(bad - ref).max() > 1e-2 * np.abs(ref).max()


def test_chord_profile_integrates_to_the_cell_area():
    for theta in (0.0, 0.1, 0.7, math.pi / 4, 1.3):
        dx, dy = math.cos(theta), math.sin(theta)
        d = np.linspace(-1.0, 1.0, 200001)  # step 1e-5: the axis view's profile is a step
        area = np.trapezoid(chord(d, dx, dy), d) * math.hypot(dx, dy)
        assert abs(area - 1.0) < 3e-5, theta
