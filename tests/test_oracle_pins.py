"""Pins of the FP64 oracle against facts that do not come from the oracle.

Each test names what fixes its expected value: a closed form, a textbook
reduction, brute-force integration, a convergence order, or a geometric
property of the detector model.  Runs on CPU only.
"""
import math

import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import workloads as W
from tests.helpers import brute_force_line_integral, ellipsoid_chord, small_geometries


# ---------------------------------------------------------------- geometry ---

def test_flat_pixel_centres_are_affine_in_row_and_column():
    """Flat detector: pixel centres form the lattice det_c + a*u + b*v whose
    mean is det_c (detector centre) and whose steps are det_u, det_v."""
    g = small_geometries()["cone_flat"]
    for v in (0, 3):
        P = np.array([[oracle.pixel_centre(g, v, r, c) for c in range(g.n_cols)] for r in range(g.n_rows)])
        np.testing.assert_allclose(P.reshape(-1, 3).mean(axis=0), g.det_c[v], atol=1e-12)
        np.testing.assert_allclose(P[:, 1:] - P[:, :-1], np.broadcast_to(g.det_u[v], P[:, 1:].shape), atol=1e-12)
        np.testing.assert_allclose(P[1:, :] - P[:-1, :], np.broadcast_to(g.det_v[v], P[1:, :].shape), atol=1e-12)


def test_cylindrical_pixel_centres_lie_on_the_source_centred_cylinder():
    """Cylindrical detector: every pixel centre is at distance R from the axis
    through the source along det_v, adjacent columns subtend |u|/R, the middle
    column of an odd count sits at det_c, rows step by det_v."""
    g = small_geometries()["helical_cyl"]
    assert g.n_cols % 2 == 1
    for v in (0, 4):
        s, dc, du, dv = g.src[v], g.det_c[v], g.det_u[v], g.det_v[v]
        vh = dv / np.linalg.norm(dv)
        w = dc - s
        R = np.linalg.norm(w - (w @ vh) * vh)
        P = np.array([[oracle.pixel_centre(g, v, r, c) for c in range(g.n_cols)] for r in range(g.n_rows)])
        rel = P - s
        perp = rel - (rel @ vh)[..., None] * vh
        np.testing.assert_allclose(np.linalg.norm(perp, axis=-1), R, rtol=1e-12)
        chord = np.linalg.norm(perp[:, 1:] - perp[:, :-1], axis=-1)
        np.testing.assert_allclose(chord, 2 * R * math.sin(np.linalg.norm(du) / (2 * R)), rtol=1e-10)
        mid = g.n_cols // 2
        rmid = (g.n_rows - 1) / 2
        for r in range(g.n_rows):
            np.testing.assert_allclose(P[r, mid], dc + (r - rmid) * dv, atol=1e-10)
        # the column angle increases along +u
        assert (perp[0, mid + 1] - perp[0, mid]) @ du > 0


def test_ray_endpoints_cone_and_parallel():
    """Cone: the ray runs from the source to the pixel centre.  Parallel: the
    endpoints lie on the line through the pixel centre along the view
    direction, on opposite sides, both outside the volume box."""
    g = small_geometries()["cone_flat"]
    a, b = oracle.ray_endpoints(g, 2, 3, 4)
    np.testing.assert_array_equal(a, g.src[2])
    np.testing.assert_array_equal(b, oracle.pixel_centre(g, 2, 3, 4))
    g = small_geometries()["parallel"]
    lo = np.array(g.origin)
    hi = lo + np.array([g.nx, g.ny, g.nz]) * np.array(g.spacing)
    for v, r, c in [(0, 0, 0), (3, 2, 7), (5, 4, 12)]:
        a, b = oracle.ray_endpoints(g, v, r, c)
        p = oracle.pixel_centre(g, v, r, c)
        dhat = g.src[v] / np.linalg.norm(g.src[v])
        np.testing.assert_allclose(np.cross(b - a, dhat), 0, atol=1e-9)
        np.testing.assert_allclose(np.cross(p - a, dhat), 0, atol=1e-9)
        assert (b - a) @ dhat > 0 and (p - a) @ dhat > 0 and (b - p) @ dhat > 0
        for e in (a, b):
            assert np.any(e < lo) or np.any(e > hi)


# ------------------------------------------------------------ closed forms ---

def _box_geom(theta, nx=40, ny=24, nz=7, sp=(0.5, 1.25, 2.0), n_cols=9, n_rows=3, pitch=0.77):
    src, dc, du, dv = W.parallel_trajectory(1, start=theta, pitch_u=pitch, pitch_v=0.61)
    return W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, n_rows, n_cols, src, dc, du, dv, nx, ny, nz,
                      W.centred_origin(nx, ny, nz, sp), sp)


@pytest.mark.parametrize("theta", [0.0, 0.3, 0.7853981633974483, 1.1, math.pi / 2, 2.0, 2.9])
def test_uniform_box_central_chord(theta):
    """x = 1 on a W x H x D box: the in-plane ray through the box centre has
    line integral min(W/|cos t|, H/|sin t|) (rectangle chord through its centre)."""
    g = _box_geom(theta)
    Wd, Hd = g.nx * g.spacing[0], g.ny * g.spacing[1]
    y = oracle.forward(g, np.ones(g.vol_shape, np.float32))
    c = math.cos(theta)
    s = math.sin(theta)
    expect = min(Wd / abs(c) if abs(c) > 1e-15 else math.inf, Hd / abs(s) if abs(s) > 1e-15 else math.inf)
    assert y[0, 1, 4] == pytest.approx(expect, rel=1e-12)


def test_uniform_box_offset_chords_against_rectangle_geometry():
    """Off-centre in-plane rays through a W x H rectangle: the chord at
    perpendicular offset q is the length of {t : |q n + t d| inside}, here
    computed from the rectangle's four edge lines in closed form."""
    theta = 0.41
    g = _box_geom(theta)
    Wd, Hd = g.nx * g.spacing[0], g.ny * g.spacing[1]
    y = oracle.forward(g, np.ones(g.vol_shape, np.float32))
    d = np.array([math.cos(theta), math.sin(theta)])
    n = np.array([-math.sin(theta), math.cos(theta)])
    for c in range(g.n_cols):
        q = (c - (g.n_cols - 1) / 2) * 0.77
        p = q * n
        # |p_x + t d_x| <= W/2 and |p_y + t d_y| <= H/2
        ts = sorted([(-Wd / 2 - p[0]) / d[0], (Wd / 2 - p[0]) / d[0]])
        us = sorted([(-Hd / 2 - p[1]) / d[1], (Hd / 2 - p[1]) / d[1]])
        expect = max(0.0, min(ts[1], us[1]) - max(ts[0], us[0]))
        assert y[0, 1, c] == pytest.approx(expect, rel=1e-12, abs=1e-12)


def test_cone_axis_aligned_chord_through_box():
    """A cone ray along +x from a source outside the box, at fixed (y, z)
    inside it, crosses the full box width nx*dx; a pixel far outside the
    box's shadow gives 0."""
    nx, ny, nz = 12, 10, 9
    sp = (0.9, 1.1, 1.3)
    o = W.centred_origin(nx, ny, nz, sp)
    src = np.array([[-30.0, 0.21, -0.37]])
    dc = np.array([[25.0, 0.21, -0.37]])
    du = np.array([[0.0, 40.0, 0.0]])     # columns at y = 0.21 + (c-1)*40
    dv = np.array([[0.0, 0.0, 1.0]])
    g = W.Geometry(W.BEAM_CONE, W.DET_FLAT, 1, 3, src, dc, du, dv, nx, ny, nz, o, sp)
    y = oracle.forward(g, np.ones(g.vol_shape, np.float32))
    assert y[0, 0, 1] == pytest.approx(nx * sp[0], rel=1e-12)
    # y = 40.21 at x = 25: at the box face x = 5.4 the ray is at y > 26 > 5.5
    assert y[0, 0, 2] == 0.0 and y[0, 0, 0] == 0.0


def test_cone_segment_ends_at_an_endpoint_inside_the_box():
    """A cone ray is the segment from the source to the pixel, not a line: an
    axis-aligned ray whose source lies inside the box integrates from the
    source to the far face; one whose pixel lies inside integrates from the
    near face to the pixel (box widths, closed form)."""
    nx, ny, nz = 10, 8, 6
    sp = (1.0, 1.0, 1.0)
    o = W.centred_origin(nx, ny, nz, sp)   # box [-5, 5) x [-4, 4) x [-3, 3)
    # view 0: source inside at x = 1.3, pixel far outside along +x
    # view 1: source far outside at x = -40, pixel inside at x = 2.2
    src = np.array([[1.3, -0.7, 0.4], [-40.0, 0.3, 0.2]])
    dc = np.array([[40.0, -0.7, 0.4], [2.2, 0.3, 0.2]])
    du = np.array([[0.0, 30.0, 0.0], [0.0, 30.0, 0.0]])   # the side columns miss the box
    dv = np.array([[0.0, 0.0, 1.0], [0.0, 0.0, 1.0]])
    g = W.Geometry(W.BEAM_CONE, W.DET_FLAT, 1, 3, src, dc, du, dv, nx, ny, nz, o, sp)
    y = oracle.forward(g, np.ones(g.vol_shape, np.float32))
    assert y[0, 0, 1] == pytest.approx(5.0 - 1.3, rel=1e-12)
    assert y[1, 0, 1] == pytest.approx(2.2 + 5.0, rel=1e-12)


def test_textbook_reduction_axis_aligned_views():
    """Parallel views along +x and +y through voxel centres reduce to a numpy
    sum along that axis times the pitch (exact in FP64 up to summation order)."""
    nx, ny, nz = 9, 6, 5
    sp = (0.7, 1.3, 0.9)
    rng = np.random.default_rng(3)
    vol = rng.random((nz, ny, nx)).astype(np.float32)
    o = W.centred_origin(nx, ny, nz, sp)
    # view 0: along +x; columns step +y by dy; rows step +z by dz
    src = np.array([[1.0, 0, 0], [0, 1.0, 0]])
    dc = np.zeros((2, 3))
    du = np.array([[0, sp[1], 0], [-sp[0], 0, 0]])
    dv = np.array([[0, 0, sp[2]], [0, 0, sp[2]]])
    g0 = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, nz, ny, src[:1], dc[:1], du[:1], dv[:1], nx, ny, nz, o, sp)
    y0 = oracle.forward(g0, vol)[0]
    np.testing.assert_allclose(y0, vol.astype(np.float64).sum(axis=2) * sp[0], rtol=1e-13)
    # view 1: along +y; column c sits at x = -(c - (nx-1)/2) dx, i.e. reversed x
    g1 = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, nz, nx, src[1:], dc[1:], du[1:], dv[1:], nx, ny, nz, o, sp)
    y1 = oracle.forward(g1, vol)[0]
    np.testing.assert_allclose(y1, vol.astype(np.float64).sum(axis=1)[:, ::-1] * sp[1], rtol=1e-13)


def test_config0_axis_views_are_numpy_sums():
    """Workload 0 holds views at 0 and 90 degrees whose rays pass through voxel
    centres: those sinogram views are plain sums of the phantom."""
    wl = W.workload(0)
    g = wl.geom
    vol = wl.phantom()
    y = oracle.forward(g.subset_views([0, 32]), vol)
    np.testing.assert_allclose(y[0], vol.astype(np.float64).sum(axis=2), rtol=1e-12)
    np.testing.assert_allclose(y[1], vol.astype(np.float64).sum(axis=1)[:, ::-1], rtol=1e-12)


def test_single_voxel_chord_matches_brute_force():
    """x = e_j: forward gives the chord of every ray through voxel j; checked
    against midpoint-rule integration along the ray."""
    for name, g in small_geometries().items():
        rng = np.random.default_rng(11)
        for _ in range(3):
            vol = np.zeros(g.vol_shape, np.float32)
            k, j, i = (rng.integers(2, n - 2) for n in g.vol_shape)
            vol[k, j, i] = 1.0
            y = oracle.forward(g, vol)
            hits = np.argwhere(y > 0)
            assert hits.shape[0] > 0, name
            for v, r, c in hits[:: max(1, hits.shape[0] // 6)]:
                a, b = oracle.ray_endpoints(g, int(v), int(r), int(c))
                bf, bound = brute_force_line_integral(vol, g.origin, g.spacing, a, b, 400_000)
                assert abs(y[v, r, c] - bf) <= bound + 1e-12, (name, v, r, c, y[v, r, c], bf, bound)


@pytest.mark.parametrize("name", ["parallel", "cone_flat", "helical_cyl"])
def test_random_volume_matches_brute_force(name):
    """Random volume, every geometry kind: forward equals brute-force
    integration along the same ray within the integrator's bound."""
    g = small_geometries()[name]
    rng = np.random.default_rng(5)
    vol = rng.random(g.vol_shape).astype(np.float32)
    y = oracle.forward(g, vol)
    for _ in range(12):
        v, r, c = rng.integers(g.n_views), rng.integers(g.n_rows), rng.integers(g.n_cols)
        a, b = oracle.ray_endpoints(g, v, r, c)
        bf, bound = brute_force_line_integral(vol, g.origin, g.spacing, a, b, 400_000)
        assert abs(y[v, r, c] - bf) <= bound + 1e-12, (v, r, c, y[v, r, c], bf, bound)


def test_update_count_axis_aligned():
    """An axis-aligned parallel view has exactly nx segments per hitting ray."""
    nx, ny, nz = 9, 6, 5
    sp = (0.7, 1.3, 0.9)
    o = W.centred_origin(nx, ny, nz, sp)
    g = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, nz, ny, np.array([[1.0, 0, 0]]), np.zeros((1, 3)),
                   np.array([[0, sp[1], 0]]), np.array([[0, 0, sp[2]]]), nx, ny, nz, o, sp)
    assert oracle.count_updates(g) == nz * ny * nx


# --------------------------------------------------- analytic ellipsoids ---

def _ellipsoid_scene(n):
    """Fixed physical box [-16, 16]^3 sampled on an n^3 grid; two ellipsoids;
    a cone and a parallel view set with irrational detector offsets."""
    sp = (32.0 / n,) * 3
    rng = np.random.default_rng(21)
    ells = []
    for _ in range(2):
        ells.append(W.Ellipsoid(centre=rng.uniform(-3, 3, 3), semi_axes=rng.uniform(5, 9, 3),
                                rotation=W._random_rotation(rng), density=float(rng.uniform(0.5, 2))))
    vol = W.rasterise_ellipsoids(np.zeros((n, n, n), np.float32), ells, W.centred_origin(n, n, n, sp), sp)
    gp = W.make_parallel(n, n, n, 3, 13, 13, pitch_u=2.03, pitch_v=2.07, spacing=sp, start=0.37)
    gp.det_c = gp.det_c + np.array([0.1234, 0.0567, 0.0891])
    gc = W.make_cone(n, n, n, 3, 13, 13, sid=60.0, sdd=100.0, pitch_u=3.1, pitch_v=3.3, spacing=sp, start=0.21)
    gc.det_c = gc.det_c + np.array([0.0311, 0.0729, 0.1113])
    return vol, ells, [gp, gc]


def _analytic(g, ells):
    out = np.zeros(g.sino_shape)
    for v in range(g.n_views):
        for r in range(g.n_rows):
            for c in range(g.n_cols):
                a, b = oracle.ray_endpoints(g, v, r, c)
                out[v, r, c] = sum(e.density * ellipsoid_chord(e, a, b) for e in ells)
    return out


def test_ellipsoid_line_integrals_converge_first_order():
    """The voxelised ellipsoid's Siddon projection converges to the analytic
    line integral (density x chord) with observed order >= 0.8 under grid
    refinement 32 -> 64 -> 128 at fixed physical geometry."""
    errs = {0: [], 1: []}
    for n in (32, 64, 128):
        vol, ells, geoms = _ellipsoid_scene(n)
        for gi, g in enumerate(geoms):
            y = oracle.forward(g, vol)
            ya = _analytic(g, ells)
            mask = ya > 0
            errs[gi].append(np.linalg.norm((y - ya)[mask]) / np.linalg.norm(ya[mask]))
    for gi, e in errs.items():
        order = math.log2(e[0] / e[2]) / 2
        assert order >= 0.8, (gi, e)
        # first-order model e ~ C h: the finest grid within 1.5x of e32 / 4
        assert e[2] <= 1.5 * e[0] / 4, (gi, e)


def test_ellipsoid_bound_per_ray():
    """|Siddon - analytic| <= density * sqrt(3) h * (boundary voxels crossed):
    only voxels cut by the surface can be wrongly in or out."""
    vol, ells, geoms = _ellipsoid_scene(32)
    h = 1.0
    for g in geoms:
        y = oracle.forward(g, vol)
        ya = _analytic(g, ells)
        for v in range(g.n_views):
            for r in range(0, g.n_rows, 3):
                for c in range(0, g.n_cols, 3):
                    idx, w = oracle.ray_segments(g, v, r, c)
                    # voxels on the ray whose value differs from a neighbour's along the ray
                    vals = vol.reshape(-1)[idx]
                    nb = int(np.count_nonzero(np.diff(vals))) + 2
                    dens = sum(e.density for e in ells)
                    assert abs(y[v, r, c] - ya[v, r, c]) <= dens * math.sqrt(3) * h * nb + 1e-9


# ------------------------------------------------------ transpose pins ---

def test_dense_transpose_8cubed_every_geometry_kind():
    """Brute-force system matrix on an 8^3 volume: columns A e_j from forward,
    rows A^T e_i from back; back must be the exact transpose of forward."""
    geoms = {
        "parallel": W.make_parallel(8, 8, 8, 3, 5, 7, pitch_u=1.3, pitch_v=1.1, start=0.2),
        "cone_flat": W.make_cone(8, 8, 8, 3, 5, 7, sid=20.0, sdd=35.0, pitch_u=2.1, pitch_v=1.9, start=0.4),
        "helical_cyl": W.make_cone(8, 8, 8, 3, 5, 7, sid=20.0, sdd=35.0,
                                   pitch_u=W.helical_fan_pitch(7, 5.5, 20.0, 35.0), pitch_v=1.7,
                                   detector=W.DET_CYLINDRICAL, z_start=-2.0, z_end=2.0, start=0.1),
    }
    for name, g in geoms.items():
        n_vox, n_rays = g.n_vox, g.n_rays
        A = np.zeros((n_rays, n_vox))
        for j in range(n_vox):
            e = np.zeros(n_vox, np.float32)
            e[j] = 1
            A[:, j] = oracle.forward(g, e.reshape(g.vol_shape)).reshape(-1)
        B = np.zeros((n_vox, n_rays))
        for i in range(n_rays):
            e = np.zeros(n_rays, np.float32)
            e[i] = 1
            B[:, i] = oracle.back(g, e.reshape(g.sino_shape)).reshape(-1)
        assert np.count_nonzero(A) > n_rays, name
        np.testing.assert_allclose(B, A.T, rtol=0, atol=1e-13)
        np.testing.assert_allclose(oracle.dense_matrix(g), A, rtol=0, atol=1e-13)


@pytest.mark.parametrize("name", ["parallel", "cone_flat", "helical_cyl"])
def test_adjoint_identity(name):
    """<A x, y> = <x, A^T y> to 1e-12 relative for random x, y."""
    g = small_geometries()[name]
    rng = np.random.default_rng(9)
    x = rng.random(g.vol_shape).astype(np.float32)
    y = rng.random(g.sino_shape).astype(np.float32)
    lhs = float((oracle.forward(g, x) * y.astype(np.float64)).sum())
    rhs = float((x.astype(np.float64) * oracle.back(g, y)).sum())
    assert abs(lhs - rhs) <= 1e-12 * abs(lhs)


def test_back_coefficient_powers():
    """Power 0 counts segments per voxel, power 2 squares the coefficients."""
    g = small_geometries()["cone_flat"]
    ones = np.ones(g.sino_shape, np.float32)
    b0 = oracle.back(g, ones, power=0)
    assert b0.sum() == oracle.count_updates(g)
    A = oracle.dense_matrix(g)
    np.testing.assert_allclose(oracle.back(g, ones, power=2).reshape(-1), (A ** 2).sum(axis=0), atol=1e-12)
    np.testing.assert_allclose(oracle.back(g, ones, power=1).reshape(-1), A.sum(axis=0), atol=1e-12)


def test_view_ranges_compose():
    """Forward over view ranges concatenates; back over ranges sums."""
    g = small_geometries()["helical_cyl"]
    rng = np.random.default_rng(2)
    x = rng.random(g.vol_shape).astype(np.float32)
    y = rng.random(g.sino_shape).astype(np.float32)
    full = oracle.forward(g, x)
    np.testing.assert_array_equal(np.concatenate([oracle.forward(g, x, (0, 3)), oracle.forward(g, x, (3, 7))]), full)
    np.testing.assert_allclose(oracle.back(g, y[:3], (0, 3)) + oracle.back(g, y[3:], (3, 7)), oracle.back(g, y),
                               atol=1e-12)


# ------------------------------------------- geometry gradient reference ---

def test_fd_geometry_gradient_matches_rectangle_chord_slope():
    """Uniform W x H box, one in-plane parallel ray at offset q: the chord is
    a trapezoid in q; shifting det_c along the detector's column direction by
    e moves the ray by e, so dy/d(det_c . u_hat) is the trapezoid's slope,
    computed from the rectangle's edge lines (closed form), and shifting
    det_c along the ray direction changes nothing.  The levers of det_u and
    det_v (the pixel's column and row offsets) and the turn of the ray about
    its pixel under a tilt of the direction follow from the same closed form."""
    from oracle.geometry_grad import geometry_gradient_fd
    theta = 0.41
    pitch = 3.9   # columns 0, 1, 7, 8 fall on the ramps of the 20 x 30 rectangle's chord profile
    g = _box_geom(theta, pitch=pitch)
    vol = np.ones(g.vol_shape, np.float32)
    Wd, Hd = g.nx * g.spacing[0], g.ny * g.spacing[1]
    d = np.array([math.cos(theta), math.sin(theta)])
    n = np.array([-math.sin(theta), math.cos(theta)])

    def chord(q):
        p = q * n
        ts = sorted([(-Wd / 2 - p[0]) / d[0], (Wd / 2 - p[0]) / d[0]])
        us = sorted([(-Hd / 2 - p[1]) / d[1], (Hd / 2 - p[1]) / d[1]])
        return max(0.0, min(ts[1], us[1]) - max(ts[0], us[0]))

    def chord_line(p, u):
        """Chord of the line p + t u (u any length) through the rectangle."""
        u = u / np.hypot(u[0], u[1])
        ts = sorted([(-Wd / 2 - p[0]) / u[0], (Wd / 2 - p[0]) / u[0]])
        us = sorted([(-Hd / 2 - p[1]) / u[1], (Hd / 2 - p[1]) / u[1]])
        return max(0.0, min(ts[1], us[1]) - max(ts[0], us[0]))

    n3 = np.array([n[0], n[1], 0.0])
    for c in (0, 1, 7, 8):   # rays on the sloped part of the trapezoid
        lever = c - (g.n_cols - 1) / 2
        q = lever * pitch
        slope = (chord(q + 1e-4) - chord(q - 1e-4)) / 2e-4
        assert abs(slope) > 0.5   # a ramp, so every check below has a nonzero target
        up = np.zeros(g.sino_shape)
        up[0, 1, c] = 1.0
        grad = geometry_gradient_fd(g, vol, up)
        assert grad[0, 1] @ n3 == pytest.approx(slope, rel=1e-6, abs=1e-7)
        assert grad[0, 1] @ np.array([d[0], d[1], 0.0]) == pytest.approx(0.0, abs=1e-6)
        # det_u moves column c by (c - cc) times the step; det_v moves row 1,
        # the middle row, not at all
        assert grad[0, 2] @ n3 == pytest.approx(lever * slope, rel=1e-6, abs=1e-6)
        assert grad[0, 3] @ n3 == pytest.approx(0.0, abs=1e-6)
        # tilting the direction turns the ray about its pixel
        turn = (chord_line(q * n, d + 1e-5 * n) - chord_line(q * n, d - 1e-5 * n)) / 2e-5
        assert grad[0, 0] @ n3 == pytest.approx(turn, rel=1e-5, abs=1e-6)
        # the bottom row (r = 0) moves with det_v by -1 times the step
        up = np.zeros(g.sino_shape)
        up[0, 0, c] = 1.0
        assert geometry_gradient_fd(g, vol, up)[0, 3] @ n3 == pytest.approx(-slope, rel=1e-6, abs=1e-6)
