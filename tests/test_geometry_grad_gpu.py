"""Geometry gradients on the GPU (ctp_geometry_gradient) against central
finite differences of the FP64 oracle's forward projection.

The line integral is piecewise linear in the geometry, so away from kinks
the finite difference is exact up to rounding; the seeded geometries are
perturbed off the voxel lattice so that no ray sits within the step of a
kink.  The GPU walks in FP32 (crossing distances to a few ulp of the ray
length) and sums in FP64, so the bound is relative to the largest entry."""
import numpy as np
import pytest

from oracle.geometry_grad import geometry_gradient_fd
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import projector

pytestmark = pytest.mark.gpu

REL = 2e-4
ELEMENT_FLOOR = 1e-6


def _jitter(g, seed, scale=0.03):
    """Move every vector off the lattice by a small seeded amount."""
    rng = np.random.default_rng(seed)
    for name in ("src", "det_c", "det_u", "det_v"):
        a = getattr(g, name).copy()
        ref = np.abs(a).max()
        setattr(g, name, a + scale * max(ref, 1.0) * 0.01 * rng.standard_normal(a.shape))
    return g


def _gpu_grad(g, vol, gs):
    import torch
    P = projector(g)
    out = P.geometry_gradient(torch.from_numpy(vol).cuda(), torch.from_numpy(gs).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check(g, seed, vol=None, h=1e-6, rel=REL):
    rng = np.random.default_rng(seed)
    if vol is None:
        vol = rng.random(g.vol_shape).astype(np.float32)
    gs = rng.standard_normal(g.sino_shape).astype(np.float32)
    ref = geometry_gradient_fd(g, vol, gs.astype(np.float64), h=h)
    got = _gpu_grad(g, vol, gs)
    assert got.shape == (g.n_views, 4, 3)
    scale = np.abs(ref).max()
    assert scale > 0
    err = np.abs(got - ref)
    assert err.max() <= rel * scale, (err.max(), scale)
    # entry by entry: relative to the entry, plus a floor relative to the
    # largest entry of the view set (the FP32 crossing positions carry a few
    # ulp of the ray length whatever the entry's own size)
    floor = ELEMENT_FLOOR * scale
    worst = float(((err - 1e-4 * np.abs(ref)) / scale).max())
    print(f"element floor used: {worst:.2e} of the largest entry")
    assert np.all(err <= 1e-4 * np.abs(ref) + floor), worst
    return ref, got


def _helical_cylindrical():
    """Helical source, cylindrical detector centred on the source's axis and
    raised above the source plane; det_u stays orthogonal to det_v and to
    det_c - src, as the projector requires, so only the source path and the
    start angle are off the lattice."""
    pu = W.helical_fan_pitch(9, 4.0, 20.0, 33.0)
    g = W.make_cone(9, 8, 7, 3, 5, 9, sid=20.0, sdd=33.0, pitch_u=pu, pitch_v=0.9, detector=W.DET_CYLINDRICAL,
                    z_start=-1.3, z_end=1.1, start=0.37)
    g.det_c = g.det_c + np.array([0.0, 0.0, 0.31])
    return g


CASES = {
    # cone, source and detector outside the volume; ragged detector tiles
    "cone_outside": lambda: _jitter(W.make_cone(10, 9, 7, 4, 6, 37, sid=30.0, sdd=55.0, pitch_u=1.3,
                                                pitch_v=1.4, start=0.2), 1),
    # detector plane through the volume: pixels inside, the t = 1 endpoint term
    "cone_pixels_inside": lambda: _jitter(W.make_cone(10, 9, 7, 3, 9, 11, sid=20.0, sdd=21.5, pitch_u=1.1,
                                                      pitch_v=0.9, start=0.4), 2),
    # source inside the volume: the source is the parameter origin
    "cone_source_inside": lambda: _jitter(W.make_cone(10, 9, 7, 3, 7, 9, sid=2.5, sdd=30.0, pitch_u=2.1,
                                                      pitch_v=1.7, start=0.7), 3),
    # helical source path, anisotropic voxels and a shifted volume
    "helical_flat": lambda: _jitter(W.make_cone(8, 10, 6, 5, 5, 9, sid=25.0, sdd=45.0, pitch_u=1.6, pitch_v=1.5,
                                                spacing=(1.1, 0.9, 1.3), z_start=-3.0, z_end=2.0, start=0.1,
                                                origin=(-4.7, -4.1, -3.3)), 4),
    "parallel": lambda: _jitter(W.make_parallel(9, 8, 7, 5, 6, 35, pitch_u=0.8, pitch_v=0.9, start=0.13), 5),
    "helical_cylindrical": _helical_cylindrical,
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_geometry_gradient_matches_finite_differences(name):
    g = CASES[name]()
    if name == "parallel":
        src = g.src.copy()
        src[:, 2] += 0.3     # rays oblique to the z planes
        src *= 1.7           # a direction that is not unit length
        g.src = src
    ref, got = _check(g, 10)
    if name == "parallel":
        # the length of the direction does not matter: no gradient along it
        for v in range(g.n_views):
            assert abs(got[v, 0] @ g.src[v]) <= 1e-5 * np.abs(got[v, 0]).max() * np.linalg.norm(g.src[v])


def test_geometry_gradient_on_workload1_phantom():
    """Cone 64^3 phantom of the 16-view workload, two views off the lattice,
    128x128 detector: a piecewise-constant object with many edges."""
    wl = W.workload(1)
    g = _jitter(wl.geom.subset_views([3, 11]), 6)
    _check(g, 11, vol=wl.phantom())


def test_geometry_gradient_on_workload3_cylindrical_view():
    """One view of the helical cylindrical workload (its phantom), the
    central 184 of its 736 columns (the same rays: the sub-detector keeps
    det_c on the middle of the arc).  On the whole view some of the 47k rays
    pass within the step of a voxel edge, a kink of the line integral
    (central differences with steps 1e-6 and 1e-7 differ by 3e-4 of the
    largest entry); on these 11.8k rays steps 1e-6, 1e-7 and 3e-8 agree to
    2e-6, so the standard bound applies."""
    import dataclasses
    wl = W.workload(3)
    g = dataclasses.replace(wl.geom.subset_views([401]), n_cols=184)
    _check(g, 12, vol=wl.phantom())


def test_geometry_gradient_on_workload4_volume():
    """The bench's volume: the 512^3 phantom of the parallel workload, one
    view, a 16 x 24 window of its detector (rows 300-315, columns 500-523)
    made its own detector, so rays cross up to 724 voxels.  Finite
    differences with steps 1e-6, 1e-7 and 3e-8 agree to 1e-8 of the largest
    entry here."""
    import dataclasses
    wl = W.workload(4)
    g = wl.geom.subset_views([301])
    shift = (300 - 0.5 * (g.n_rows - 1) + 7.5) * g.det_v[0] + (500 - 0.5 * (g.n_cols - 1) + 11.5) * g.det_u[0]
    g = dataclasses.replace(g, n_rows=16, n_cols=24, det_c=g.det_c + shift)
    _check(g, 13, vol=wl.phantom())


def test_zero_inputs_give_zero():
    import torch
    g = CASES["cone_outside"]()
    P = projector(g)
    vol = torch.rand(g.vol_shape, device="cuda")
    gs = torch.zeros(g.sino_shape, device="cuda")
    out = torch.full((g.n_views, 4, 3), 7.0, dtype=torch.float64, device="cuda")
    P.geometry_gradient(vol, gs, out=out)
    assert torch.count_nonzero(out).item() == 0
    P.geometry_gradient(torch.zeros_like(vol), torch.randn_like(gs), out=out)
    assert torch.count_nonzero(out).item() == 0
    with pytest.raises(ValueError):
        P.geometry_gradient(vol, gs, out=torch.empty((g.n_views, 4, 3), dtype=torch.float32, device="cuda"))


def _slice_geometry(name):
    """Parallel beams whose rays lie in z-planes and whose rows step along z
    (decoupled slices), moved off the voxel lattice in x and y only, so they
    keep that property; rows sit at half-integer heights."""
    import dataclasses
    if name == "workload0":
        g = W.workload(0).geom
    elif name == "ragged":
        g = W.make_parallel(70, 45, 33, 9, 36, 77, pitch_u=1.1, pitch_v=1.0, spacing=(1.0, 1.1, 1.0), start=0.05)
    else:
        g = W.make_parallel(40, 36, 14, 7, 24, 45, pitch_u=1.0, pitch_v=1.0, start=0.3)
        g.det_c = g.det_c + np.array([0.0, 0.0, 3.0])  # some rows above the volume
    return dataclasses.replace(g, det_c=g.det_c + np.array([0.0131, -0.0217, 0.0]))


@pytest.mark.parametrize("name", ["ragged", "rows_outside", "workload0"])
def test_slice_rows_geometry_gradient_equals_one_walk_per_ray(name):
    """Four rows per (x, y) walk on the interleaved volume: every row's
    crossing sums are those of its own walk, so only the FP64 order of the
    per-view sums differs from one walk per ray."""
    import torch
    g = _slice_geometry(name)
    rng = np.random.default_rng(41)
    vol = torch.from_numpy(rng.random(g.vol_shape).astype(np.float32)).cuda()
    gs = torch.from_numpy(rng.standard_normal(g.sino_shape).astype(np.float32)).cuda()
    P1 = projector(g, {"slice_rows": 1})
    P4 = projector(g, {"slice_rows": 4})
    assert P4.info()["interleaved_slices"] == 1 and P1.info()["slice_rows"] == 1
    a = P1.geometry_gradient(vol, gs).cpu().numpy()
    b = P4.geometry_gradient(vol, gs).cpu().numpy()
    np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-12 * np.abs(a).max())


def test_slice_rows_geometry_gradient_matches_finite_differences():
    """The same path against central finite differences of the oracle."""
    import torch
    g = _slice_geometry("rows_outside")
    rng = np.random.default_rng(42)
    vol = rng.random(g.vol_shape).astype(np.float32)
    gs = rng.standard_normal(g.sino_shape).astype(np.float32)
    ref = geometry_gradient_fd(g, vol, gs.astype(np.float64), h=1e-6)
    P = projector(g, {"slice_rows": 4})
    assert P.info()["interleaved_slices"] == 1
    got = P.geometry_gradient(torch.from_numpy(vol).cuda(), torch.from_numpy(gs).cuda()).cpu().numpy()
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    assert err.max() <= REL * scale, (err.max(), scale)
    assert np.all(err <= 1e-4 * np.abs(ref) + ELEMENT_FLOOR * scale)
