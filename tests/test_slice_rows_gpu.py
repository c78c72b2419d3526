"""Shared (x, y) walks for parallel slices (plan.slice_rows).

When every ray lies in a z-plane and detector rows step along z only, the
forward projection and the scatter adjoint walk one (x, y) path per detector
column for 2 or 4 rows at a time.  Each row sees exactly the segments of its
own walk, so the forward must be bit-identical to one walk per ray, and the
adjoint must meet the oracle's tolerances; geometries whose slices couple
keep one walk per ray.
"""
import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import adjoint_mismatch, check_back, gpu_back, gpu_forward, projector
from tests.helpers import small_geometries

pytestmark = pytest.mark.gpu


def slice_geometries():
    gs = {"parallel": small_geometries()["parallel"]}
    # rows finer and coarser than the slices, some rows above and below the volume
    g = W.make_parallel(70, 45, 33, 9, 37, 77, pitch_u=1.1, pitch_v=0.9, spacing=(1.0, 1.1, 0.95), start=0.05)
    gs["parallel_ragged"] = g
    g = W.make_parallel(40, 36, 12, 7, 23, 45, pitch_u=1.0, pitch_v=0.7, spacing=(1.0, 1.0, 1.3), start=0.3)
    g.det_c = g.det_c + np.array([0.0, 0.0, 2.1])  # rows run past the top of the volume
    gs["parallel_rows_outside"] = g
    # det_u with a z component: the slice of a row changes along the row
    src, dc, du, dv = W.parallel_trajectory(5, start=0.4)
    du[:, 2] = 0.05
    gs["parallel_slanted_rows"] = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, 19, 41, src, dc, du, dv, 36, 30, 16,
                                             W.centred_origin(36, 30, 16), (1.0, 1.0, 1.0))
    gs["workload0"] = W.workload(0).geom
    return gs


@pytest.mark.parametrize("rows", [2, 4])
@pytest.mark.parametrize("name", sorted(slice_geometries()))
def test_slice_rows_forward_is_bit_identical(name, rows):
    g = slice_geometries()[name]
    vol = np.random.default_rng(31).random(g.vol_shape).astype(np.float32)
    P1 = projector(g, {"slice_rows": 1})
    Pr = projector(g, {"slice_rows": rows})
    assert P1.info()["slice_rows"] == 1 and Pr.info()["slice_rows"] == rows
    np.testing.assert_array_equal(gpu_forward(Pr, vol), gpu_forward(P1, vol))


@pytest.mark.parametrize("power", [1, 2])
@pytest.mark.parametrize("rows", [2, 4])
@pytest.mark.parametrize("name", sorted(slice_geometries()))
def test_slice_rows_scatter_adjoint_matches_oracle(name, rows, power):
    import torch
    g = slice_geometries()[name]
    sino = np.random.default_rng(32).random(g.sino_shape).astype(np.float32)
    P = projector(g, {"slice_rows": rows, "adjoint_variant": 3})
    assert P.info()["slice_rows"] == rows
    x = P.back_power(torch.from_numpy(sino).cuda(), power)
    torch.cuda.synchronize()
    diag = float(np.linalg.norm(g.spacing))
    local = min(float(np.linalg.norm(np.array([g.nx, g.ny, g.nz]) * np.array(g.spacing))), 65.0 * diag)
    check_back(x.cpu().numpy(), oracle.back(g, sino, power=power), oracle.back(g, sino, power=0),
               local * (2.0 * diag if power == 2 else 1.0), f"{name} rows {rows} power {power}")
    if power == 1:
        assert adjoint_mismatch(P, g) <= 1e-5


def test_slice_rows_keep_zero_and_non_finite_rows():
    """A zero row adds nothing; a NaN reaches the voxels its ray crosses."""
    g = slice_geometries()["parallel_ragged"]
    sino = np.random.default_rng(33).random(g.sino_shape).astype(np.float32)
    sino[:, 5] = 0.0
    sino[2, 11, 40] = np.nan
    P = projector(g, {"slice_rows": 4, "adjoint_variant": 3})
    x = gpu_back(P, sino)
    assert np.isnan(x).any()
    finite = sino.copy()
    finite[2, 11, 40] = 0.0
    ref = oracle.back(g, finite)
    mask = ~np.isnan(x)
    np.testing.assert_allclose(x[mask], ref[mask], rtol=1e-4, atol=1e-5 * np.abs(ref).max())


@pytest.mark.parametrize("name", ["parallel_tilted", "cone"])
def test_coupled_slices_keep_one_walk_per_ray(name):
    if name == "cone":
        g = small_geometries()["cone_flat"]
    else:
        src, dc, du, dv = W.parallel_trajectory(6, start=0.2)
        src[:, 2] = 0.31
        g = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, 21, 35, src, dc, du, dv, 30, 28, 26,
                       W.centred_origin(30, 28, 26), (1.0, 1.0, 1.0))
    P = projector(g, {"slice_rows": 4})
    assert P.info()["slice_rows"] == 1
