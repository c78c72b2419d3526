"""The gather adjoint (CTP_ADJOINT_GATHER) against the FP64 oracle.

Parallel beams whose rays lie in z-planes with detector rows stepping along
z: the adjoint is computed voxel by voxel from closed-form chords and the
sinogram's slice sums (forced through the plan on these small geometries,
where the automatic choice is the scatter).  Checked: the adjoint
tolerances (relative L2, per voxel), squared coefficients, the adjoint
identity, bitwise reproducibility,
non-finite propagation, batches, slice counts that take every lane layout
(1, 2 and 4 float4 groups per lane, several slice chunks), the automatic
choice and the geometries it refuses."""
import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import ctp
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import adjoint_mismatch, back_errors, gpu_back, projector
from tests.test_slice_rows_gpu import slice_geometries

pytestmark = pytest.mark.gpu

GATHER = 4


def gather_geometries():
    gs = dict(slice_geometries())
    # rows stepping downwards: slices are summed from the last row up
    gs["rows_downwards"] = W.make_parallel(12, 10, 9, 4, 11, 15, pitch_v=-0.8, start=0.3)
    # views on the axes (0 and 90 degrees; the latter's direction has a 6e-17
    # x component), rays half a voxel from the grid lines
    gs["axis_views"] = W.make_parallel(16, 16, 8, 8, 8, 16)
    # slice counts for 2 float4 groups per lane, and 4 with two slice chunks
    gs["slices_200"] = W.make_parallel(10, 9, 200, 3, 210, 13, pitch_u=1.1, start=0.4)
    gs["slices_600"] = W.make_parallel(7, 6, 600, 2, 600, 9, pitch_u=0.9, start=0.7)
    return gs


def _tolerances(be, label):
    assert be["rel_l2"] <= 1e-5, (label, be)
    assert be["worst_rel"] <= 1e-4, (label, be)
    assert be["worst_abs_other_over_max"] <= 1e-6, (label, be)


@pytest.mark.parametrize("name", sorted(gather_geometries()))
def test_gather_matches_oracle(name):
    g = gather_geometries()[name]
    P = projector(g, {"adjoint_variant": GATHER})
    assert P.info()["adjoint_variant"] == GATHER
    rng = np.random.default_rng(21)
    sino = rng.random(g.sino_shape).astype(np.float32)
    be = back_errors(gpu_back(P, sino), oracle.back(g, sino))
    print(name, be)
    _tolerances(be, name)
    import torch
    x2 = P.back_power(torch.from_numpy(sino).cuda(), 2).cpu().numpy()
    _tolerances(back_errors(x2, oracle.back(g, sino, power=2)), name + " power 2")
    assert adjoint_mismatch(P, g) <= 1e-5


def test_gather_workload0_meets_the_oracle_and_the_automatic_choice():
    """Workload 0 through the gather; the automatic choice takes the gather
    once its grid holds four blocks per SM and the volume has more than 128
    slices (workload 4), the scatter otherwise (workload 0: 256 blocks, 64
    slices)."""
    wl = W.workload(0)
    P = projector(wl.geom, {"adjoint_variant": GATHER})
    sino = wl.sinogram()
    _tolerances(back_errors(gpu_back(P, sino), oracle.back(wl.geom, sino)), wl.name)
    assert projector(wl.geom).info()["adjoint_variant"] == 3
    assert projector(W.workload(4).geom).info()["adjoint_variant"] == GATHER


def test_gather_is_bitwise_reproducible_and_batches_member_by_member():
    import torch
    g = gather_geometries()["parallel_ragged"]
    P = projector(g, {"adjoint_variant": GATHER})
    torch.manual_seed(8)
    sino = torch.rand((3,) + tuple(g.sino_shape), device="cuda")
    single = [P.back(sino[b].contiguous()) for b in range(3)]
    batch = P.back(sino)
    for b in range(3):
        assert torch.equal(batch[b], single[b])
        assert torch.equal(P.back(sino[b].contiguous()), single[b])


def test_gather_propagates_a_non_finite_ray_to_the_voxels_it_crosses():
    import torch
    g = gather_geometries()["parallel_ragged"]
    P = projector(g, {"adjoint_variant": GATHER})
    v, r, c = 4, 17, 40
    sino = np.random.default_rng(2).random(g.sino_shape).astype(np.float32)
    sino[v, r, c] = np.nan
    x = P.back(torch.from_numpy(sino).cuda()).cpu().numpy()
    one = np.zeros(g.sino_shape, np.float32)
    one[v, r, c] = 1.0
    path = oracle.back(g, one)
    nan = np.isnan(x)
    assert nan.any()
    assert np.all(path[nan] > 0.0)
    assert np.all(nan[path > 1e-6 * path.max()])
    assert np.all(np.isfinite(x[path == 0.0]))


def _grid_line_axis_view():
    # 13 columns of pitch 0.9 on an 11-voxel-wide volume: at 90 degrees (x
    # direction 6e-17) column 1's ray lies on the grid line x = 0 of voxel units
    return W.make_parallel(11, 9, 7, 6, 5, 13, pitch_u=0.9, pitch_v=1.1, start=0.0)


def test_gather_refusals_fall_back_automatically():
    tilted_src, dc, du, dv = W.parallel_trajectory(6, start=0.2)
    tilted_src[:, 2] = 0.31
    tilted = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, 21, 35, tilted_src, dc, du, dv, 30, 28, 26,
                        W.centred_origin(30, 28, 26), (1.0, 1.0, 1.0))
    cone = W.make_cone(16, 16, 16, 4, 12, 20, sid=60.0, sdd=110.0, start=0.1)
    for label, g in (("grid line", _grid_line_axis_view()), ("tilted", tilted), ("cone", cone)):
        P = projector(g)
        assert P.info()["adjoint_variant"] in (2, 3), label
        with pytest.raises(ctp.CtpError) as err:
            projector(g, {"adjoint_variant": GATHER})
        assert err.value.status == ctp.CTP_ERR_UNSUPPORTED, label
        assert "gather adjoint" in err.value.detail, label


def test_gather_forced_other_variants_still_available():
    g = gather_geometries()["parallel_ragged"]
    rng = np.random.default_rng(5)
    sino = rng.random(g.sino_shape).astype(np.float32)
    ref = oracle.back(g, sino)
    out = {}
    for variant in (1, 2, 3, GATHER):
        P = projector(g, {"adjoint_variant": variant})
        assert P.info()["adjoint_variant"] == variant
        out[variant] = gpu_back(P, sino)
        _tolerances(back_errors(out[variant], ref), f"variant {variant}")
