"""GPU parity: the CUDA projector pair against the FP64 oracle.

Every case calls the library through its C ABI (ctypes binding) on seeded
inputs.  Small and ragged geometries of every kind, and workloads 0 and 1,
are compared element by element; the full-size workloads 2-4 are compared on
sampled rays, on sparse sinograms whose back projection the oracle builds
segment by segment, and through the adjoint identity.
"""
import math

import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import (EPS32, adjoint_mismatch, check_back, check_forward, gpu_back, gpu_forward,
                               oracle_chords, projector, rel_l2)
from tests.helpers import small_geometries

pytestmark = pytest.mark.gpu


def ragged_geometries():
    """Sizes that leave partial tiles everywhere: detector tiles are 32 columns
    x 8 rows, adjoint bricks 64x64x4 (parallel) and 32x32x16 (cone)."""
    gs = dict(small_geometries())
    gs["parallel_ragged"] = W.make_parallel(70, 45, 33, 9, 37, 77, pitch_u=1.1, pitch_v=0.9,
                                            spacing=(1.0, 1.1, 0.95), start=0.05)
    g = W.make_cone(48, 40, 36, 7, 29, 51, sid=120.0, sdd=210.0, pitch_u=1.9, pitch_v=2.1,
                    spacing=(1.0, 0.9, 1.1), start=0.17)
    g.det_c = g.det_c + np.array([0.0123, -0.0211, 0.0377])
    gs["cone_ragged"] = g
    pu = W.helical_fan_pitch(61, 30.0, 70.0, 120.0)
    g = W.make_cone(56, 50, 24, 21, 13, 61, sid=70.0, sdd=120.0, pitch_u=pu, pitch_v=1.3,
                    spacing=(1.0, 1.05, 0.95), detector=W.DET_CYLINDRICAL, z_start=-9.3, z_end=8.9, start=0.11)
    gs["helical_ragged"] = g
    # parallel beam whose rays tilt out of the slice planes (3-D traversal)
    src, dc, du, dv = W.parallel_trajectory(6, start=0.2)
    src[:, 2] = 0.31
    gs["parallel_tilted"] = W.Geometry(W.BEAM_PARALLEL, W.DET_FLAT, 21, 35, src, dc, du, dv, 30, 28, 26,
                                       W.centred_origin(30, 28, 26), (1.0, 1.0, 1.0))
    return gs


def _local_len(P, geom):
    """Longest distance over which an adjoint variant measures FP32 crossing
    positions: the brick diagonal for the brick adjoint; for the ray-driven
    variants (sort, scatter), whose walks re-anchor every 64 slabs, 65 voxel
    diagonals, or the volume diagonal if that is shorter."""
    if P.info()["adjoint_variant"] == 1:
        b = np.array(P.info()["brick"], dtype=np.float64) * np.array(geom.spacing)
        return float(np.linalg.norm(b))
    vol_diag = float(np.linalg.norm(np.array([geom.nx, geom.ny, geom.nz]) * np.array(geom.spacing)))
    return min(vol_diag, 65.0 * float(np.linalg.norm(geom.spacing)))


def _seeded_volume(geom, seed):
    rng = np.random.default_rng(seed)
    return rng.random(geom.vol_shape).astype(np.float32)


@pytest.mark.parametrize("name", sorted(ragged_geometries()))
def test_forward_matches_oracle_small(name):
    g = ragged_geometries()[name]
    vol = _seeded_volume(g, 1)
    P = projector(g)
    y = gpu_forward(P, vol)
    check_forward(y, oracle.forward(g, vol), oracle_chords(g), min(g.spacing), name)


@pytest.mark.parametrize("name", sorted(ragged_geometries()))
def test_back_matches_oracle_small(name):
    g = ragged_geometries()[name]
    rng = np.random.default_rng(2)
    sino = rng.random(g.sino_shape).astype(np.float32)
    P = projector(g)
    x = gpu_back(P, sino)
    check_back(x, oracle.back(g, sino), oracle.back(g, np.abs(sino), power=0), _local_len(P, g), name)


@pytest.mark.parametrize("name", sorted(ragged_geometries()))
def test_adjoint_identity_small(name):
    g = ragged_geometries()[name]
    P = projector(g)
    assert adjoint_mismatch(P, g) <= 1e-5


@pytest.mark.parametrize("index", [0, 1])
def test_workload_full_parity(index):
    """Workloads 0 and 1 element by element, forward and back."""
    wl = W.workload(index)
    g = wl.geom
    vol = wl.phantom()
    sino = wl.sinogram()
    P = projector(g)
    y = gpu_forward(P, vol)
    check_forward(y, oracle.forward(g, vol), oracle_chords(g), min(g.spacing), wl.name)
    x = gpu_back(P, sino)
    check_back(x, oracle.back(g, sino), oracle.back(g, sino, power=0), _local_len(P, g), wl.name)
    assert adjoint_mismatch(P, g) <= 1e-5


def test_workload0_axis_views_are_plain_sums():
    """Views at 0 and 90 degrees of workload 0 pass through voxel centres: the
    GPU result equals the numpy sum along the axis to FP32 rounding."""
    wl = W.workload(0)
    vol = wl.phantom()
    P = projector(wl.geom)
    y = gpu_forward(P, vol)
    np.testing.assert_allclose(y[0], vol.astype(np.float64).sum(axis=2), rtol=2e-6)
    np.testing.assert_allclose(y[32], vol.astype(np.float64).sum(axis=1)[:, ::-1], rtol=2e-6)


@pytest.mark.parametrize("name", ["parallel_ragged", "cone_ragged", "helical_ragged"])
def test_update_count(name):
    g = ragged_geometries()[name]
    P = projector(g)
    n_gpu = P.count_updates()
    n_ref = oracle.count_updates(g)
    assert abs(n_gpu - n_ref) <= 1e-3 * n_ref, (n_gpu, n_ref)


def _sample_rays(geom, n, rng):
    return (rng.integers(0, geom.n_views, n), rng.integers(0, geom.n_rows, n), rng.integers(0, geom.n_cols, n))


@pytest.mark.slow
@pytest.mark.parametrize("index", [2, 3, 4])
def test_workload_full_size_sampled(index):
    """Full-size workloads: the whole GPU sinogram, checked on 1500 sampled
    rays against the oracle, with the per-ray criterion."""
    import torch
    wl = W.workload(index)
    g = wl.geom
    vol = wl.phantom()
    P = projector(g)
    y = P.forward(torch.from_numpy(vol).cuda())
    rng = np.random.default_rng(100 + index)
    vs, rs, cs = _sample_rays(g, 1500, rng)
    got = y[torch.from_numpy(vs).cuda(), torch.from_numpy(rs).cuda(), torch.from_numpy(cs).cuda()].cpu().numpy()
    ref = oracle.forward_rays(g, vol, vs, rs, cs)
    chord = oracle.forward_rays(g, np.ones(g.vol_shape, np.float32), vs, rs, cs)
    ymax = float(y.abs().max().item())
    err = np.abs(got - ref)
    crossing = (chord >= min(g.spacing)) & (np.abs(ref) >= 1e-3 * ymax)
    assert crossing.sum() > 100
    assert float((err[crossing] / np.abs(ref[crossing])).max()) <= 1e-4
    assert np.all(err <= 1e-4 * np.abs(ref) + 1e-6 * ymax)
    assert rel_l2(got, ref) <= 1e-5


@pytest.mark.slow
@pytest.mark.parametrize("index", [2, 3, 4])
def test_workload_full_size_sparse_back(index):
    """Full-size adjoint on a sinogram with 24 non-zero rays: the result is the
    weighted sum of those rays' oracle coefficient lists, voxel by voxel, and
    zero elsewhere."""
    import torch
    wl = W.workload(index)
    g = wl.geom
    P = projector(g)
    rng = np.random.default_rng(200 + index)
    sino = torch.zeros(g.sino_shape, dtype=torch.float32, device="cuda")
    expect = {}
    count = {}
    k = 0
    while k < 24:
        v, r, c = int(rng.integers(g.n_views)), int(rng.integers(g.n_rows)), int(rng.integers(g.n_cols))
        idx, w = oracle.ray_segments(g, v, r, c)
        if idx.size < 10 or sino[v, r, c].item() != 0:
            continue
        val = float(np.float32(rng.uniform(0.5, 2.0)))
        sino[v, r, c] = val
        for i, wi in zip(idx.tolist(), w.tolist()):
            expect[i] = expect.get(i, 0.0) + wi * val
            count[i] = count.get(i, 0.0) + val
        k += 1
    x = P.back(sino).reshape(-1)
    keys = np.array(sorted(expect))
    ref = np.array([expect[i] for i in keys])
    cnt = np.array([count[i] for i in keys])
    got = x[torch.from_numpy(keys).cuda()].double().cpu().numpy()
    tau = 8 * EPS32 * _local_len(P, g)
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + tau * cnt)
    # nothing outside the rays' support beyond FP32 crumbs
    mask = torch.ones(g.n_vox, dtype=torch.bool, device="cuda")
    mask[torch.from_numpy(keys).cuda()] = False
    outside = x[mask].abs().max().item()
    assert outside <= tau * 2.0
    assert rel_l2(got, ref) <= 1e-5


@pytest.mark.slow
@pytest.mark.parametrize("index", [2, 3, 4])
def test_workload_full_size_adjoint_identity(index):
    wl = W.workload(index)
    P = projector(wl.geom)
    assert adjoint_mismatch(P, wl.geom) <= 1e-5


def _ladder():
    rows = []
    path = __file__.replace("test_parity_gpu.py", "golden/fp32_clipping_error_ladder.txt")
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            sid, err = line.split()
            rows.append((float(sid), float(err)))
    return rows


@pytest.mark.parametrize("sid,fp32_err", _ladder())
def test_fp64_setup_beats_fp32_clipping_ladder(sid, fp32_err):
    """64^3 cone scan, 16 views, at growing source distance, the detector as
    far past the centre as the source is before it (the reading under which
    an FP32 set-up reproduces the pages' ladder, see
    test_build_variants_gpu.py).  With FP32 clipping the pages measure
    maximum errors 3e-5 / 9e-3 / 4e-2 of the sinogram's scale; the FP64 set-up
    here must stay within 1e-4 per ray at every distance, and ten times below
    the pages' figure at 1e5 and 1e6."""
    from tests.run_setup_ladder import ladder_geometry, max_error_over_max, worst_relative_error
    wl = W.workload(1)
    g = ladder_geometry(sid, "twice")
    vol = wl.phantom()
    P = projector(g)
    y = gpu_forward(P, vol).astype(np.float64)
    ref = oracle.forward(g, vol)
    assert worst_relative_error(y, ref) <= 1e-4
    if sid >= 1e5:
        assert max_error_over_max(y, ref) < fp32_err / 10


def test_rays_missing_the_volume_are_zero_and_back_is_zero():
    g = W.make_parallel(16, 16, 16, 3, 4, 6)
    g.det_c = g.det_c + np.array([0.0, 0.0, 100.0])  # detector rows far above the volume
    P = projector(g)
    y = gpu_forward(P, np.ones(g.vol_shape, np.float32))
    assert np.all(y == 0)
    x = gpu_back(P, np.ones(g.sino_shape, np.float32))
    assert np.all(x == 0)


def test_degenerate_sizes():
    """Single voxel / single pixel / single view cases against the oracle."""
    cases = [
        W.make_parallel(1, 1, 1, 1, 1, 1, start=0.3),
        W.make_parallel(1, 3, 1, 2, 1, 5, pitch_u=0.5, start=0.4),
        W.make_cone(2, 1, 3, 3, 2, 1, sid=10.0, sdd=15.0, pitch_u=0.4, pitch_v=0.6, start=0.2),
    ]
    rng = np.random.default_rng(4)
    for g in cases:
        vol = rng.random(g.vol_shape).astype(np.float32) + 0.5
        P = projector(g)
        y = gpu_forward(P, vol)
        ref = oracle.forward(g, vol)
        np.testing.assert_allclose(y, ref, rtol=1e-5, atol=1e-6)
        sino = rng.random(g.sino_shape).astype(np.float32)
        np.testing.assert_allclose(gpu_back(P, sino), oracle.back(g, sino), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("plan", [{"forward_layout": 1}, {"forward_layout": 2}, {"brick": (8, 8, 8)},
                                  {"brick": (16, 8, 4), "view_groups": 3}, {"view_groups": 1}])
def test_plan_overrides_keep_results(plan):
    """Layout, brick and view-group choices change scheduling, not values."""
    g = ragged_geometries()["cone_ragged"]
    vol = _seeded_volume(g, 5)
    rng = np.random.default_rng(6)
    sino = rng.random(g.sino_shape).astype(np.float32)
    P = projector(g, plan)
    check_forward(gpu_forward(P, vol), oracle.forward(g, vol), oracle_chords(g), min(g.spacing), str(plan))
    check_back(gpu_back(P, sino), oracle.back(g, sino), oracle.back(g, sino, power=0), _local_len(P, g), str(plan))


def test_host_pointer_is_rejected():
    import torch
    from ray_forward_back_b200 import ctp
    g = small_geometries()["parallel"]
    P = projector(g)
    host = torch.zeros(g.vol_shape, dtype=torch.float32)
    dev = torch.zeros(g.sino_shape, dtype=torch.float32, device="cuda")
    with pytest.raises(ctp.CtpError) as ei:
        ctp.ctp_forward(P.handle, host.data_ptr(), dev.data_ptr())
    assert ei.value.status == ctp.CTP_ERR_INVALID_ARGUMENT


# ------------------------------------------ sort / segment-reduce adjoint ---

@pytest.mark.parametrize("variant", [1, 2, 3])
@pytest.mark.parametrize("name", sorted(ragged_geometries()))
def test_back_variant_matches_oracle_small(name, variant):
    """Every adjoint variant (brick, sort / segment-reduce, ray scatter) meets
    the same tolerances, forced through the plan."""
    g = ragged_geometries()[name]
    rng = np.random.default_rng(12)
    sino = rng.random(g.sino_shape).astype(np.float32)
    P = projector(g, {"adjoint_variant": variant})
    assert P.info()["adjoint_variant"] == variant
    x = gpu_back(P, sino)
    check_back(x, oracle.back(g, sino), oracle.back(g, np.abs(sino), power=0), _local_len(P, g), name)
    assert adjoint_mismatch(P, g) <= 1e-5


@pytest.mark.parametrize("variant", [1, 2, 3])
@pytest.mark.parametrize("index", [0, 1])
def test_back_variant_workloads(index, variant):
    wl = W.workload(index)
    g = wl.geom
    sino = wl.sinogram()
    P = projector(g, {"adjoint_variant": variant})
    x = gpu_back(P, sino)
    check_back(x, oracle.back(g, sino), oracle.back(g, sino, power=0), _local_len(P, g), wl.name)


def high_magnification_cone():
    """Cone beam whose rays are a hundred times denser than the voxels at the
    centre: a warp's 32 rays fall into a handful of voxels."""
    return W.make_cone(16, 16, 16, 6, 64, 128, sid=15.0, sdd=1500.0, pitch_u=1.0, pitch_v=1.0, start=0.15)


def test_collision_ratio_measured_and_dispatch_consistent():
    """The ratio measured at create is >= 1 and grows with ray density; the
    automatic choice is the sort adjoint for dense rays (ratio >= 13.5) and
    the scatter adjoint otherwise (on geometries without decoupled slices,
    where the gather adjoint does not apply), and both results meet the
    tolerances."""
    dense = high_magnification_cone()
    sparse = ragged_geometries()["cone_ragged"]
    Pd, Ps = projector(dense), projector(sparse)
    rd, rs = Pd.info()["collision_ratio"], Ps.info()["collision_ratio"]
    assert rs >= 1.0 and rd >= 1.0
    assert rd > 2.0 * rs, (rd, rs)
    assert Pd.info()["adjoint_variant"] == (2 if rd >= 13.5 else 3)
    assert Ps.info()["adjoint_variant"] == (2 if rs >= 13.5 else 3)
    assert Pd.info()["adjoint_variant"] == 2 and Ps.info()["adjoint_variant"] == 3, (rd, rs)
    for P, g in ((Pd, dense), (Ps, sparse)):
        rng = np.random.default_rng(3)
        sino = rng.random(g.sino_shape).astype(np.float32)
        ref = oracle.back(g, sino)
        check_back(gpu_back(P, sino), ref, oracle.back(g, sino, power=0), _local_len(P, g), "auto")


def _stored_counts():
    rows = {}
    path = __file__.replace("test_parity_gpu.py", "golden/update_counts.txt")
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            i, n = line.split()
            rows[int(i)] = int(n)
    return rows


@pytest.mark.parametrize("index", [0, 1, 2, 3])
def test_device_update_count_matches_oracle_fixture(index):
    """The device's count of positive-length segments for each full workload
    equals the oracle's exact count (stored by tests/golden/make_update_counts.py)
    up to segments whose length rounds across zero (ties at voxel corners)."""
    ref = _stored_counts()[index]
    P = projector(W.workload(index).geom)
    got = P.count_updates()
    assert abs(got - ref) <= 1e-4 * ref, (got, ref)


# ------------------------------------------------ coefficient powers (NEXT) ---

@pytest.mark.parametrize("variant", [1, 2, 3])
@pytest.mark.parametrize("name", ["parallel_ragged", "cone_ragged", "helical_ragged", "parallel_tilted"])
def test_back_squared_coefficients(name, variant):
    """Back projection with squared weights (the normal operator's diagonal)
    against the oracle's power-2 back projection.  A segment error d in len
    becomes 2 len d in len^2, so the per-segment term of the tolerance is
    scaled by 2 x the voxel diagonal."""
    g = ragged_geometries()[name]
    rng = np.random.default_rng(21)
    sino = rng.random(g.sino_shape).astype(np.float32)
    P = projector(g, {"adjoint_variant": variant})
    import torch
    x = P.back_power(torch.from_numpy(sino).cuda(), 2)
    torch.cuda.synchronize()
    diag = float(np.linalg.norm(g.spacing))
    local = _local_len(P, g)
    check_back(x.cpu().numpy(), oracle.back(g, sino, power=2), oracle.back(g, np.abs(sino), power=0),
               2.0 * diag * local, f"{name} power 2")


@pytest.mark.parametrize("variant", [1, 3])
def test_back_power_one_is_back(variant):
    """Power 1 is the plain adjoint: bit for bit with the brick adjoint (exact
    integer sums), to FP32 accumulation order with the scatter adjoint."""
    import torch
    g = ragged_geometries()["cone_ragged"]
    P = projector(g, {"adjoint_variant": variant})
    sino = torch.rand(g.sino_shape, device="cuda")
    a = P.back(sino)
    b = P.back_power(sino, 1)
    torch.cuda.synchronize()
    if variant == 1:
        assert torch.equal(a, b)
    else:
        torch.testing.assert_close(a, b, rtol=1e-5, atol=1e-6 * float(a.abs().max()))


def test_sirt_normalisers_are_projections_of_ones():
    """Row sums A 1 (ray lengths through the volume) and column sums A^T 1
    (total ray length per voxel) against the oracle."""
    import torch
    g = ragged_geometries()["helical_ragged"]
    P = projector(g)
    rows = P.forward(torch.ones(g.vol_shape, device="cuda"))
    cols = P.back(torch.ones(g.sino_shape, device="cuda"))
    torch.cuda.synchronize()
    ones_v = np.ones(g.vol_shape, np.float32)
    ones_s = np.ones(g.sino_shape, np.float32)
    check_forward(rows.cpu().numpy(), oracle.forward(g, ones_v), oracle_chords(g), min(g.spacing), "A 1")
    check_back(cols.cpu().numpy(), oracle.back(g, ones_s), oracle.back(g, ones_s, power=0), _local_len(P, g), "A^T 1")


def test_back_power_rejects_other_powers():
    import torch
    from ray_forward_back_b200 import ctp
    g = small_geometries()["parallel"]
    P = projector(g)
    with pytest.raises(ctp.CtpError) as ei:
        P.back_power(torch.zeros(g.sino_shape, device="cuda"), 3)
    assert ei.value.status == ctp.CTP_ERR_INVALID_ARGUMENT
