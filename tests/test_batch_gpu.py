"""Leading batch dimensions (ctp_forward_batch / ctp_back_batch): every
member's projection must equal the single-volume call on that member, bit for
bit (the fused forward walks each ray once for a chunk of members and adds
each member's segments in the same order), and each member must meet the
oracle's tolerances.  Empty batches do nothing."""
import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import ctp
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import check_forward, oracle_chords, projector
from tests.helpers import small_geometries

pytestmark = pytest.mark.gpu


def _geoms():
    gs = small_geometries()
    # views over the whole half turn: both forward layouts (x- and y-fastest) occur
    gs["parallel_both_layouts"] = W.make_parallel(21, 19, 6, 9, 5, 37, pitch_u=0.8, pitch_v=1.1, start=0.05)
    return gs


@pytest.mark.parametrize("chunk", [1, 2, 4])
@pytest.mark.parametrize("name", sorted(_geoms()))
def test_batched_forward_equals_single_calls(name, chunk):
    import torch
    g = _geoms()[name]
    P = projector(g, plan={"batch_chunk": chunk})
    info = P.info()
    assert info["batch_chunk"] == chunk
    torch.manual_seed(3)
    for n in (1, 3, 5, 7):
        vol = torch.rand((n,) + tuple(g.vol_shape), device="cuda")
        y = P.forward(vol)
        assert y.shape == (n,) + tuple(g.sino_shape)
        for b in range(n):
            assert torch.equal(y[b], P.forward(vol[b].contiguous())), (name, chunk, n, b)


def test_batched_members_meet_the_oracle():
    import torch
    g = _geoms()["parallel_both_layouts"]
    P = projector(g, plan={"batch_chunk": 4})
    assert P.info()["n_transposed_views"] not in (0, g.n_views)
    rng = np.random.default_rng(4)
    vols = rng.random((5,) + tuple(g.vol_shape)).astype(np.float32)
    y = P.forward(torch.from_numpy(vols).cuda()).cpu().numpy()
    chord = oracle_chords(g)
    for b in range(5):
        check_forward(y[b], oracle.forward(g, vols[b]), chord, min(g.spacing), f"member {b}")


@pytest.mark.parametrize("name,variant", [("cone_flat", 1), ("cone_flat", 3), ("parallel_both_layouts", 1),
                                          ("parallel_both_layouts", 3), ("parallel_both_layouts", 4)])
def test_batched_back_equals_single_calls(name, variant):
    """Member by member, the batched adjoint is the single call: bit for bit
    with the brick adjoint (integer sums, fixed order) and the gather adjoint
    (each voxel summed by one thread in a fixed order), to FP32 accumulation
    order with the scatter adjoint (float adds in whatever order the atomics
    land)."""
    import torch
    g = _geoms()[name]
    P = projector(g, plan={"adjoint_variant": variant})
    torch.manual_seed(5)
    sino = torch.rand((2, 2) + tuple(g.sino_shape), device="cuda")
    x = P.back(sino)
    assert x.shape == (2, 2) + tuple(g.vol_shape)
    for a in range(2):
        for b in range(2):
            single = P.back(sino[a, b].contiguous())
            if variant in (1, 4):
                assert torch.equal(x[a, b], single)
            else:
                torch.testing.assert_close(x[a, b], single, rtol=1e-5, atol=1e-6 * float(single.abs().max()))


def test_leading_dimensions_empty_and_errors():
    import torch
    g = _geoms()["cone_flat"]
    P = projector(g, plan={"batch_chunk": 2})
    vol = torch.rand((2, 3) + tuple(g.vol_shape), device="cuda")
    y = P.forward(vol)
    assert y.shape == (2, 3) + tuple(g.sino_shape)
    assert torch.equal(y[1, 2], P.forward(vol[1, 2].contiguous()))
    empty = torch.empty((0, 4) + tuple(g.vol_shape), device="cuda")
    assert P.forward(empty).shape == (0, 4) + tuple(g.sino_shape)
    assert P.back(torch.empty((3, 0) + tuple(g.sino_shape), device="cuda")).shape == (3, 0) + tuple(g.vol_shape)
    with pytest.raises(ctp.CtpError) as ei:
        ctp.ctp_forward_batch(P.handle, vol, y, -1)
    assert ei.value.status == ctp.CTP_ERR_INVALID_ARGUMENT
    with pytest.raises(ValueError):
        P.forward(vol[:, :, 1:])


def test_scratch_grows_with_the_chunk_only_when_views_are_transposed():
    g = _geoms()["parallel_both_layouts"]
    one = projector(g, plan={"batch_chunk": 1}).info()
    four = projector(g, plan={"batch_chunk": 4}).info()
    assert one["n_transposed_views"] > 0
    assert four["scratch_bytes"] - one["scratch_bytes"] == 3 * 4 * g.n_vox
    x_only = projector(g, plan={"batch_chunk": 4, "forward_layout": 1}).info()
    assert x_only["n_transposed_views"] == 0
    assert x_only["scratch_bytes"] < one["scratch_bytes"]


@pytest.mark.parametrize("name", ["parallel_both_layouts", "cone_flat", "helical_cyl"])
@pytest.mark.parametrize("chunk,n", [(2, 2), (2, 3), (4, 5)])
def test_fused_batched_back_meets_the_oracle(name, chunk, n):
    """plan.batch_chunk >= 2: member pairs share each ray's walk in one
    launch (a brick half as deep in y, two fixed-point accumulators).  Each
    member meets the oracle's tolerances and agrees with its single call to
    FP32 accumulation (the two use different bricks, hence different
    fixed-point scales); an odd last member runs alone."""
    import torch
    from tests.gpu_helpers import check_back
    g = _geoms()[name]
    P = projector(g, plan={"batch_chunk": chunk, "adjoint_variant": 1})
    rng = np.random.default_rng(7)
    sino = rng.random((n,) + tuple(g.sino_shape)).astype(np.float32)
    x = P.back(torch.from_numpy(sino).cuda()).cpu().numpy()
    local_len = float(np.linalg.norm(np.array(P.info()["brick"]) * np.array(g.spacing)))
    for b in range(n):
        ref = oracle.back(g, sino[b])
        check_back(x[b], ref, oracle.back(g, sino[b], power=0), local_len, f"{name} member {b}")
        single = P.back(torch.from_numpy(sino[b]).cuda()).cpu().numpy()
        np.testing.assert_allclose(x[b], single, rtol=1e-5, atol=1e-6 * np.abs(single).max())


def test_fused_batched_back_keeps_members_apart():
    """A non-finite value in one member reaches only that member's voxels; an
    all-zero member gives exactly zero."""
    import torch
    g = _geoms()["parallel_both_layouts"]
    P = projector(g, plan={"batch_chunk": 2, "adjoint_variant": 1})
    rng = np.random.default_rng(8)
    sino = rng.random((2,) + tuple(g.sino_shape)).astype(np.float32)
    sino[0, 3, 2, 10] = np.nan
    x = P.back(torch.from_numpy(sino).cuda()).cpu().numpy()
    assert np.isnan(x[0]).any()
    single = P.back(torch.from_numpy(sino[1]).cuda()).cpu().numpy()
    assert np.isfinite(x[1]).all()
    np.testing.assert_allclose(x[1], single, rtol=1e-5, atol=1e-6 * np.abs(single).max())
    sino[0] = 0.0
    x = P.back(torch.from_numpy(sino).cuda()).cpu().numpy()
    assert np.count_nonzero(x[0]) == 0 and np.isfinite(x[1]).all()
