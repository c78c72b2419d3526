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


@pytest.mark.parametrize("name", ["cone_flat", "parallel_both_layouts"])
def test_batched_back_equals_single_calls(name):
    import torch
    g = _geoms()[name]
    P = projector(g)
    torch.manual_seed(5)
    sino = torch.rand((2, 2) + tuple(g.sino_shape), device="cuda")
    x = P.back(sino)
    assert x.shape == (2, 2) + tuple(g.vol_shape)
    for a in range(2):
        for b in range(2):
            assert torch.equal(x[a, b], P.back(sino[a, b].contiguous()))


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
