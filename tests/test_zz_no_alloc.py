"""ctp_forward_noalloc: the forward projection for callers that cannot
allocate device memory.

Some callers cannot call cudaMalloc at all -- a real-time loop with a fixed
memory budget, an allocator-free runtime, or a process whose device memory
is owned by another framework -- so they cannot create a geometry handle
either.  For them the library offers one entry point that takes the
acquisition description directly and keeps everything it needs in a fixed
device array built into the library.  These tests call it through the C ABI
and compare it with the ordinary handle-based ctp_forward.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest

from ray_forward_back_b200 import ctp
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import projector, rel_l2
from tests.helpers import small_geometries

pytestmark = pytest.mark.gpu


def _close(got, ref):
    """The parity tests' forward tolerance: relative L2 <= 1e-5 and every
    ray within 1e-4 relative plus 1e-6 of the largest value."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert rel_l2(got, ref) <= 1e-5
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-6 * np.abs(ref).max())


def _noalloc_forward(geom, vol_t):
    import torch
    out = torch.full(geom.sino_shape, float("nan"), dtype=torch.float32, device=vol_t.device)
    ctp.ctp_forward_noalloc(geom, vol_t, out, device=vol_t.device.index or 0)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_noalloc_matches_ctp_forward_on_two_calls_in_a_row():
    import torch
    torch.cuda.init()
    dev = torch.device("cuda", torch.cuda.current_device())
    # first call: a flat cone geometry whose volume copy is needed;
    # second call: a different (cylindrical, helical) geometry and volume,
    # which must overwrite every part of the shared scratch correctly
    cases = [W.workload(1).geom, small_geometries()["helical_cyl"]]
    rng = np.random.default_rng(77)
    for g in cases:
        vol = torch.from_numpy(rng.random(g.vol_shape).astype(np.float32)).to(dev)
        P = projector(g)
        ref = P.forward(vol)
        torch.cuda.synchronize()
        got = _noalloc_forward(g, vol)
        _close(got, ref.cpu().numpy())
        P.close()


def test_noalloc_rejects_a_description_beyond_its_scratch():
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    # views near 0 degrees need the y-fastest copy: 256 x 256 x 160 voxels x 4 B = 40 MiB > 32 MiB
    g = W.make_parallel(256, 256, 160, 4, 8, 8, start=0.1)
    vol = torch.zeros(g.vol_shape, dtype=torch.float32, device=dev)
    sino = torch.zeros(g.sino_shape, dtype=torch.float32, device=dev)
    with pytest.raises(ctp.CtpError) as ei:
        ctp.ctp_forward_noalloc(g, vol, sino, device=dev.index or 0)
    assert ei.value.status == ctp.CTP_ERR_OUT_OF_RANGE
    assert "scratch" in ei.value.detail
