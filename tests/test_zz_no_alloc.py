"""ctp_forward_noalloc: the forward projection for callers that cannot
allocate device memory.

Some callers cannot call cudaMalloc at all -- a real-time loop with a fixed
memory budget, an allocator-free runtime, or a process whose device memory
is owned by another framework -- so they cannot create a geometry handle
either.  For them the library offers one entry point that takes the
acquisition description directly and keeps everything it needs in a fixed
device array built into the library.  These tests call it through the C ABI
and compare it with the ordinary handle-based ctp_forward and with the FP64
oracle.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest

import oracle
from ray_forward_back_b200 import ctp
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import check_forward, oracle_chords, projector, rel_l2
from tests.helpers import small_geometries

pytestmark = pytest.mark.gpu


def _close(got, ref):
    """The parity tests' forward tolerance: relative L2 <= 1e-5 and every
    ray within 1e-4 relative plus 1e-6 of the largest value."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert rel_l2(got, ref) <= 1e-5
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-6 * np.abs(ref).max())


def _noalloc_forward(geom, vol_t, stream=None):
    import torch
    out = torch.full(geom.sino_shape, float("nan"), dtype=torch.float32, device=vol_t.device)
    ctp.ctp_forward_noalloc(geom, vol_t, out, device=vol_t.device.index or 0, stream=stream)
    return out


def _wide_cylindrical(n_cols):
    """A cylindrical detector wider than one staged column row."""
    pu = W.helical_fan_pitch(n_cols, 8.0, 60.0, 100.0)
    return W.make_cone(16, 14, 12, 2, 2, n_cols, sid=60.0, sdd=100.0, pitch_u=pu, pitch_v=1.1,
                       detector=W.DET_CYLINDRICAL, z_start=-1.3, z_end=1.1, start=0.21)


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
        vol_np = rng.random(g.vol_shape).astype(np.float32)
        vol = torch.from_numpy(vol_np).to(dev)
        P = projector(g)
        ref = P.forward(vol)
        got = _noalloc_forward(g, vol)
        torch.cuda.synchronize()
        _close(got.cpu().numpy(), ref.cpu().numpy())
        # the same records, layouts and walks: bit for bit
        assert torch.equal(got, ref)
        check_forward(got.cpu().numpy(), oracle.forward(g, vol_np), oracle_chords(g), min(g.spacing), "noalloc")
        P.close()


def test_noalloc_two_geometries_queued_on_one_stream():
    """Two calls enqueued back to back on one stream, one synchronisation:
    the second call's uploads are ordered after the first call's kernels, so
    both results stand."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    g1, g2 = small_geometries()["cone_flat"], small_geometries()["helical_cyl"]
    rng = np.random.default_rng(78)
    v1 = rng.random(g1.vol_shape).astype(np.float32)
    v2 = rng.random(g2.vol_shape).astype(np.float32)
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        t1, t2 = torch.from_numpy(v1).to(dev), torch.from_numpy(v2).to(dev)
        y1 = _noalloc_forward(g1, t1, stream=s)
        y2 = _noalloc_forward(g2, t2, stream=s)
    s.synchronize()
    check_forward(y1.cpu().numpy(), oracle.forward(g1, v1), oracle_chords(g1), min(g1.spacing), "first")
    check_forward(y2.cpu().numpy(), oracle.forward(g2, v2), oracle_chords(g2), min(g2.spacing), "second")


def test_noalloc_equals_the_shared_slice_forward():
    """A parallel beam whose slices decouple: ctp_forward shares one walk
    between 4 rows on interleaved copies, the no-allocation forward walks
    every ray on its own; the sinograms are the same bit for bit."""
    import torch
    g = W.make_parallel(48, 40, 24, 30, 32, 61, pitch_u=1.0, pitch_v=1.0, start=0.05)
    P = projector(g, {"slice_rows": 4})
    assert P.info()["interleaved_slices"] == 1
    vol = torch.from_numpy(np.random.default_rng(80).random(g.vol_shape).astype(np.float32)).cuda()
    ref = P.forward(vol)
    got = _noalloc_forward(g, vol)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("n_cols", [1500, 33000])
def test_noalloc_wide_cylindrical_detector(n_cols):
    """Column rows packed several views to a copy (1500 columns) and a row
    wider than the staging array, sent in pieces (33000 columns)."""
    import torch
    g = _wide_cylindrical(n_cols)
    vol = np.random.default_rng(79).random(g.vol_shape).astype(np.float32)
    got = _noalloc_forward(g, torch.from_numpy(vol).cuda())
    torch.cuda.synchronize()
    check_forward(got.cpu().numpy(), oracle.forward(g, vol), oracle_chords(g), min(g.spacing), f"{n_cols} cols")


def test_noalloc_refuses_a_capturing_stream():
    """Its uploads read host memory of the call itself, so a stream being
    captured into a graph is refused before anything is enqueued."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    g = small_geometries()["cone_flat"]
    vol = torch.rand(g.vol_shape, device=dev)
    out = torch.zeros(g.sino_shape, dtype=torch.float32, device=dev)
    s = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=s):
        out.fill_(1.0)
        with pytest.raises(ctp.CtpError) as ei:
            ctp.ctp_forward_noalloc(g, vol, out, device=dev.index or 0, stream=s)
    assert ei.value.status == ctp.CTP_ERR_UNSUPPORTED
    graph.replay()
    torch.cuda.synchronize()
    assert bool((out == 1.0).all())
    # outside the capture the same call works
    got = _noalloc_forward(g, vol)
    torch.cuda.synchronize()
    assert torch.isfinite(got).all()


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
