"""The view-sharded projector on the GPU path: the CUDA library per rank and
NCCL for the reductions.  Only one GPU is available to a test, so the group
has one rank; the multi-rank logic is covered by the gloo tests."""
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_single_rank_nccl_sharded_equals_projector():
    import datetime

    import torch
    import torch.distributed as dist

    from ray_forward_back_b200 import workloads as W
    from ray_forward_back_b200.sharded import ShardedProjector
    from tests.gpu_helpers import projector
    g = W.make_cone(40, 36, 24, 9, 20, 30, sid=80.0, sdd=140.0, pitch_u=1.5, pitch_v=1.5, start=0.3)
    dev = torch.device("cuda", torch.cuda.current_device())
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60), device_id=dev)
    try:
        S = ShardedProjector(g, device=dev.index)
        P = projector(g)
        vol = torch.rand(g.vol_shape, device=dev)
        sino = torch.rand(g.sino_shape, device=dev)
        assert torch.equal(S.forward(vol), P.forward(vol))
        x_ref = P.back(sino)
        # the adjoint adds FP32 contributions in whatever order the atomics land
        tol = dict(rtol=1e-5, atol=1e-6 * float(x_ref.abs().max()))
        torch.testing.assert_close(S.back(sino), x_ref, **tol)
        z0, z1, slab = S.back_slab(sino)
        assert (z0, z1) == (0, g.nz)
        torch.testing.assert_close(slab, x_ref, **tol)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_slice_sharded_gpu_projection_equals_the_whole(world):
    """Slice sharding (no collective): ranks emulated one after another on
    this GPU.  The forward rows are bit-identical to the whole-volume
    forward (the rays' x-y walks are the same); the adjoint slabs agree to
    FP32 accumulation order."""
    import torch
    from ray_forward_back_b200 import workloads as W
    from ray_forward_back_b200.sharded import SliceShardedProjector
    from tests.gpu_helpers import projector
    g = W.make_parallel(70, 45, 33, 24, 33, 77, pitch_u=0.9, pitch_v=1.0, start=0.13)
    torch.manual_seed(2)
    vol = torch.rand(g.vol_shape, device="cuda")
    sino = torch.rand(g.sino_shape, device="cuda")
    P = projector(g)
    y_all, x_all = P.forward(vol), P.back(sino)
    y = torch.zeros_like(y_all)
    x = torch.zeros_like(x_all)
    for rank in range(world):
        S = SliceShardedProjector(g, rank=rank, world=world, make_projector=projector)
        y[:, S.r0:S.r1] = S.forward(vol[S.z0:S.z1].contiguous())
        x[S.z0:S.z1] = S.back(sino[:, S.r0:S.r1].contiguous())
    assert torch.equal(y, y_all)
    assert torch.allclose(x, x_all, rtol=1e-6, atol=1e-6 * x_all.abs().max().item())


def _two_rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    from ray_forward_back_b200 import workloads as W
    from ray_forward_back_b200.sharded import ShardedProjector
    from tests.gpu_helpers import projector
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["NCCL_NVLS_ENABLE"] = "0"
    torch.cuda.set_device(rank)
    dev = torch.device("cuda", rank)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60),
                            device_id=dev)
    try:
        g = W.make_cone(40, 36, 24, 9, 20, 30, sid=80.0, sdd=140.0, pitch_u=1.5, pitch_v=1.5, start=0.3)
        rng = np.random.default_rng(0)
        vol = rng.random(g.vol_shape).astype(np.float32)
        sino = rng.random(g.sino_shape).astype(np.float32)
        S = ShardedProjector(g, device=rank, make_projector=lambda geom: projector(geom))
        y = S.forward(torch.from_numpy(vol).to(dev)).cpu().numpy()
        z0, z1, slab = S.back_slab(torch.from_numpy(sino[S.v0:S.v1]).to(dev))
        out[rank] = (S.v0, S.v1, y, z0, z1, slab.cpu().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_process_nccl_view_shards_against_the_oracle():
    """Two processes on two GPUs: each projects its view shard; the gathered
    shards are the whole forward projection and the reduce-scattered slabs
    the whole adjoint, both against the FP64 oracle.  Runs only where the
    box has two GPUs."""
    import torch
    import torch.multiprocessing as mp

    import oracle
    from ray_forward_back_b200 import workloads as W
    from tests.gpu_helpers import check_back, check_forward, oracle_chords
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_two_rank_main, args=(world, _port(), out), nprocs=world, join=True)
    g = W.make_cone(40, 36, 24, 9, 20, 30, sid=80.0, sdd=140.0, pitch_u=1.5, pitch_v=1.5, start=0.3)
    rng = np.random.default_rng(0)
    vol = rng.random(g.vol_shape).astype(np.float32)
    sino = rng.random(g.sino_shape).astype(np.float32)
    y = np.zeros(g.sino_shape, np.float32)
    x = np.zeros(g.vol_shape, np.float32)
    for rank in range(world):
        v0, v1, yr, z0, z1, slab = out[rank]
        y[v0:v1] = yr
        x[z0:z1] = slab
    check_forward(y, oracle.forward(g, vol), oracle_chords(g), min(g.spacing), "two ranks")
    local = min(float(np.linalg.norm(np.array([g.nx, g.ny, g.nz]) * np.array(g.spacing))),
                65.0 * float(np.linalg.norm(g.spacing)))
    check_back(x, oracle.back(g, sino), oracle.back(g, sino, power=0), local, "two ranks")
