"""View-sharded projector: partition rules (pure), and the sharded forward /
adjoint on 2 and 3 gloo ranks on CPU, with each rank's local projector
standing in by the FP64 oracle restricted to that rank's views.  The
sharded results must equal the unsharded oracle's; a third rank with an
empty shard takes part in the collectives normally."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from ray_forward_back_b200.sharded import view_shard, z_slab


def test_view_shards_cover_every_view_once_balanced():
    for n in (1, 2, 5, 16, 17, 900):
        for world in (1, 2, 3, 4, 8):
            shards = [view_shard(n, r, world) for r in range(world)]
            assert shards[0][0] == 0 and shards[-1][1] == n
            for (a0, a1), (b0, b1) in zip(shards, shards[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in shards]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


def test_z_slabs_pad_to_equal_shares():
    for nz in (1, 7, 64, 65):
        for world in (1, 2, 3, 8):
            slabs = [z_slab(nz, r, world) for r in range(world)]
            h = slabs[0][2]
            assert all(s[2] == h for s in slabs) and h * world >= nz > (h - 1) * world
            covered = sum(z1 - z0 for z0, z1, _ in slabs)
            assert covered == nz


class _OracleProjector:
    """CPU stand-in for one rank's projector: the oracle on its views."""

    def __init__(self, geom):
        self.geom = geom

    def forward(self, vol):
        import torch
        import oracle
        return torch.from_numpy(oracle.forward(self.geom, vol.numpy()).astype(np.float32))

    def back(self, sino):
        import torch
        import oracle
        return torch.from_numpy(oracle.back(self.geom, sino.numpy()).astype(np.float32))


def _geometry(n_views):
    from ray_forward_back_b200 import workloads as W
    return W.make_cone(10, 9, 7, n_views, 6, 8, sid=30.0, sdd=55.0, pitch_u=1.3, pitch_v=1.4, start=0.2)


def _rank_main(rank, world, port, n_views, out):
    import torch
    import torch.distributed as dist

    from ray_forward_back_b200.sharded import ShardedProjector
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = _geometry(n_views)
        rng = np.random.default_rng(0)
        vol = torch.from_numpy(rng.random(g.vol_shape).astype(np.float32))
        sino = torch.from_numpy(rng.random(g.sino_shape).astype(np.float32))
        S = ShardedProjector(g, make_projector=_OracleProjector)
        y_local = S.forward(vol)
        x_full = S.back(sino[S.v0:S.v1].contiguous(), device="cpu")
        z0, z1, slab = S.back_slab(sino[S.v0:S.v1].contiguous(), device="cpu")
        out[rank] = (S.v0, S.v1, y_local.numpy(), x_full.numpy(), z0, z1, slab.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,n_views", [(2, 5), (3, 2)])
def test_sharded_projection_equals_unsharded(world, n_views):
    import oracle
    g = _geometry(n_views)
    rng = np.random.default_rng(0)
    vol = rng.random(g.vol_shape).astype(np.float32)
    sino = rng.random(g.sino_shape).astype(np.float32)
    y_ref = oracle.forward(g, vol).astype(np.float32)
    # the sharded sum adds per-rank FP32 partial volumes: compare in FP32 terms
    x_ref = oracle.back(g, sino)
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), n_views, out), nprocs=world, join=True)
    ys = [out[r][2] for r in range(world)]
    np.testing.assert_array_equal(np.concatenate(ys, axis=0), y_ref)
    if world > n_views:
        assert any(out[r][1] == out[r][0] for r in range(world))   # an empty shard took part
    for r in range(world):
        np.testing.assert_allclose(out[r][3], x_ref, rtol=1e-6, atol=1e-6 * np.abs(x_ref).max())
    slabs = sorted((out[r][4], out[r][5], out[r][6]) for r in range(world))
    x_slabs = np.concatenate([s for _, _, s in slabs], axis=0)
    np.testing.assert_allclose(x_slabs, x_ref, rtol=1e-6, atol=1e-6 * np.abs(x_ref).max())
