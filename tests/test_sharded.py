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


# ------------------------------------------------------------ slice sharding --

def _slice_geometries():
    from ray_forward_back_b200 import workloads as W
    gs = {}
    # one row per slice, rows and slices aligned
    gs["aligned"] = W.make_parallel(9, 8, 7, 5, 7, 11, pitch_u=0.9, pitch_v=1.0, start=0.21)
    # several rows per slice, rows beyond the volume on both sides
    gs["dense_rows"] = W.make_parallel(9, 8, 5, 4, 13, 10, pitch_u=1.1, pitch_v=0.55, start=0.37,
                                       spacing=(1.0, 1.0, 1.3))
    # coarse rows: some slices hold no row; rows step downwards
    g = W.make_parallel(8, 9, 9, 3, 4, 9, pitch_u=1.0, pitch_v=2.1, start=0.11)
    g.det_v = -g.det_v
    gs["coarse_descending"] = g
    return gs


@pytest.mark.parametrize("name", sorted(_slice_geometries()))
def test_slice_partition_covers_the_rows_inside_the_volume_once(name):
    from ray_forward_back_b200.sharded import slice_partition
    g = _slice_geometries()[name]
    rc = 0.5 * (g.n_rows - 1)
    z = g.det_c[0, 2] + (np.arange(g.n_rows) - rc) * g.det_v[0, 2]
    inside = (z >= g.origin[2]) & (z < g.origin[2] + g.nz * g.spacing[2])
    for world in (1, 2, 3, g.nz + 2):
        owned = np.zeros(g.n_rows, dtype=int)
        for r in range(world):
            z0, z1, r0, r1 = slice_partition(g, r, world)
            owned[r0:r1] += 1
            sl = np.floor((z[r0:r1] - g.origin[2]) / g.spacing[2])
            assert np.all((sl >= z0) & (sl < z1))
        np.testing.assert_array_equal(owned, inside.astype(int))


@pytest.mark.parametrize("name", sorted(_slice_geometries()))
def test_slice_sharded_projection_equals_unsharded(name):
    """Ranks emulated in one process (they exchange nothing): the rows and
    slabs they produce reassemble the unsharded oracle projections."""
    import torch
    import oracle
    from ray_forward_back_b200.sharded import SliceShardedProjector
    g = _slice_geometries()[name]
    rng = np.random.default_rng(1)
    vol = rng.random(g.vol_shape).astype(np.float32)
    sino = rng.random(g.sino_shape).astype(np.float32)
    y_ref = oracle.forward(g, vol)
    x_ref = oracle.back(g, sino)
    for world in (2, 3):
        y = np.zeros(g.sino_shape)
        x = np.zeros(g.vol_shape)
        for rank in range(world):
            S = SliceShardedProjector(g, make_projector=_OracleProjector, rank=rank, world=world)
            y[:, S.r0:S.r1] = S.forward(torch.from_numpy(vol[S.z0:S.z1].copy())).numpy()
            x[S.z0:S.z1] = S.back(torch.from_numpy(sino[:, S.r0:S.r1].copy())).numpy()
        np.testing.assert_allclose(y, y_ref.astype(np.float32), rtol=1e-6, atol=1e-6 * np.abs(y_ref).max())
        np.testing.assert_allclose(x, x_ref.astype(np.float32), rtol=1e-6, atol=1e-6 * np.abs(x_ref).max())


def test_slice_sharding_rejects_coupled_slices():
    from ray_forward_back_b200 import workloads as W
    from ray_forward_back_b200.sharded import slice_partition
    cone = W.make_cone(8, 8, 8, 3, 4, 5, sid=30.0, sdd=50.0)
    with pytest.raises(ValueError):
        slice_partition(cone, 0, 2)
    tilted = W.make_parallel(8, 8, 8, 3, 4, 5)
    src = tilted.src.copy()
    src[:, 2] = 0.1
    tilted.src = src
    with pytest.raises(ValueError):
        slice_partition(tilted, 0, 2)
    helix_like = W.make_parallel(8, 8, 8, 3, 4, 5)
    dc = helix_like.det_c.copy()
    dc[1, 2] += 0.25
    helix_like.det_c = dc
    with pytest.raises(ValueError):
        slice_partition(helix_like, 0, 2)


def _slice_rank_main(rank, world, port, out):
    import torch.distributed as dist
    from ray_forward_back_b200.sharded import SliceShardedProjector
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = _slice_geometries()["aligned"]
        S = SliceShardedProjector(g, make_projector=_OracleProjector)
        out[rank] = (S.rank, S.world, S.z0, S.z1, S.r0, S.r1)
    finally:
        dist.destroy_process_group()


def test_slice_sharding_takes_rank_and_world_from_the_group():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_slice_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    assert out[0] == (0, 2, 0, 4, 0, 4) and out[1] == (1, 2, 4, 7, 4, 7)
