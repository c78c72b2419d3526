"""View-sharded projector pair over several ranks (one process per GPU).

Each rank owns a balanced, contiguous shard of the views and projects it
with its own single-GPU projector:

  * forward: the volume is replicated on every rank; each rank computes its
    own sinogram views.  No collective (rays are independent).
  * adjoint: each rank back-projects its views into a partial volume; the
    partial volumes are summed across ranks, either into every rank's copy
    (all-reduce) or into z-slabs, one per rank (reduce-scatter, the volume
    zero-padded to equal slabs).

This follows diffct "Execution", section "Hybrid ownership and losses" (view
ranks own view shards; adjoint volume tiles sum across view ranks; empty and
uneven shards participate normally) and MBIRJAX "Sharding overview", section
"Forward and back projection by bands" (back projection is a reduction over
views followed by a scatter to slice owners; inert zero padding makes equal
shares).  The collectives are torch.distributed's (NCCL over NVLink on GPUs,
gloo on CPUs); every rank takes the same collective steps in the same order.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import numpy as np


def view_shard(n_views: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous balanced view range [v0, v1) of `rank`; the first
    n_views % world ranks get one extra view; a shard may be empty."""
    base, extra = divmod(n_views, world)
    v0 = rank * base + min(rank, extra)
    return v0, v0 + base + (1 if rank < extra else 0)


def z_slab(nz: int, rank: int, world: int) -> Tuple[int, int, int]:
    """(z0, z1, padded slab height) of `rank`'s slab of a volume with nz
    slices zero-padded to world equal slabs."""
    h = -(-nz // world)
    z0 = min(rank * h, nz)
    return z0, min(z0 + h, nz), h


class ShardedProjector:
    """Matched projector pair with the views sharded over a process group.

    ``make_projector(geometry)`` builds the local single-GPU projector (by
    default :class:`ray_forward_back_b200.ctp.Projector` on ``device``); it
    is not called on a rank whose shard is empty.
    """

    def __init__(self, geom, group=None, device: Optional[int] = None,
                 make_projector: Optional[Callable] = None):
        import torch.distributed as dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.geom = geom
        self.v0, self.v1 = view_shard(geom.n_views, self.rank, self.world)
        self.local_geom = geom.subset_views(np.arange(self.v0, self.v1)) if self.v1 > self.v0 else None
        if make_projector is None:
            from ray_forward_back_b200 import ctp
            make_projector = lambda g: ctp.Projector(g, device=device if device is not None else 0)
        self.local = make_projector(self.local_geom) if self.local_geom is not None else None

    @property
    def local_sino_shape(self):
        return (self.v1 - self.v0, self.geom.n_rows, self.geom.n_cols)

    def forward(self, vol):
        """This rank's sinogram views [v0, v1) of A vol (vol replicated)."""
        import torch
        if self.local is None:
            return torch.zeros(self.local_sino_shape, dtype=torch.float32, device=vol.device)
        return self.local.forward(vol)

    def _partial_back(self, sino_shard, device):
        import torch
        if self.local is None:
            return torch.zeros(self.geom.vol_shape, dtype=torch.float32, device=device)
        return self.local.back(sino_shard)

    def back(self, sino_shard, device=None):
        """A^T y with y sharded by views; every rank receives the whole volume."""
        import torch.distributed as dist
        part = self._partial_back(sino_shard, device if device is not None else sino_shard.device)
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        return part

    def back_slab(self, sino_shard, device=None):
        """A^T y with y sharded by views, reduce-scattered into z-slabs.
        Returns (z0, z1, slab) with slab the voxels [z0, z1) of the volume."""
        import torch
        import torch.distributed as dist
        dev = device if device is not None else sino_shard.device
        part = self._partial_back(sino_shard, dev)
        nz, ny, nx = self.geom.vol_shape
        z0, z1, h = z_slab(nz, self.rank, self.world)
        if h * self.world != nz:
            padded = torch.zeros((h * self.world, ny, nx), dtype=part.dtype, device=part.device)
            padded[:nz] = part
            part = padded
        out = torch.empty((h, ny, nx), dtype=part.dtype, device=part.device)
        dist.reduce_scatter_tensor(out, part, op=dist.ReduceOp.SUM, group=self.group)
        return z0, z1, out[: z1 - z0]


# --------------------------------------------------------------------------
# Slice sharding for parallel beams whose rays lie in z-planes.
#
# When every ray is perpendicular to z (direction and detector columns with
# no z component) and the detector rows step along z by the same amount in
# every view, detector row r sees exactly one volume slice, the one holding
# its height (MBIRJAX "Sharding overview", section "Why cone beam": a
# parallel beam decouples the slices).  Sharding z-slabs of the volume
# together with the rows that fall in them makes the ranks fully independent:
# neither projection needs a collective.


def slice_partition(geom, rank: int, world: int):
    """(z0, z1, r0, r1) of `rank`: the volume slices [z0, z1) (balanced, as
    ``z_slab``) and the detector rows [r0, r1) whose heights fall in them.
    Raises ValueError when the geometry's slices do not decouple."""
    src, dc, du, dv = (np.asarray(a, dtype=np.float64) for a in (geom.src, geom.det_c, geom.det_u, geom.det_v))
    if geom.beam != 0:
        raise ValueError("slice sharding needs a parallel beam")
    if np.any(src[:, 2] != 0.0) or np.any(du[:, 2] != 0.0) or np.any(dv[:, :2] != 0.0):
        raise ValueError("slice sharding needs rays and detector columns in z-planes and rows along z")
    if np.any(dv[:, 2] != dv[0, 2]) or np.any(dc[:, 2] != dc[0, 2]):
        raise ValueError("slice sharding needs the same row heights in every view")
    rc = 0.5 * (geom.n_rows - 1)
    z_rows = dc[0, 2] + (np.arange(geom.n_rows) - rc) * dv[0, 2]
    sl = np.floor((z_rows - geom.origin[2]) / geom.spacing[2]).astype(np.int64)
    z0, z1, _ = z_slab(geom.nz, rank, world)
    rows = np.nonzero((sl >= z0) & (sl < z1))[0]
    if rows.size == 0:
        return z0, z1, 0, 0
    return z0, z1, int(rows.min()), int(rows.max()) + 1


def slice_geometry(geom, z0: int, z1: int, r0: int, r1: int):
    """The sub-acquisition of slices [z0, z1) and detector rows [r0, r1)."""
    import dataclasses
    dv = np.asarray(geom.det_v, dtype=np.float64)
    shift = 0.5 * (r0 + r1 - 1) - 0.5 * (geom.n_rows - 1)
    origin = (geom.origin[0], geom.origin[1], geom.origin[2] + z0 * geom.spacing[2])
    return dataclasses.replace(geom, nz=z1 - z0, n_rows=r1 - r0, origin=origin,
                               det_c=np.ascontiguousarray(np.asarray(geom.det_c, dtype=np.float64) + shift * dv))


class SliceShardedProjector:
    """Projector pair with the volume sharded into z-slabs and the sinogram
    into the matching detector rows, for geometries whose slices decouple
    (see ``slice_partition``).  ``forward`` maps this rank's slab
    [z0, z1) to its rows [r0, r1) of every view; ``back`` the reverse.  Rows
    whose heights miss the volume belong to no rank (their line integrals
    are zero).  No collective is involved, so ``rank`` and ``world`` may also
    be given directly without a process group."""

    def __init__(self, geom, group=None, device: Optional[int] = None,
                 make_projector: Optional[Callable] = None, rank: Optional[int] = None,
                 world: Optional[int] = None):
        if rank is None or world is None:
            import torch.distributed as dist
            rank, world = dist.get_rank(group), dist.get_world_size(group)
        self.rank, self.world, self.geom = rank, world, geom
        self.z0, self.z1, self.r0, self.r1 = slice_partition(geom, rank, world)
        self.local_geom = None
        if self.z1 > self.z0 and self.r1 > self.r0:
            self.local_geom = slice_geometry(geom, self.z0, self.z1, self.r0, self.r1)
        if make_projector is None:
            from ray_forward_back_b200 import ctp
            make_projector = lambda g: ctp.Projector(g, device=device if device is not None else 0)
        self.local = make_projector(self.local_geom) if self.local_geom is not None else None

    @property
    def slab_shape(self):
        return (self.z1 - self.z0, self.geom.ny, self.geom.nx)

    @property
    def rows_shape(self):
        return (self.geom.n_views, self.r1 - self.r0, self.geom.n_cols)

    def forward(self, vol_slab):
        """Rows [r0, r1) of every view of A vol, from the slices [z0, z1)."""
        import torch
        if self.local is None:
            return torch.zeros(self.rows_shape, dtype=torch.float32, device=vol_slab.device)
        return self.local.forward(vol_slab)

    def back(self, sino_rows):
        """Slices [z0, z1) of A^T y, from the rows [r0, r1) of every view."""
        import torch
        if self.local is None:
            return torch.zeros(self.slab_shape, dtype=torch.float32, device=sino_rows.device)
        return self.local.back(sino_rows)
