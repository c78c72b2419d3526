"""The gather adjoint's launch map on the CPU: with the tile constants read
from the kernel source, every voxel of the volume is written by exactly one
lane, and every slice-sum group a lane reads lies inside its column, for
ragged sizes, every lane layout (1, 2 or 4 float4 groups per lane) and
several slice chunks.  A mirror of the kernel's index arithmetic, checked
before the kernel ran; the bounds-checked build checks the same indices on
the GPU."""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "ray_forward_back_b200", "csrc",
                   "ctp_gather.cu")


def constants():
    text = open(SRC).read()
    return {k: int(v) for k, v in re.findall(r"constexpr int (kGather(?:TileX|TileY|Super)) = (\d+);", text)}


def launch(nx, ny, nz):
    c = constants()
    tx_, ty_, sup = c["kGatherTileX"], c["kGatherTileY"], c["kGatherSuper"]
    tiles_x, tiles_y = -(-nx // tx_), -(-ny // ty_)
    nz4 = -(-nz // 4) * 4
    g4 = nz4 // 4
    J = 1 if g4 <= 32 else (2 if g4 <= 64 else 4)
    n_zchunks = -(-g4 // (32 * J))
    sgx, sgy = -(-tiles_x // sup), -(-tiles_y // sup)
    per_chunk = sgx * sgy * sup * sup
    return tx_, ty_, sup, tiles_x, tiles_y, g4, J, n_zchunks, sgx, per_chunk


@pytest.mark.parametrize("dims", [(64, 64, 64), (70, 45, 33), (11, 9, 7), (1, 1, 1), (5, 3, 1), (20, 70, 600),
                                  (3, 130, 1100), (9, 10, 200), (512, 8, 512)])
def test_every_voxel_written_once_and_reads_in_bounds(dims):
    nx, ny, nz = dims
    tx_, ty_, sup, tiles_x, tiles_y, g4, J, n_zchunks, sgx, per_chunk = launch(nx, ny, nz)
    blocks = np.arange(per_chunk * n_zchunks)
    zc = blocks // per_chunk
    b = blocks - zc * per_chunk
    grp, in_grp = b // (sup * sup), b % (sup * sup)
    tx = (grp % sgx) * sup + in_grp % sup
    ty = (grp // sgx) * sup + in_grp // sup
    warps = np.arange(tx_ * ty_)
    x = tx[:, None] * tx_ + warps[None, :] % tx_
    y = ty[:, None] * ty_ + warps[None, :] // tx_
    live = (tx < tiles_x)[:, None] & (ty < tiles_y)[:, None] & (x < nx) & (y < ny)
    lanes, js = np.arange(32), np.arange(J)
    q = zc[:, None, None, None] * 32 * J + lanes[None, None, :, None] + 32 * js[None, None, None, :]
    q = np.broadcast_to(q, (len(blocks), len(warps), 32, J))   # the same groups in every warp of a block
    ok = q < g4                                   # the lane's float4 group exists in the column
    assert q[ok].max() < g4 and q.min() >= 0     # reads stay inside the column of g4 groups
    count = np.zeros((nz, ny, nx), np.int64)
    for s in range(4):
        z = 4 * q + s
        sel = live[:, :, None, None] & ok & (z < nz)
        bi, wi, li, ji = np.nonzero(sel)
        np.add.at(count, (z[bi, wi, li, ji], y[bi, wi], x[bi, wi]), 1)
    assert (count == 1).all()
