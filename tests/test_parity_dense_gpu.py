"""Dense parity at full size: workloads 2, 3 and 4 element by element.

For each of the three large workloads, an evenly spaced subset of its views
(enough that every adjoint view group spans two stages of 64 views) is
projected at the workload's full volume and detector size, in the launch
configuration of the whole workload (the brick and view groups the full
geometry plans are forced on the subset).  The whole sinogram of the
workload's phantom and the back projection of a dense U[0, 1) sinogram are
compared with the FP64 oracle, run over the host's cores by
``oracle/pool.py``.  Every adjoint variant (brick, sort, scatter) is
checked against the same oracle volume.

Tolerances (the required bounds):
* forward: relative L2 <= 1e-5; per ray <= 1e-4 relative on rays crossing the
  volume (chord >= one pitch, |y| >= 1e-3 max|y|); other rays within
  1e-6 max|y|;
* adjoint: relative L2 <= 1e-5; per voxel <= 1e-4 relative on voxels with
  |x| >= 1e-3 max|x|; other voxels within 1e-6 max|x|.
The achieved values are printed (pytest -s) and, when CTP_PARITY_REPORT names
a file, appended to it as JSON lines.
"""
import json
import os

import numpy as np
import pytest

from ray_forward_back_b200 import workloads as W
from oracle import pool as oracle_pool
from tests.gpu_helpers import back_errors, forward_errors, gpu_back, gpu_forward, projector

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# views of the subset per workload: 2 view groups x 72 (workloads 2, 3) and
# 1 group x 72 (workload 4), i.e. stages of 64 + 8 views in every group
SUBSET_VIEWS = {2: 144, 3: 144, 4: 72}
VARIANTS = {1: "brick", 2: "sort", 3: "scatter"}


def _report(rec):
    print(json.dumps(rec))
    path = os.environ.get("CTP_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


@pytest.mark.parametrize("index", [2, 3, 4])
def test_dense_full_size_parity(index):
    wl = W.workload(index)
    g_full = wl.geom
    P_full = projector(g_full)
    full = P_full.info()
    P_full.close()
    views = np.linspace(0, g_full.n_views - 1, SUBSET_VIEWS[index]).round().astype(np.int64)
    g = g_full.subset_views(views)
    plan = {"brick": full["brick"], "view_groups": full["view_groups"]}

    # forward: the whole sinogram of the subset
    vol = wl.phantom()
    P = projector(g, dict(plan, adjoint_variant=full["adjoint_variant"]))
    info = P.info()
    assert info["brick"] == full["brick"] and info["view_groups"] == full["view_groups"]
    assert info["adjoint_variant"] == full["adjoint_variant"]
    per_group = -(-g.n_views // info["view_groups"])
    assert per_group > 64, "every view group spans at least two stages"
    y = gpu_forward(P, vol)
    P.close()
    y_ref = oracle_pool.forward(g, vol)
    chord = oracle_pool.forward(g, np.ones(g.vol_shape, np.float32))
    fe = forward_errors(y, y_ref, chord, min(g.spacing))
    _report({"workload": index, "views": g.n_views, "direction": "forward", **fe})
    assert fe["crossing_rays"] > 0.1 * g.n_rays
    assert fe["rel_l2"] <= 1e-5
    assert fe["worst_rel_crossing"] <= 1e-4
    assert fe["worst_abs_other_over_max"] <= 1e-6
    del y, y_ref, chord

    # adjoint of a dense sinogram, every variant
    sino = np.random.default_rng(wl.seed + 7).random(g.sino_shape, dtype=np.float32)
    x_ref = oracle_pool.back(g, sino)
    failures = []
    variants = dict(VARIANTS)
    if full["adjoint_variant"] == 4:
        variants[4] = "gather"
    for variant, name in variants.items():
        P = projector(g, dict(plan, adjoint_variant=variant))
        assert P.info()["adjoint_variant"] == variant
        x = gpu_back(P, sino)
        P.close()
        be = back_errors(x, x_ref)
        _report({"workload": index, "views": g.n_views, "direction": "back", "variant": name,
                 "default": variant == full["adjoint_variant"], "brick": list(full["brick"]),
                 "view_groups": full["view_groups"], **be})
        ok = (be["checked_voxels"] > 0.5 * g.n_vox and be["rel_l2"] <= 1e-5 and be["worst_rel"] <= 1e-4
              and be["worst_abs_other_over_max"] <= 1e-6)
        if not ok:
            failures.append((name, be))
    assert not failures, failures
