"""Every projector path once, through whichever library CTP_LIBRARY names
(the CTP_DEBUG bounds-checked build, for instance), then the bounds-check
record: prints ``debug_word <value>`` (0 when every index stayed in bounds).

Run as ``python -m tests.run_debug_paths``.  Covered: forward, every adjoint
variant (the gather adjoint on the geometries it applies to) with
coefficient powers 1 and 2, batched forward and fused batched
adjoint, shared slice walks, geometry gradients, the update count and the
no-allocation forward, on the ragged geometries of the parity tests; then
view subsets of workloads 2, 3 and 4 at their full volume and detector size.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def exercise(g, torch, ctp, dev, small=True):
    rng = np.random.default_rng(9)
    vol = torch.from_numpy(rng.random(g.vol_shape).astype(np.float32)).to(dev)
    sino = torch.from_numpy(rng.random(g.sino_shape).astype(np.float32)).to(dev)
    plans = [{"adjoint_variant": v} for v in (1, 2, 3, 4)]
    if g.beam == 0:
        plans += [{"adjoint_variant": 3, "slice_rows": r} for r in (2, 4)]
    for plan in plans:
        try:
            P = ctp.Projector(g, device=dev.index, plan=plan)
        except ctp.CtpError as e:
            # the gather adjoint (4) applies to decoupled parallel slices only
            if plan["adjoint_variant"] == 4 and e.status == ctp.CTP_ERR_UNSUPPORTED:
                continue
            raise
        with P:
            P.forward(vol)
            P.back(sino)
            P.back_power(sino, 2)
            if small or plan["adjoint_variant"] == 3:
                P.geometry_gradient(vol, sino)
            if small:
                P.count_updates()
    if small:
        with ctp.Projector(g, device=dev.index, plan={"batch_chunk": 4, "adjoint_variant": 1}) as P:
            vb = torch.rand((3,) + tuple(g.vol_shape), device=dev)
            sb = torch.rand((3,) + tuple(g.sino_shape), device=dev)
            P.forward(vb)
            P.back(sb)
        out = torch.empty(g.sino_shape, dtype=torch.float32, device=dev)
        ctp.ctp_forward_noalloc(g, vol, out, device=dev.index)
    torch.cuda.synchronize()


def main():
    import torch

    from ray_forward_back_b200 import ctp
    from ray_forward_back_b200 import workloads as W
    from tests.test_parity_gpu import ragged_geometries
    from tests.test_slice_rows_gpu import slice_geometries
    dev = torch.device("cuda", torch.cuda.current_device())
    for name, g in sorted(ragged_geometries().items()) + sorted(slice_geometries().items()):
        exercise(g, torch, ctp, dev)
        print("ok", name, flush=True)
    for index, n in ((2, 6), (3, 6), (4, 6)):
        g = W.workload(index).geom
        g = g.subset_views(np.linspace(0, g.n_views - 1, n).round().astype(np.int64))
        exercise(g, torch, ctp, dev, small=False)
        print("ok workload", index, flush=True)
    print("debug_word", ctp.ctp_debug_error_word(), flush=True)


if __name__ == "__main__":
    main()
