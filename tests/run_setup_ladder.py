"""Forward projections of the ladder geometry: a 64^3 cone scan with 16 views
and a 128 x 128 detector at source distances 1e3, 1e5 and 1e6 voxels, each
compared with the FP64 oracle.  Prints one JSON line per (reading, distance)
with the largest relative error over rays with |y| >= 1e-3 max|y| and the
largest error over the largest value.

Run as ``python -m tests.run_setup_ladder``; the library is the one
CTP_LIBRARY names (the FP32-setup ablation build, for instance).  Test
infrastructure: the oracle is called here, never by the library.

Readings of the detector distance, which the pages do not give:
* "twice": the detector as far beyond the centre as the source is before it
  (sdd = 2 sid, the ratio of the 64^3 scan at sid 1e3; at sid 1e6, 2 sid -
  2000 keeps the detector plane within the 1e6-voxel guard), so both ends of
  every ray are about sid from the volume;
* "near": the detector 1000 voxels beyond the centre (sdd = sid + 1000).
The pitch keeps half a voxel at the centre in both.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

SIDS = (1e3, 1e5, 1e6)


def ladder_geometry(sid, reading):
    from ray_forward_back_b200 import workloads as W
    if reading == "twice":
        sdd = 2.0 * sid if sid < 1e6 else 2.0 * sid - 2000.0
    else:
        sdd = sid + 1000.0
    pitch = 0.5 * sdd / sid
    return W.make_cone(64, 64, 64, 16, 128, 128, sid=sid, sdd=sdd, pitch_u=pitch, pitch_v=pitch)


def worst_relative_error(y, ref):
    """Largest per-ray relative error over rays with |y| >= 1e-3 max|y|."""
    m = np.abs(ref) >= 1e-3 * np.abs(ref).max()
    return float((np.abs(y - ref)[m] / np.abs(ref[m])).max())


def max_error_over_max(y, ref):
    """Largest absolute error over the largest value: the sinogram's maximum
    error relative to the sinogram's scale."""
    return float(np.abs(y - ref).max() / np.abs(ref).max())


def main():
    import torch

    import oracle
    from ray_forward_back_b200 import ctp
    from ray_forward_back_b200 import workloads as W
    vol = W.workload(1).phantom()
    vt = torch.from_numpy(vol).cuda()
    for reading in ("twice", "near"):
        for sid in SIDS:
            g = ladder_geometry(sid, reading)
            with ctp.Projector(g, device=torch.cuda.current_device()) as P:
                y = P.forward(vt)
                torch.cuda.synchronize()
                y = y.cpu().numpy().astype(np.float64)
            ref = oracle.forward(g, vol)
            print(json.dumps({"reading": reading, "sid": sid, "worst_rel": worst_relative_error(y, ref),
                              "max_over_max": max_error_over_max(y, ref)}), flush=True)


if __name__ == "__main__":
    main()
