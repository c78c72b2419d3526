"""GPU-side helpers for the parity tests: run the library through its C ABI
and compare with the oracle under the tolerances the tests state."""
from __future__ import annotations

import numpy as np

import oracle
from ray_forward_back_b200 import build as ctp_build
from ray_forward_back_b200 import ctp

EPS32 = float(np.finfo(np.float32).eps)


def projector(geom, plan=None):
    import torch
    ctp_build.build()
    torch.cuda.init()
    return ctp.Projector(geom, device=torch.cuda.current_device(), plan=plan)


def gpu_forward(P, vol_np):
    import torch
    vol = torch.from_numpy(np.ascontiguousarray(vol_np, dtype=np.float32)).cuda()
    y = P.forward(vol)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def gpu_back(P, sino_np):
    import torch
    sino = torch.from_numpy(np.ascontiguousarray(sino_np, dtype=np.float32)).cuda()
    x = P.back(sino)
    torch.cuda.synchronize()
    return x.cpu().numpy()


def rel_l2(a, ref):
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(np.asarray(a, dtype=np.float64) - ref) / (den if den > 0 else 1.0))


def check_forward(y_gpu, y_ref, chord, min_spacing, label=""):
    """Forward tolerances.

    * relative L2 over the whole sinogram <= 1e-5;
    * per ray, on rays crossing the volume -- chord >= one voxel pitch and
      |y| >= 1e-3 max|y| -- relative error <= 1e-4;
    * every other ray: |error| <= 1e-4 |y| + 1e-6 max|y| (the FP32 crossing
      positions carry an absolute error of a few ulp of the ray length, which
      dominates on grazing rays whose values are small).
    """
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    ymax = float(np.abs(y_ref).max()) if y_ref.size else 0.0
    err = np.abs(y_gpu - y_ref)
    r = rel_l2(y_gpu, y_ref)
    assert r <= 1e-5, f"{label}: forward rel L2 {r:.3e}"
    crossing = (chord >= min_spacing) & (np.abs(y_ref) >= 1e-3 * ymax)
    if np.any(crossing):
        worst = float((err[crossing] / np.abs(y_ref[crossing])).max())
        assert worst <= 1e-4, f"{label}: per-ray rel error {worst:.3e}"
    bound = 1e-4 * np.abs(y_ref) + 1e-6 * ymax
    bad = err > bound
    assert not np.any(bad), f"{label}: {int(bad.sum())} rays beyond the absolute bound, worst {float((err - bound).max()):.3e}"
    return r


def check_back(x_gpu, x_ref, x_count_ref, local_len, label=""):
    """Adjoint tolerances.

    * relative L2 over the whole volume <= 1e-5;
    * per voxel: |error| <= 1e-4 |x| + tau * sum_i |y_i| over the segments of
      voxel j (x_count_ref is the oracle's back projection of |y| with unit
      coefficients), tau = 8 eps32 * local_len: each segment's end points
      carry an FP32 error of a few ulp of the local walk length.
    """
    x_gpu = np.asarray(x_gpu, dtype=np.float64)
    x_ref = np.asarray(x_ref, dtype=np.float64)
    r = rel_l2(x_gpu, x_ref)
    assert r <= 1e-5, f"{label}: back rel L2 {r:.3e}"
    tau = 8 * EPS32 * local_len
    bound = 1e-4 * np.abs(x_ref) + tau * x_count_ref + 1e-30
    err = np.abs(x_gpu - x_ref)
    bad = err > bound
    assert not np.any(bad), f"{label}: {int(bad.sum())} voxels beyond bound, worst ratio {float((err / bound).max()):.3e}"
    return r


def adjoint_mismatch(P, geom, seed=0):
    """|<Ax, y> - <x, A^T y>| / |<Ax, y>| with dot products in FP64 on the GPU."""
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.rand(geom.vol_shape, device="cuda", generator=g, dtype=torch.float32)
    y = torch.rand(geom.sino_shape, device="cuda", generator=g, dtype=torch.float32)
    Ax = P.forward(x)
    Aty = P.back(y)
    lhs = torch.dot(Ax.reshape(-1).double(), y.reshape(-1).double()).item()
    rhs = torch.dot(x.reshape(-1).double(), Aty.reshape(-1).double()).item()
    return abs(lhs - rhs) / abs(lhs)


def oracle_chords(geom):
    """Physical chord of every ray through the volume box (forward of ones)."""
    return oracle.forward(geom, np.ones(geom.vol_shape, np.float32))


def forward_errors(y_gpu, y_ref, chord, min_spacing):
    """Achieved errors of a forward projection under the forward tolerances:
    relative L2; the worst relative error on rays crossing the volume (chord
    >= one pitch and |y| >= 1e-3 max|y|); the worst |error| / max|y| on the
    other rays."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    ymax = float(np.abs(y_ref).max())
    err = np.abs(y_gpu - y_ref)
    crossing = (chord >= min_spacing) & (np.abs(y_ref) >= 1e-3 * ymax)
    return {"rel_l2": rel_l2(y_gpu, y_ref),
            "crossing_rays": int(crossing.sum()),
            "worst_rel_crossing": float((err[crossing] / np.abs(y_ref[crossing])).max()) if crossing.any() else 0.0,
            "worst_abs_other_over_max": float(err[~crossing].max() / ymax) if (~crossing).any() else 0.0}


def back_errors(x_gpu, x_ref):
    """Achieved errors of a back projection under the adjoint tolerances:
    relative L2; the worst relative error on voxels with |x| >= 1e-3 max|x|;
    the worst |error| / max|x| on the other voxels."""
    x_gpu = np.asarray(x_gpu, dtype=np.float64)
    x_ref = np.asarray(x_ref, dtype=np.float64)
    xmax = float(np.abs(x_ref).max())
    err = np.abs(x_gpu - x_ref)
    big = np.abs(x_ref) >= 1e-3 * xmax
    return {"rel_l2": rel_l2(x_gpu, x_ref),
            "checked_voxels": int(big.sum()),
            "worst_rel": float((err[big] / np.abs(x_ref[big])).max()) if big.any() else 0.0,
            "worst_abs_other_over_max": float(err[~big].max() / xmax) if (~big).any() else 0.0}
