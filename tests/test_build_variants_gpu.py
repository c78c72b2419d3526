"""Two compile-time builds of the library, each run in a child process that
loads it through CTP_LIBRARY.

* CTP_DEBUG: every global and shared-memory index of the kernels is checked
  before its access (the memory-safety check of this library; the access is
  skipped and recorded, nothing traps).  Every projector path on the ragged
  geometries and on full-size view subsets of workloads 2-4 must leave the
  record at 0.
* CTP_FP32_SETUP: the per-ray set-up in FP32 instead of FP64, the ablation of
  diffct "Execution", section "Precision, training and reconstruction" (the
  paragraph on FP32 clipping on Apple MPS: max relative sinogram error ~3e-5
  / ~9e-3 / ~4e-2 at source distances 1e3 / 1e5 / 1e6 on a 64^3, 16-view cone
  scan, tests/golden/fp32_clipping_error_ladder.txt).  The FP32 build must
  reproduce that ladder, and the FP64 set-up of the default build stay far
  below it, on the same geometries.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BUILD = os.path.join(ROOT, "_build")

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _build(name, define):
    from ray_forward_back_b200 import build
    os.makedirs(BUILD, exist_ok=True)
    return build.build(out=os.path.join(BUILD, f"libctp_{name}.so"), defines=(define,))


def _child(module, lib, timeout):
    env = dict(os.environ, CTP_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", module], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=timeout)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return r.stdout


def _ladder():
    rows = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "fp32_clipping_error_ladder.txt")):
        if line.strip() and not line.startswith("#"):
            sid, err = line.split()
            rows[float(sid)] = float(err)
    return rows


def test_debug_build_keeps_every_index_in_bounds():
    out = _child("tests.run_debug_paths", _build("debug", "CTP_DEBUG"), 1500)
    word = [line for line in out.splitlines() if line.startswith("debug_word")]
    assert word == ["debug_word 0"], out[-2000:]


def test_fp32_setup_reproduces_the_pages_error_ladder():
    """The pages' "maximum relative sinogram error" is read as the largest
    error over the largest value.  With the detector about as far past the
    centre as the source is before it, the FP32-setup build lands within an
    order of magnitude of each printed value and grows with the source
    distance as they do; with the detector 1000 voxels past the centre it
    barely grows, so that reading does not reproduce the ladder.  The FP64
    set-up of the default build stays below 1e-4 per ray on the same
    geometries, and more than ten times below the FP32 build at 1e5 and 1e6."""
    pages = _ladder()
    out = _child("tests.run_setup_ladder", _build("fp32setup", "CTP_FP32_SETUP"), 900)
    fp32 = {(d["reading"], d["sid"]): d for d in map(json.loads, out.splitlines())}
    print(json.dumps({f"{k[0]} {k[1]:g}": v["max_over_max"] for k, v in fp32.items()}))
    for sid, page in pages.items():
        got = fp32[("twice", sid)]["max_over_max"]
        assert page / 10 <= got <= page * 10, (sid, got, page)
    assert fp32[("twice", 1e5)]["max_over_max"] >= 30 * fp32[("twice", 1e3)]["max_over_max"]
    assert fp32[("near", 1e6)]["max_over_max"] <= 3 * fp32[("near", 1e3)]["max_over_max"]
    # the FP64 set-up of the default build on the same geometries
    import numpy as np

    import oracle
    from ray_forward_back_b200 import workloads as W
    from tests.gpu_helpers import gpu_forward, projector
    from tests.run_setup_ladder import ladder_geometry, max_error_over_max, worst_relative_error
    vol = W.workload(1).phantom()
    for sid in pages:
        g = ladder_geometry(sid, "twice")
        y = gpu_forward(projector(g), vol).astype(np.float64)
        ref = oracle.forward(g, vol)
        assert worst_relative_error(y, ref) <= 1e-4, sid
        if sid >= 1e5:
            assert max_error_over_max(y, ref) < fp32[("twice", sid)]["max_over_max"] / 10, sid
