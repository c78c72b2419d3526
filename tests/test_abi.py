"""The C-ABI library builds, loads and exports every declared entry point;
host-side validation rejects bad geometry before any CUDA call.  CPU only."""
import ctypes
import os
import re

import numpy as np
import pytest

from ray_forward_back_b200 import build as ctp_build
from ray_forward_back_b200 import ctp
from ray_forward_back_b200 import workloads as W
from tests.helpers import small_geometries

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ctp.h")


@pytest.fixture(scope="module")
def lib():
    ctp_build.build()
    return ctp.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ctp_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "ctp_forward" in names and "ctp_back" in names and "ctp_geom_create" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(ctp.EXPORTED)


def test_status_strings(lib):
    assert ctp.status_string(ctp.CTP_OK) == "ok"
    assert ctp.status_string(ctp.CTP_ERR_CUDA) == "CUDA error"
    assert ctp.ctp_version().count(".") == 2


def _expect(status, geom, plan=None):
    with pytest.raises(ctp.CtpError) as ei:
        ctp.ctp_geom_create(geom, 0, plan)
    assert ei.value.status == status, ei.value.detail
    return ei.value.detail


def _cone():
    return small_geometries()["cone_flat"]


def test_rejects_bad_sizes(lib):
    g = _cone()
    g.n_rows = 0
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, g)
    g = _cone()
    g.nx = -3
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, g)


def test_rejects_non_finite_vectors(lib):
    g = _cone()
    g.det_u = g.det_u.copy()
    g.det_u[2, 1] = np.nan
    assert "view 2" in _expect(ctp.CTP_ERR_INVALID_ARGUMENT, g)


def test_pitch_guards(lib):
    g = _cone()
    g.spacing = (1e-7, 1.0, 1.0)
    _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)
    g.spacing = (1e-3, 20.0, 1.0)
    _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)      # ratio 2e4 > 1e4
    g.spacing = (2e6, 2e6, 2e6)
    _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)


def test_distance_guards(lib):
    # both endpoints beyond 1e6 voxels of the centre
    g = W.make_cone(16, 16, 16, 2, 4, 4, sid=2e6, sdd=4e6)
    assert "1e6" in _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)
    # an endpoint beyond 1e15
    g = W.make_cone(16, 16, 16, 2, 4, 4, sid=2e15, sdd=2e15 + 10)
    assert "1e15" in _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)
    # per-axis pitch enters the distance: 5e5 world units at dx = 0.1 is 5e6 voxels
    g = W.make_cone(16, 16, 16, 2, 4, 4, sid=5e5, sdd=1e6, spacing=(0.1, 0.1, 0.1))
    _expect(ctp.CTP_ERR_OUT_OF_RANGE, g)


def test_source_on_a_pixel_centre_is_degenerate(lib):
    g = W.make_cone(8, 8, 8, 1, 3, 3, sid=20.0, sdd=35.0)
    # put the detector plane through the source, centred on it
    g.det_c = g.src.copy()
    assert "coincides" in _expect(ctp.CTP_ERR_DEGENERATE_RAY, g)


def test_parallel_zero_direction(lib):
    g = small_geometries()["parallel"]
    g.src = g.src.copy()
    g.src[1] = 0
    _expect(ctp.CTP_ERR_DEGENERATE_RAY, g)


def test_cylindrical_needs_cone_and_orthogonal_frame(lib):
    g = small_geometries()["parallel"]
    g.detector = W.DET_CYLINDRICAL
    _expect(ctp.CTP_ERR_UNSUPPORTED, g)
    g = small_geometries()["helical_cyl"]
    g.det_u = g.det_u + 0.1 * g.det_v
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, g)


def test_header_constants_match_the_binding():
    """Every enumerator of include/ctp.h has the binding's value."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    consts = dict((k, int(v)) for k, v in re.findall(r"\b(CTP_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert {"CTP_ADJOINT_GATHER", "CTP_ADJOINT_SCATTER", "CTP_ERR_UNSUPPORTED", "CTP_DET_CYLINDRICAL"} <= set(consts)
    for name, value in consts.items():
        assert getattr(ctp, name) == value, name


def test_bad_plan(lib):
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"adjoint_variant": 7})
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"adjoint_variant": 5})
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"adjoint_variant": -1})
    _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"brick": (0, -1, 0)})
    for chunk in (-1, 3, 8):
        _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"batch_chunk": chunk})
    for rows in (-1, 3, 16):
        _expect(ctp.CTP_ERR_INVALID_ARGUMENT, _cone(), {"slice_rows": rows})


def test_valid_geometry_without_a_gpu_fails_with_cuda_status(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    _expect(ctp.CTP_ERR_CUDA, _cone())


def test_null_arguments(lib):
    h = ctypes.c_void_p()
    assert lib.ctp_geom_create(None, ctypes.byref(h)) == ctp.CTP_ERR_INVALID_ARGUMENT
    assert lib.ctp_forward(None, None, None, None) == ctp.CTP_ERR_INVALID_ARGUMENT
    assert lib.ctp_back(None, None, None, None) == ctp.CTP_ERR_INVALID_ARGUMENT
    assert lib.ctp_forward_batch(None, None, None, 0, None) == ctp.CTP_ERR_INVALID_ARGUMENT
    assert lib.ctp_back_batch(None, None, None, 2, None) == ctp.CTP_ERR_INVALID_ARGUMENT
    lib.ctp_geom_destroy(None)
