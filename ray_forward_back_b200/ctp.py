"""Python binding of libctp (ctypes): argument marshalling only.

The names mirror the C ABI in include/ctp.h: ``ctp_geom_create``,
``ctp_forward``, ``ctp_back``, ``ctp_count_updates`` ...  Every step of the
projectors runs in the library's CUDA kernels; there is no fallback.  If the
library is missing or CUDA is unavailable the calls raise.

``Projector`` is the convenience wrapper over a geometry handle that takes
torch CUDA tensors and the current torch stream.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libctp.so")

CTP_OK = 0
CTP_ERR_INVALID_ARGUMENT = 1
CTP_ERR_DEGENERATE_RAY = 2
CTP_ERR_OUT_OF_RANGE = 3
CTP_ERR_UNSUPPORTED = 4
CTP_ERR_OUT_OF_MEMORY = 5
CTP_ERR_CUDA = 6

CTP_BEAM_PARALLEL = 0
CTP_BEAM_CONE = 1
CTP_DET_FLAT = 0
CTP_DET_CYLINDRICAL = 1
CTP_ADJOINT_AUTO = 0
CTP_ADJOINT_BRICK = 1
CTP_ADJOINT_SORT = 2
CTP_ADJOINT_SCATTER = 3
CTP_ADJOINT_GATHER = 4

EXPORTED = ["ctp_geom_create", "ctp_geom_destroy", "ctp_geom_query", "ctp_forward", "ctp_back",
            "ctp_forward_batch", "ctp_back_batch", "ctp_back_power", "ctp_geometry_gradient", "ctp_count_updates", "ctp_forward_noalloc", "ctp_solve", "ctp_solver_workspace_bytes",
            "ctp_debug_error_word", "ctp_status_string", "ctp_last_error_detail", "ctp_version"]
CTP_SOLVER_CGLS = 1
CTP_SOLVER_SIRT = 2


class ctp_plan(ctypes.Structure):
    _fields_ = [("adjoint_variant", ctypes.c_int32), ("brick", ctypes.c_int32 * 3),
                ("view_groups", ctypes.c_int32), ("forward_layout", ctypes.c_int32),
                ("batch_chunk", ctypes.c_int32), ("slice_rows", ctypes.c_int32), ("reserved", ctypes.c_int32 * 8)]


class ctp_geom_desc(ctypes.Structure):
    _fields_ = [("beam", ctypes.c_int32), ("detector", ctypes.c_int32),
                ("n_views", ctypes.c_int64), ("n_rows", ctypes.c_int64), ("n_cols", ctypes.c_int64),
                ("src", ctypes.c_void_p), ("det_c", ctypes.c_void_p),
                ("det_u", ctypes.c_void_p), ("det_v", ctypes.c_void_p),
                ("nx", ctypes.c_int64), ("ny", ctypes.c_int64), ("nz", ctypes.c_int64),
                ("origin", ctypes.c_double * 3), ("spacing", ctypes.c_double * 3),
                ("device", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("plan", ctypes.POINTER(ctp_plan))]


class ctp_geom_info(ctypes.Structure):
    _fields_ = [("n_rays", ctypes.c_int64), ("n_vox", ctypes.c_int64), ("scratch_bytes", ctypes.c_int64),
                ("adjoint_variant", ctypes.c_int32), ("brick", ctypes.c_int32 * 3),
                ("view_groups", ctypes.c_int32), ("n_transposed_views", ctypes.c_int32),
                ("collision_ratio", ctypes.c_double), ("batch_chunk", ctypes.c_int32),
                ("slice_rows", ctypes.c_int32), ("interleaved_slices", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class ctp_solver_options(ctypes.Structure):
    _fields_ = [("method", ctypes.c_int32), ("iterations", ctypes.c_int32), ("atol", ctypes.c_double),
                ("rtol", ctypes.c_double), ("relaxation", ctypes.c_double), ("nonnegative", ctypes.c_int32),
                ("use_x0", ctypes.c_int32)]


class ctp_solver_result(ctypes.Structure):
    _fields_ = [("iterations", ctypes.c_int32), ("converged", ctypes.c_int32)]


class CtpError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{status_string(status)}: {detail}")
        self.status = status
        self.detail = detail


_lib = None


def load(path: str = None):
    """Load libctp.so (built by ``ray_forward_back_b200.build``).  The
    CTP_LIBRARY environment variable selects another build of the library."""
    global _lib
    if _lib is None:
        if path is None:
            path = os.environ.get("CTP_LIBRARY") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"libctp.so is not built ({path}); run python -m ray_forward_back_b200.build")
        lib = ctypes.CDLL(path)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        lib.ctp_geom_create.argtypes = [ctypes.POINTER(ctp_geom_desc), ctypes.POINTER(vp)]
        lib.ctp_geom_create.restype = ctypes.c_int
        lib.ctp_geom_destroy.argtypes = [vp]
        lib.ctp_geom_destroy.restype = None
        lib.ctp_geom_query.argtypes = [vp, ctypes.POINTER(ctp_geom_info)]
        lib.ctp_geom_query.restype = ctypes.c_int
        lib.ctp_forward.argtypes = [vp, vp, vp, vp]
        lib.ctp_forward.restype = ctypes.c_int
        lib.ctp_back.argtypes = [vp, vp, vp, vp]
        lib.ctp_back.restype = ctypes.c_int
        lib.ctp_forward_batch.argtypes = [vp, vp, vp, i64, vp]
        lib.ctp_forward_batch.restype = ctypes.c_int
        lib.ctp_back_batch.argtypes = [vp, vp, vp, i64, vp]
        lib.ctp_back_batch.restype = ctypes.c_int
        lib.ctp_back_power.argtypes = [vp, vp, vp, ctypes.c_int, vp]
        lib.ctp_back_power.restype = ctypes.c_int
        lib.ctp_geometry_gradient.argtypes = [vp, vp, vp, vp, vp]
        lib.ctp_geometry_gradient.restype = ctypes.c_int
        lib.ctp_count_updates.argtypes = [vp, ctypes.POINTER(i64), vp]
        lib.ctp_count_updates.restype = ctypes.c_int
        lib.ctp_forward_noalloc.argtypes = [ctypes.POINTER(ctp_geom_desc), vp, vp, vp]
        lib.ctp_forward_noalloc.restype = ctypes.c_int
        lib.ctp_solver_workspace_bytes.argtypes = [vp, ctypes.c_int32]
        lib.ctp_solver_workspace_bytes.restype = ctypes.c_size_t
        lib.ctp_solve.argtypes = [vp, vp, vp, ctypes.POINTER(ctp_solver_options), vp, ctypes.c_size_t,
                                  ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctp_solver_result), vp]
        lib.ctp_solve.restype = ctypes.c_int
        lib.ctp_debug_error_word.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        lib.ctp_debug_error_word.restype = ctypes.c_int
        lib.ctp_status_string.argtypes = [ctypes.c_int]
        lib.ctp_status_string.restype = ctypes.c_char_p
        lib.ctp_last_error_detail.argtypes = []
        lib.ctp_last_error_detail.restype = ctypes.c_char_p
        lib.ctp_version.argtypes = []
        lib.ctp_version.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().ctp_status_string(status).decode()


def last_error_detail() -> str:
    return load().ctp_last_error_detail().decode()


def _check(status: int):
    if status != CTP_OK:
        raise CtpError(status, last_error_detail())


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream_handle(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


class _Desc:
    """A ctp_geom_desc with the host arrays it points at kept alive."""

    def __init__(self, geom, device: int = 0, plan: Optional[dict] = None):
        self.arrays = [np.ascontiguousarray(a, dtype=np.float64) for a in
                       (geom.src, geom.det_c, geom.det_u, geom.det_v)]
        for a in self.arrays:
            if a.shape != (geom.n_views, 3):
                raise ValueError("per-view vectors must have shape (n_views, 3)")
        d = ctp_geom_desc()
        d.beam, d.detector = int(geom.beam), int(geom.detector)
        d.n_views, d.n_rows, d.n_cols = int(geom.n_views), int(geom.n_rows), int(geom.n_cols)
        d.src, d.det_c, d.det_u, d.det_v = [a.ctypes.data for a in self.arrays]
        d.nx, d.ny, d.nz = int(geom.nx), int(geom.ny), int(geom.nz)
        d.origin[:] = [float(x) for x in geom.origin]
        d.spacing[:] = [float(x) for x in geom.spacing]
        d.device = int(device)
        self.plan = None
        if plan:
            p = ctp_plan()
            p.adjoint_variant = int(plan.get("adjoint_variant", 0))
            p.brick[:] = [int(x) for x in plan.get("brick", (0, 0, 0))]
            p.view_groups = int(plan.get("view_groups", 0))
            p.forward_layout = int(plan.get("forward_layout", 0))
            p.batch_chunk = int(plan.get("batch_chunk", 0))
            p.slice_rows = int(plan.get("slice_rows", 0))
            self.plan = p
            d.plan = ctypes.pointer(p)
        self.desc = d


def ctp_geom_create(geom, device: int = 0, plan: Optional[dict] = None) -> int:
    """Validate and upload a geometry; returns the opaque handle."""
    lib = load()
    desc = _Desc(geom, device, plan)
    h = ctypes.c_void_p()
    _check(lib.ctp_geom_create(ctypes.byref(desc.desc), ctypes.byref(h)))
    return int(h.value)


def ctp_geom_destroy(handle: int) -> None:
    if handle:
        load().ctp_geom_destroy(handle)


def ctp_geom_query(handle: int) -> dict:
    info = ctp_geom_info()
    _check(load().ctp_geom_query(handle, ctypes.byref(info)))
    return {"n_rays": info.n_rays, "n_vox": info.n_vox, "scratch_bytes": info.scratch_bytes,
            "adjoint_variant": info.adjoint_variant, "brick": tuple(info.brick), "view_groups": info.view_groups,
            "n_transposed_views": info.n_transposed_views, "collision_ratio": info.collision_ratio,
            "batch_chunk": info.batch_chunk, "slice_rows": info.slice_rows,
            "interleaved_slices": info.interleaved_slices}


def ctp_forward(handle: int, vol, sino, stream=None) -> None:
    _check(load().ctp_forward(handle, _ptr(vol), _ptr(sino), _stream_handle(stream)))


def ctp_back(handle: int, sino, vol, stream=None) -> None:
    _check(load().ctp_back(handle, _ptr(sino), _ptr(vol), _stream_handle(stream)))


def ctp_forward_batch(handle: int, vol, sino, n_batch: int, stream=None) -> None:
    _check(load().ctp_forward_batch(handle, _ptr(vol), _ptr(sino), int(n_batch), _stream_handle(stream)))


def ctp_back_batch(handle: int, sino, vol, n_batch: int, stream=None) -> None:
    _check(load().ctp_back_batch(handle, _ptr(sino), _ptr(vol), int(n_batch), _stream_handle(stream)))


def ctp_back_power(handle: int, sino, vol, power: int, stream=None) -> None:
    _check(load().ctp_back_power(handle, _ptr(sino), _ptr(vol), int(power), _stream_handle(stream)))


def ctp_geometry_gradient(handle: int, vol, sino_grad, grad, stream=None) -> None:
    _check(load().ctp_geometry_gradient(handle, _ptr(vol), _ptr(sino_grad), _ptr(grad), _stream_handle(stream)))


def ctp_count_updates(handle: int, stream=None) -> int:
    n = ctypes.c_int64()
    _check(load().ctp_count_updates(handle, ctypes.byref(n), _stream_handle(stream)))
    return int(n.value)


def ctp_forward_noalloc(geom, vol, sino, device: int = 0, plan: Optional[dict] = None, stream=None) -> None:
    """Forward projection without any allocation by the library: the
    geometry is passed as a description, scratch is the library's fixed
    device array (see include/ctp.h)."""
    desc = _Desc(geom, device, plan)
    _check(load().ctp_forward_noalloc(ctypes.byref(desc.desc), _ptr(vol), _ptr(sino), _stream_handle(stream)))


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def ctp_solver_workspace_bytes(handle: int, method: int) -> int:
    return int(load().ctp_solver_workspace_bytes(handle, int(method)))


def ctp_solve(handle: int, sino, vol, method: int, iterations: int, atol=0.0, rtol=0.0, relaxation=1.0,
              nonnegative=True, use_x0=False, workspace=None, stream=None):
    """Run CGLS or SIRT; returns (history list, converged).  ``workspace`` is
    a device buffer of at least ctp_solver_workspace_bytes bytes (allocated
    here from torch when omitted)."""
    import torch
    need = ctp_solver_workspace_bytes(handle, method)
    if workspace is None:
        workspace = torch.empty(need + 256, dtype=torch.uint8, device=sino.device)
    base = _ptr(workspace)
    base_aligned = (base + 255) & ~255
    size = int(workspace.numel() * workspace.element_size()) - (base_aligned - base)
    opts = ctp_solver_options(int(method), int(iterations), float(atol), float(rtol), float(relaxation),
                              1 if nonnegative else 0, 1 if use_x0 else 0)
    hist = (ctypes.c_double * (int(iterations) + 1))()
    res = ctp_solver_result()
    _check(load().ctp_solve(handle, _ptr(sino), _ptr(vol), ctypes.byref(opts), base_aligned, size, hist,
                            ctypes.byref(res), _stream_handle(stream)))
    return [hist[i] for i in range(res.iterations + 1)], bool(res.converged)


def ctp_debug_error_word() -> int:
    """Bounds-check record of a CTP_DEBUG build (0: every index in bounds);
    raises CtpError(CTP_ERR_UNSUPPORTED) in other builds."""
    w = ctypes.c_uint64()
    _check(load().ctp_debug_error_word(ctypes.byref(w)))
    return int(w.value)


def ctp_version() -> str:
    return load().ctp_version().decode()


class Projector:
    """Matched forward / back projector on one CUDA device.

    ``forward(vol)`` takes a float32 CUDA tensor (..., nz, ny, nx) and returns
    the sinogram (..., n_views, n_rows, n_cols); ``back(sino)`` the reverse.
    Leading batch dimensions are preserved, empty ones included.  Both run on
    the current torch stream unless a stream is given, and never synchronise.
    """

    def __init__(self, geom, device: int = 0, plan: Optional[dict] = None):
        self.geom = geom
        self.device = device
        self.handle = ctp_geom_create(geom, device, plan)

    def close(self):
        if getattr(self, "handle", 0):
            ctp_geom_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def info(self) -> dict:
        return ctp_geom_query(self.handle)

    def _check_tensor(self, t, shape, name):
        import torch
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda:
            raise TypeError(f"{name} must be a float32 CUDA tensor")
        if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous with shape {tuple(shape)}")

    def _lead(self, t, inner, name):
        """Leading batch shape of t, whose trailing dimensions must be `inner`."""
        import torch
        if not isinstance(t, torch.Tensor) or t.dim() < len(inner):
            raise TypeError(f"{name} must be a float32 CUDA tensor (..., {', '.join(map(str, inner))})")
        lead = tuple(t.shape[: t.dim() - len(inner)])
        self._check_tensor(t, lead + tuple(inner), name)
        return lead

    def forward(self, vol, out=None, stream=None):
        import torch
        lead = self._lead(vol, self.geom.vol_shape, "vol")
        shape = lead + tuple(self.geom.sino_shape)
        if out is None:
            out = torch.empty(shape, dtype=torch.float32, device=vol.device)
        self._check_tensor(out, shape, "out")
        if lead:
            ctp_forward_batch(self.handle, vol, out, math.prod(lead), stream)
        else:
            ctp_forward(self.handle, vol, out, stream)
        return out

    def back(self, sino, out=None, stream=None):
        import torch
        lead = self._lead(sino, self.geom.sino_shape, "sino")
        shape = lead + tuple(self.geom.vol_shape)
        if out is None:
            out = torch.empty(shape, dtype=torch.float32, device=sino.device)
        self._check_tensor(out, shape, "out")
        if lead:
            ctp_back_batch(self.handle, sino, out, math.prod(lead), stream)
        else:
            ctp_back(self.handle, sino, out, stream)
        return out

    def back_power(self, sino, power: int, out=None, stream=None):
        """Back projection with every coefficient raised to ``power`` (1 or 2)."""
        import torch
        self._check_tensor(sino, self.geom.sino_shape, "sino")
        if out is None:
            out = torch.empty(self.geom.vol_shape, dtype=torch.float32, device=sino.device)
        self._check_tensor(out, self.geom.vol_shape, "out")
        ctp_back_power(self.handle, sino, out, power, stream)
        return out

    def geometry_gradient(self, vol, sino_grad, out=None, stream=None):
        """d(loss)/d(src, det_c, det_u, det_v) per view, float64 [n_views, 4, 3],
        given the volume and the loss's gradient on the sinogram."""
        import torch
        self._check_tensor(vol, self.geom.vol_shape, "vol")
        self._check_tensor(sino_grad, self.geom.sino_shape, "sino_grad")
        shape = (self.geom.n_views, 4, 3)
        if out is None:
            out = torch.empty(shape, dtype=torch.float64, device=vol.device)
        if out.dtype != torch.float64 or not out.is_cuda or tuple(out.shape) != shape or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous float64 CUDA tensor of shape {shape}")
        ctp_geometry_gradient(self.handle, vol, sino_grad, out, stream)
        return out

    def solve(self, sino, method="cgls", iterations=10, atol=0.0, rtol=0.0, relaxation=1.0, nonnegative=True,
              x0=None, stream=None):
        """CGLS or SIRT reconstruction; returns (volume, residual history, converged)."""
        import torch
        self._check_tensor(sino, self.geom.sino_shape, "sino")
        m = {"cgls": CTP_SOLVER_CGLS, "sirt": CTP_SOLVER_SIRT}[method]
        vol = torch.empty(self.geom.vol_shape, dtype=torch.float32, device=sino.device)
        if x0 is not None:
            vol.copy_(x0)
        hist, conv = ctp_solve(self.handle, sino, vol, m, iterations, atol, rtol, relaxation, nonnegative,
                               x0 is not None, stream=stream)
        return vol, hist, conv

    def count_updates(self, stream=None) -> int:
        return ctp_count_updates(self.handle, stream)
