"""The FP64 oracle over several host threads, for parity at full size.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests and the
benchmark's CPU-baseline leg call it, the product library never does.  Each
thread runs the unchanged single-threaded oracle (``forward`` / ``back`` of
this package) on its own contiguous range of views; the C oracle keeps no global state and ctypes releases the GIL for the
duration of each call, so the ranges run in parallel.  The forward
concatenates the ranges' sinograms in view order; the back projection sums
the ranges' FP64 partial volumes in range order, so the result does not
depend on thread timing.  Threads, not processes: a pool forked after CUDA
has been initialised would hang.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from oracle import back as _back, forward as _forward


def host_threads() -> int:
    """Threads the oracle may use: the cores this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _ranges(n_views: int, parts: int):
    parts = max(1, min(parts, n_views))
    edges = np.linspace(0, n_views, parts + 1).round().astype(np.int64)
    return [(int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def forward(geom, vol, threads: int = 0) -> np.ndarray:
    """y = A x in FP64, every view, views split over threads."""
    threads = threads or host_threads()
    vol = np.ascontiguousarray(vol, dtype=np.float32)
    ranges = _ranges(geom.n_views, 4 * threads)
    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(lambda r: _forward(geom, vol, views=r), ranges))
    return np.concatenate(parts, axis=0)


def back(geom, sino, power: int = 1, threads: int = 0, max_host_bytes: float = 0.0) -> np.ndarray:
    """x = A^T y in FP64; each thread holds one FP64 partial volume, so the
    thread count is also capped by ``max_host_bytes`` (default: half the
    host memory available now)."""
    threads = threads or host_threads()
    if not max_host_bytes:
        try:
            import psutil
            max_host_bytes = 0.5 * psutil.virtual_memory().available
        except Exception:
            max_host_bytes = 8e9
    vol_bytes = 8.0 * geom.n_vox
    threads = int(max(1, min(threads, max_host_bytes // vol_bytes - 1)))
    sino = np.ascontiguousarray(sino, dtype=np.float32)
    ranges = _ranges(geom.n_views, threads)
    with ThreadPoolExecutor(len(ranges)) as ex:
        parts = list(ex.map(lambda r: _back(geom, sino[r[0]:r[1]], views=r, power=power), ranges))
    total = parts[0]
    for p in parts[1:]:
        total += p
    return total
