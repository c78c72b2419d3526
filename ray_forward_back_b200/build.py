"""Build libctp.so in-tree with nvcc for sm_100a.

    python -m ray_forward_back_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libctp.so")
SOURCES = ["ctp_api.cu", "ctp_kernels.cu", "ctp_grad.cu", "ctp_gather.cu", "ctp_noalloc.cu", "ctp_solvers.cu"]
HEADERS = [os.path.join(CSRC, "ctp_internal.h"), os.path.join(CSRC, "ctp_ray.cuh"), os.path.join(CSRC, "ctp_gather.h"),
           os.path.join(INCLUDE, "ctp.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, out: str = None, defines=()) -> str:
    """Compile the library; ``defines`` are extra -D tuning macros and ``out``
    another output path (the default build goes in-tree)."""
    lib = out or LIB
    if not force and out is None and not defines and not _stale():
        return LIB
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", tmp]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [f"-D{d}" for d in defines]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
