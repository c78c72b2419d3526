"""Matched cell-constant Siddon projector pair for NVIDIA B200 (sm_100a).

The compute path is libctp.so (hand-written CUDA, C ABI in include/ctp.h);
``ray_forward_back_b200.ctp`` is its ctypes binding and
``ray_forward_back_b200.workloads`` builds seeded synthetic inputs.  The
library is loaded on first use, and every call raises if it is missing.
"""
__all__ = ["ctp", "workloads", "build"]
