"""Throughput of the matched Siddon projector pair on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

A step is one forward projection and one back projection of the workload
(default: parallel beam, 512^3 volume, 900 views, 512x736 detector), inputs
resident in HBM.  value = (forward updates + back updates) / step time, in
Gupdates/s (ray-voxel updates).  With N > 1 processes (one per GPU) the
workload is split (strong scaling): --split views (the default) shards the
views, the adjoint's partial volumes reduce-scattered by NCCL into z-slabs;
--split slices shards z-slabs with their detector rows where the slices
decouple (no collective); --split replicas runs a whole copy per rank
(independent problems, weak scaling).  Timings are CUDA events, max over
ranks; rank 0 prints one JSON line.  The geometry gradient is timed on its
own after the single-GPU step and reported under "geometry_gradient"; it is
not part of the step.

--impl reference times the FP64 CPU oracle on a bounded sample of the same
workload (the reference arm; slow by design).  --solver cgls|sirt prints the
solvers' iteration time against one forward + back instead; --batch B the
per-member time of the batched calls against single calls.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fwd & adjoint Gupdates/s (ray-voxel) and achieved HBM GB/s vs roofline, 1 B200"
UNIT = "Gupdates/s"
FALLBACK_HBM_GBS = 6650.0


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(wl):
    g = wl.geom
    beam = "parallel" if g.beam == 0 else ("helical cone" if np.ptp(g.src[:, 2]) > 0 else "circular cone")
    det = "flat" if g.detector == 0 else "cylindrical"
    return {"workload": wl.name, "index": wl.index, "beam": beam, "detector": det,
            "volume_zyx": [g.nz, g.ny, g.nx], "n_views": g.n_views, "detector_rows_cols": [g.n_rows, g.n_cols],
            "seed": wl.seed, "l2": "inputs larger than L2 (volume and sinogram each > 126 MB)"}


def code_digest(paths):
    """SHA-256 of the C++/CUDA code in `paths` with comments and whitespace
    removed: edits to comments do not count as a change of the kernel."""
    import hashlib
    import re
    h = hashlib.sha256()
    for path in paths:
        with open(os.path.join(ROOT, path)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()


def kernel_counters(kernel, workload_index):
    """Committed ncu counters of `kernel` on workload `workload_index`
    (profiles/kernel_counters.json), captured on a view subset of it: DRAM
    bytes and warp instructions per launch there, and the ray-voxel updates
    of that subset.  None when there is no capture for that workload or the
    kernel's code has changed since it was taken (a digest of its sources
    without comments or whitespace)."""
    path = os.path.join(ROOT, "profiles", "kernel_counters.json")
    try:
        with open(path) as f:
            k = json.load(f)["kernels"][kernel][str(workload_index)]
        digest = code_digest(k["sources"])
    except Exception:
        return None
    if digest != k.get("code_sha256"):
        return None
    return k


def measured_traffic(kernel, workload_index, n_views):
    """DRAM bytes of one full launch: the small capture's bytes scaled by the
    view count (each view's rays are an equal share of the work), except a
    part that does not depend on the views (fixed_dram_bytes: the gather
    adjoint's output volume, written once)."""
    k = kernel_counters(kernel, workload_index)
    if k is None:
        return None
    fixed = k.get("fixed_dram_bytes", 0)
    return int(round(fixed + (k["dram_bytes"] - fixed) * n_views / k["views"]))


def issue_fraction(kernel, workload_index, updates_per_s, sm_mhz, n_sm):
    """Achieved updates/s over the instruction-issue ceiling: every SM issues
    at most one warp instruction per clock on each of its four schedulers, so
    the ceiling is (SMs x 4 x clock) / (warp instructions per update), the
    latter from the committed capture."""
    k = kernel_counters(kernel, workload_index)
    if k is None or not sm_mhz:
        return None
    ipu = k["warp_instructions"] / k["updates"]
    ceiling = n_sm * 4 * sm_mhz * 1e6 / ipu
    return {"frac": updates_per_s / ceiling, "warp_instructions_per_update": ipu,
            "ceiling_gupdates_s": ceiling / 1e9, "sm_mhz": sm_mhz, "sms": n_sm}


def kernel_names(info):
    """Names of the step's forward and adjoint kernels for this plan."""
    rows = info.get("slice_rows", 1) > 1
    inter = "4" if info.get("interleaved_slices") else ""
    fwd = f"forward_rows{inter}_kernel" if rows else "forward_kernel"
    back = {1: "back_brick_kernel", 2: "back_sort_kernel",
            3: f"back_scatter_rows{inter}_kernel" if rows else "back_scatter_kernel",
            4: "back_gather_kernel"}[info["adjoint_variant"]]
    return fwd, back


def launches_per_step(info):
    """Kernels of the library launched by one forward + one back projection
    (memsets are not kernels of the library)."""
    t = 1 if info["n_transposed_views"] > 0 else 0
    if info["adjoint_variant"] == 4:                       # slice sums + gather
        fwd = 2 if info.get("interleaved_slices") else 1 + t
        return fwd + 2
    if info.get("interleaved_slices") and info["adjoint_variant"] == 3:
        return 4                      # interleave + forward, adjoint + deinterleave
    if info.get("interleaved_slices"):
        return 2 + 1                  # interleave + forward, adjoint
    fwd = 1 + t                       # transpose_xy + forward
    back = 1 + (t if info["adjoint_variant"] == 3 else 0)   # + transpose_add for the scatter adjoint
    return fwd + back


def host_facts():
    """The host the CPU baseline ran on: core count and CPU model."""
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def algorithmic_bytes(U, n_vox, n_rays):
    """4 B per ray-voxel update (one FP32 voxel read or accumulation) plus the
    compulsory read/write of every voxel and every sinogram element once."""
    return 4.0 * U + 4.0 * n_vox + 4.0 * n_rays


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"ctp_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def aggregate_over_ranks(times_ms, world, device=None):
    """Max over ranks of each timing (barrier semantics: the job is as slow as
    its slowest rank).  Works with any initialised process group (nccl, gloo)."""
    import torch
    t = torch.tensor([float(x) for x in times_ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def throughput(updates_per_rank_step, world, ms_per_step):
    """Whole-job Gupdates/s: every rank's updates over the slowest rank's time."""
    return world * updates_per_rank_step / (ms_per_step * 1e-3) / 1e9


def cpu_oracle_parallel_sample(wl, n_views_sample):
    """The FP64 oracle forward + back over an evenly spaced view subset, the
    views split over one thread per host core (oracle/pool.py).
    Returns (updates/s, wall seconds, updates, threads)."""
    import oracle
    from oracle import pool as oracle_pool
    g = wl.geom
    views = np.linspace(0, g.n_views - 1, n_views_sample).round().astype(np.int64)
    gs = g.subset_views(views)
    vol = np.random.default_rng(wl.seed).random(g.vol_shape, dtype=np.float32)
    sino = np.random.default_rng(wl.seed + 1).random(gs.sino_shape, dtype=np.float32)
    U = oracle.count_updates(gs)
    threads = oracle_pool.host_threads()
    t0 = time.perf_counter()
    oracle_pool.forward(gs, vol, threads=threads)
    oracle_pool.back(gs, sino, threads=threads)
    dt = time.perf_counter() - t0
    return 2 * U / dt, dt, 2 * U, threads


def cpu_oracle_sample(wl, n_views_sample=1):
    """FP64 oracle forward + back over an evenly spaced subset of views, on one
    host core.  Returns (updates/s, seconds, updates, description)."""
    import oracle
    g = wl.geom
    views = np.linspace(0, g.n_views - 1, n_views_sample).round().astype(np.int64)
    gs = g.subset_views(views)
    vol = np.random.default_rng(wl.seed).random(g.vol_shape, dtype=np.float32)
    sino = np.random.default_rng(wl.seed + 1).random(gs.sino_shape, dtype=np.float32)
    U = oracle.count_updates(gs)
    t0 = time.perf_counter()
    oracle.forward(gs, vol)
    oracle.back(gs, sino)
    dt = time.perf_counter() - t0
    desc = (f"FP64 oracle forward + back of {n_views_sample} of {g.n_views} views (evenly spaced) of workload "
            f"{wl.index}, {2 * U} updates, one host thread")
    return 2 * U / dt, dt, 2 * U, desc


def select_workload(args):
    import dataclasses

    from ray_forward_back_b200 import workloads as W
    wl = W.workload(args.workload)
    if args.views and args.views < wl.geom.n_views:
        if args.first >= 0:
            views = np.arange(args.first, min(args.first + args.views, wl.geom.n_views))
            what = f"views {views[0]}-{views[-1]}"
        else:
            views = np.linspace(0, wl.geom.n_views - 1, args.views).round().astype(np.int64)
            what = f"views subset: {args.views}"
        wl = dataclasses.replace(wl, geom=wl.geom.subset_views(views), name=f"{wl.name} ({what})")
    return wl


VARIANTS = {"auto": 0, "brick": 1, "sort": 2, "scatter": 3, "gather": 4}


def plan_of(args):
    """Plan overrides from the command line (none by default)."""
    plan = {}
    if args.variant != "auto":
        plan["adjoint_variant"] = VARIANTS[args.variant]
    if args.slice_rows:
        plan["slice_rows"] = args.slice_rows
    return plan or None


def run_reference(args, rank, world):
    from ray_forward_back_b200 import workloads as W
    if rank != 0:
        return 0
    wl = select_workload(args)
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, 1)
    desc = ""
    for _ in range(args.steps):
        v, dt, U, desc = cpu_oracle_sample(wl, 1)
        vals.append(v / 1e9)
    value = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                             "host": host_facts()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, P, g, wl, vol_host, U, world, dev):
    """End-to-end steps through the public API from and to pinned host
    memory: every step copies its volume and sinogram in and its sinogram and
    volume results out.  Copies run on their own streams with double-buffered
    device buffers, so step k's transfers overlap the neighbouring steps'
    projections; the timed region spans the first copy-in to the last
    copy-out, CUDA events, max over ranks."""
    import torch
    vol_pin = torch.from_numpy(vol_host).pin_memory()
    sino_pin = torch.from_numpy(wl.sinogram()).pin_memory()
    sino_res = torch.empty(g.sino_shape, dtype=torch.float32).pin_memory()
    vol_res = torch.empty(g.vol_shape, dtype=torch.float32).pin_memory()
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    vol_d = [torch.empty(g.vol_shape, dtype=torch.float32, device=dev) for _ in range(2)]
    sino_d = [torch.empty(g.sino_shape, dtype=torch.float32, device=dev) for _ in range(2)]
    y_d = [torch.empty(g.sino_shape, dtype=torch.float32, device=dev) for _ in range(2)]
    x_d = [torch.empty(g.vol_shape, dtype=torch.float32, device=dev) for _ in range(2)]
    done_out = [torch.cuda.Event() for _ in range(2)]   # buffer b free again
    done_comp = [torch.cuda.Event() for _ in range(2)]

    def step(k):
        b = k & 1
        ev_in = torch.cuda.Event()
        s_in.wait_event(done_comp[b])          # inputs of buffer b no longer read
        with torch.cuda.stream(s_in):
            vol_d[b].copy_(vol_pin, non_blocking=True)
            sino_d[b].copy_(sino_pin, non_blocking=True)
        ev_in.record(s_in)
        s_comp.wait_event(ev_in)
        s_comp.wait_event(done_out[b])         # outputs of buffer b already copied out
        P.forward(vol_d[b], out=y_d[b], stream=s_comp)
        ev_y = torch.cuda.Event()
        ev_y.record(s_comp)
        P.back(sino_d[b], out=x_d[b], stream=s_comp)
        done_comp[b].record(s_comp)
        s_out.wait_event(ev_y)
        with torch.cuda.stream(s_out):
            sino_res.copy_(y_d[b], non_blocking=True)
        s_out.wait_event(done_comp[b])
        with torch.cuda.stream(s_out):
            vol_res.copy_(x_d[b], non_blocking=True)
        done_out[b].record(s_out)

    for b in range(2):
        done_out[b].record(s_out)
        done_comp[b].record(s_comp)
    for k in range(max(1, min(args.warmup, 2))):
        step(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_comp.wait_event(t0)
    s_out.wait_event(t0)
    for k in range(args.steps):
        step(k)
    s_in.wait_event(done_out[(args.steps - 1) & 1])
    t1.record(s_in)
    torch.cuda.synchronize(dev)
    e2e_ms = aggregate_over_ranks([t0.elapsed_time(t1) / args.steps], world, dev)[0]
    return {"value": throughput(2 * U, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": int(vol_pin.numel() * 4 + sino_pin.numel() * 4),
            "d2h_bytes_per_step": int(sino_res.numel() * 4 + vol_res.numel() * 4),
            "pipelining": "copies on separate streams, double-buffered device buffers"}


def time_geometry_gradient(args, P, g, vol, sino_grad, stream, U, world, dev):
    """Device time of ctp_geometry_gradient (one traversal of every ray,
    reading the volume and an upstream sinogram gradient), CUDA events on the
    launching stream after warm-up, max over ranks."""
    import torch
    out = torch.empty((g.n_views, 4, 3), dtype=torch.float64, device=dev)
    for _ in range(max(1, args.warmup)):
        P.geometry_gradient(vol, sino_grad, out=out, stream=stream)
    stream.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        P.geometry_gradient(vol, sino_grad, out=out, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = aggregate_over_ranks([t0.elapsed_time(t1) / args.steps], world, dev)[0]
    info = P.info()
    if info.get("interleaved_slices"):
        kernel, launches = "geometry_gradient_rows4_kernel", 2      # interleave + gradient
    else:
        kernel, launches = "geometry_gradient_kernel", 1 + (1 if info["n_transposed_views"] > 0 else 0)
    return {"ms": ms, "gupdates_s": U / (ms * 1e-3) / 1e9, "kernel": kernel, "launches_per_call": launches}


def run_solver(args, rank, world, local_rank):
    """Iteration time of the device solvers (ctp_solve) against one forward +
    back projection of the same workload: every CGLS or SIRT iteration is one
    forward and one adjoint plus a few vector kernels and one host read of
    the step's norms.  Per-iteration time is the difference of two runs of
    different lengths (so the set-up, e.g. SIRT's row and column sums, drops
    out), CUDA events on the launching stream, max over ranks."""
    import torch

    from ray_forward_back_b200 import ctp
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = select_workload(args)
    g = wl.geom
    P = ctp.Projector(g, device=local_rank)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        vol = torch.from_numpy(wl.phantom()).to(dev)
        sino = P.forward(vol, stream=stream)   # consistent data: A x of the phantom
        xo = torch.empty(g.vol_shape, dtype=torch.float32, device=dev)
    stream.synchronize()
    method = args.solver

    def run(iters):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            P.solve(sino, method, iterations=iters, stream=stream)
            e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1)

    for _ in range(max(1, args.warmup)):
        run(2)
    short, long_ = run(2), run(2 + args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        P.forward(vol, out=sino, stream=stream)
        P.back(sino, out=xo, stream=stream)
    e1.record(stream)
    stream.synchronize()
    pair = e0.elapsed_time(e1) / args.steps
    per_iter, short, pair = aggregate_over_ranks([(long_ - short) / args.steps, short, pair], world, dev)
    if rank != 0:
        return 0
    line = {"metric": f"{method} iterations/s on one B200", "value": world * 1000.0 / per_iter,
            "unit": "iterations/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_iteration": per_iter, "setup_ms": short - 2 * per_iter, "projector_pair_ms": pair,
            "overhead_vs_pair": per_iter / pair - 1.0, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 (fp64 ray setup, fp64 norms)", "data": "synthetic",
            "config": workload_config(wl)}
    print(json.dumps(line), flush=True)
    return 0


def run_batch(args, rank, world, local_rank):
    """Per-member time of the batched calls (ctp_forward_batch, ctp_back_batch
    with plan.batch_chunk = min(B, 4)) against the single-volume calls on the
    same workload: B volumes and B sinograms resident in HBM, CUDA events on
    the launching stream, K timed repetitions after W warm-ups, max over
    ranks."""
    import torch

    from ray_forward_back_b200 import ctp
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = select_workload(args)
    g = wl.geom
    B = args.batch
    chunk = 4 if B >= 4 else (2 if B >= 2 else 1)
    P = ctp.Projector(g, device=local_rank, plan={"batch_chunk": chunk})
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        vols = torch.rand((B,) + tuple(g.vol_shape), device=dev)
        sinos = torch.rand((B,) + tuple(g.sino_shape), device=dev)
        yo = torch.empty_like(sinos)
        xo = torch.empty_like(vols)
    stream.synchronize()

    def timed(fn):
        for _ in range(max(1, args.warmup)):
            fn()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) / args.steps

    fwd_b = timed(lambda: P.forward(vols, out=yo, stream=stream)) / B
    back_b = timed(lambda: P.back(sinos, out=xo, stream=stream)) / B
    fwd_1 = timed(lambda: P.forward(vols[0], out=yo[0], stream=stream))
    back_1 = timed(lambda: P.back(sinos[0], out=xo[0], stream=stream))
    fwd_b, back_b, fwd_1, back_1 = aggregate_over_ranks([fwd_b, back_b, fwd_1, back_1], world, dev)
    if rank != 0:
        return 0
    U = P.count_updates(stream=stream)
    line = {"metric": f"batched forward + back Gupdates/s, batch of {B}", "unit": "Gupdates/s",
            "value": world * 2 * U / ((fwd_b + back_b) * 1e-3) / 1e9, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 (fp64 ray setup)", "data": "synthetic", "config": workload_config(wl),
            "batch": B, "batch_chunk": P.info()["batch_chunk"],
            "forward_ms_per_member": fwd_b, "back_ms_per_member": back_b,
            "forward_ms_single": fwd_1, "back_ms_single": back_1,
            "forward_speedup": fwd_1 / fwd_b, "back_speedup": back_1 / back_b}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from ray_forward_back_b200 import ctp
    from ray_forward_back_b200 import workloads as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = select_workload(args)
    g = wl.geom
    P = ctp.Projector(g, device=local_rank, plan=plan_of(args))
    info = P.info()
    stream = torch.cuda.Stream(device=dev)
    vol_host = wl.phantom()
    with torch.cuda.stream(stream):
        vol = torch.from_numpy(vol_host).to(dev)
        sino_in = torch.from_numpy(wl.sinogram()).to(dev)
        sino_out = torch.empty(g.sino_shape, dtype=torch.float32, device=dev)
        vol_out = torch.empty(g.vol_shape, dtype=torch.float32, device=dev)
    stream.synchronize()
    U = P.count_updates(stream=stream)

    def step():
        P.forward(vol, out=sino_out, stream=stream)
        P.back(sino_in, out=vol_out, stream=stream)

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        e0, e1, e2 = ev[k]
        e0.record(stream)
        P.forward(vol, out=sino_out, stream=stream)
        e1.record(stream)
        P.back(sino_in, out=vol_out, stream=stream)
        e2.record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    total_ms = start.elapsed_time(end)
    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(args.steps)]
    back_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(args.steps)]
    (total_ms, fwd_avg, back_avg, fwd_med, back_med, fwd_min, back_min) = aggregate_over_ranks(
        [total_ms, np.mean(fwd_ms), np.mean(back_ms), np.median(fwd_ms), np.median(back_ms), np.min(fwd_ms),
         np.min(back_ms)], world, dev)
    ms_per_step = total_ms / args.steps
    value = throughput(2 * U, world, ms_per_step)

    # end to end through the public API with host buffers (pinned), every step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, P, g, wl, vol_host, U, world, dev)
    # geometry gradients: timed on their own after the step
    grad = None
    if not args.no_extras:
        grad = time_geometry_gradient(args, P, g, vol, sino_in, stream, U, world, dev)
    if rank != 0:
        return 0
    peak, peak_kind = measured_hbm_peak()
    wl_key = wl.index if not args.views else None
    if grad is not None:
        gb = algorithmic_bytes(U, g.n_vox, g.n_rays) / (grad["ms"] * 1e-3) / 1e9
        grad.update({"effective_gbs": gb, "frac_of_hbm": gb / peak,
                     "traffic": measured_traffic(grad["kernel"], wl_key, g.n_views)})
    B = algorithmic_bytes(U, g.n_vox, g.n_rays)
    fwd_kernel, back_kernel = kernel_names(info)
    dominant = "back" if back_avg >= fwd_avg else "forward"
    dom_kernel = back_kernel if dominant == "back" else fwd_kernel
    dom_ms = max(back_avg, fwd_avg)
    achieved = B / (dom_ms * 1e-3) / 1e9
    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    issue_fwd = issue_fraction(fwd_kernel, wl_key, U / (fwd_avg * 1e-3), sm_mhz, n_sm)
    issue_back = issue_fraction(back_kernel, wl_key, U / (back_avg * 1e-3), sm_mhz, n_sm)
    dom_issue = issue_back if dominant == "back" else issue_fwd
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, dt, Ucpu, desc = cpu_oracle_sample(wl, 1)
        cpu = {"value": v / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
               "seconds": round(dt, 2), "host": host_facts()}
        n_par = max(1, min(g.n_views, 2 * host_facts()["nproc"]))
        vp, dtp, Up, threads = cpu_oracle_parallel_sample(wl, n_par)
        cpu["all_cores"] = {"value": vp / 1e9, "unit": UNIT, "threads": threads, "seconds": round(dtp, 2),
                            "sample": f"FP64 oracle forward + back of {n_par} of {g.n_views} views (evenly "
                                      f"spaced), views split over {threads} host threads, {Up} updates",
                            "whole_workload_seconds_estimate": round(2 * U / vp, 1)}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (fp64 ray setup)", "data": "synthetic",
        "config": workload_config(wl),
        "updates_per_direction": U,
        "forward": {"kernel": fwd_kernel, "ms": fwd_avg, "ms_median": fwd_med, "ms_min": fwd_min,
                    "gupdates_s": U / (fwd_avg * 1e-3) / 1e9,
                    "views_s": g.n_views / (fwd_avg * 1e-3),
                    "effective_gbs": B / (fwd_avg * 1e-3) / 1e9,
                    "frac_of_hbm": B / (fwd_avg * 1e-3) / 1e9 / peak,
                    "issue": issue_fwd, "traffic": measured_traffic(fwd_kernel, wl_key, g.n_views),
                    "slice_rows": info.get("slice_rows", 1)},
        "back": {"kernel": back_kernel, "ms": back_avg, "ms_median": back_med, "ms_min": back_min,
                 "gupdates_s": U / (back_avg * 1e-3) / 1e9,
                 "views_s": g.n_views / (back_avg * 1e-3),
                 "effective_gbs": B / (back_avg * 1e-3) / 1e9,
                 "frac_of_hbm": B / (back_avg * 1e-3) / 1e9 / peak,
                 "issue": issue_back, "traffic": measured_traffic(back_kernel, wl_key, g.n_views),
                 "variant": {1: "brick", 2: "sort", 3: "scatter", 4: "gather"}[info["adjoint_variant"]],
                 "collision_ratio": info["collision_ratio"], "slice_rows": info.get("slice_rows", 1)},
        "roofline": {"kernel": dom_kernel,
                     "bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs",
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(dom_kernel, wl_key, g.n_views),
                     "algorithmic_bytes_per_launch": B,
                     "issue_frac": dom_issue["frac"] if dom_issue else None},
        "geometry_gradient": grad,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step(info),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args, rank, world, local_rank):
    """The workload split over `world` GPUs, one process each (strong
    scaling: the job is the whole workload).

    --split views: each rank projects a balanced contiguous shard of the
    views; the forward needs no collective (the volume is replicated); the
    adjoint back-projects the rank's views into a partial volume that NCCL
    reduce-scatters into z-slabs, one per rank.  --split slices (geometries
    whose slices decouple, as workload 4's): each rank owns a z-slab of the
    volume and the detector rows that fall in it; no collective at all.
    Every timing is CUDA events on the rank's stream, then the max over
    ranks; value = all updates of the workload / the slowest rank's step."""
    import torch
    import torch.distributed as dist

    from ray_forward_back_b200 import ctp
    from ray_forward_back_b200.sharded import ShardedProjector, SliceShardedProjector
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = select_workload(args)
    g = wl.geom
    make = lambda geom: ctp.Projector(geom, device=local_rank)
    stream = torch.cuda.Stream(device=dev)
    vol_host = wl.phantom()
    sino_host = wl.sinogram()
    if args.split == "views":
        S = ShardedProjector(g, device=local_rank, make_projector=make)
        vol_in = vol_host                                   # replicated
        sino_part = sino_host[S.v0:S.v1]
        scaling = "strong (view shards + reduce-scatter)"
        shard = {"views": [S.v0, S.v1]}
    else:
        S = SliceShardedProjector(g, make_projector=make)
        vol_in = vol_host[S.z0:S.z1]
        sino_part = sino_host[:, S.r0:S.r1]
        scaling = "strong (slice shards, no collective)"
        shard = {"slices": [S.z0, S.z1], "rows": [S.r0, S.r1]}
    with torch.cuda.stream(stream):
        vol = torch.from_numpy(np.ascontiguousarray(vol_in)).to(dev)
        sino = torch.from_numpy(np.ascontiguousarray(sino_part)).to(dev)
    stream.synchronize()
    U_local = S.local.count_updates(stream=stream) if S.local is not None else 0
    t = torch.tensor([float(U_local)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    U = int(round(t.item()))
    info = S.local.info() if S.local is not None else None

    def step(ev=None):
        with torch.cuda.stream(stream):
            if ev:
                ev[0].record(stream)
            y = S.forward(vol)
            if ev:
                ev[1].record(stream)
            if args.split == "views":
                part = S._partial_back(sino, dev)
                if ev:
                    ev[2].record(stream)
                nz, ny, nx = g.vol_shape
                from ray_forward_back_b200.sharded import z_slab
                z0, z1, h = z_slab(nz, S.rank, S.world)
                if h * S.world != nz:
                    padded = torch.zeros((h * S.world, ny, nx), dtype=part.dtype, device=dev)
                    padded[:nz] = part
                    part = padded
                out = torch.empty((h, ny, nx), dtype=part.dtype, device=dev)
                dist.reduce_scatter_tensor(out, part, op=dist.ReduceOp.SUM)
            else:
                out = S.back(sino)
                if ev:
                    ev[2].record(stream)
            if ev:
                ev[3].record(stream)
        return y, out

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    dist.barrier()
    start.record(stream)
    for k in range(args.steps):
        step(ev[k])
    end.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    # end to end: every step copies this rank's inputs in from pinned host
    # memory and its outputs (sinogram shard, volume slab) back out
    e2e = None
    if not args.no_e2e:
        vin = torch.from_numpy(np.ascontiguousarray(vol_in)).pin_memory()
        sin = torch.from_numpy(np.ascontiguousarray(sino_part)).pin_memory()
        y0, x0 = step()
        yout = torch.empty(tuple(y0.shape), dtype=torch.float32).pin_memory()
        xout = torch.empty(tuple(x0.shape), dtype=torch.float32).pin_memory()
        torch.cuda.synchronize(dev)
        dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                vol.copy_(vin, non_blocking=True)
                sino.copy_(sin, non_blocking=True)
            yk, xk = step()
            with torch.cuda.stream(stream):
                yout.copy_(yk, non_blocking=True)
                xout.copy_(xk, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = aggregate_over_ranks([e0.elapsed_time(e1) / args.steps], world, dev)[0]
        e2e = {"value": 2 * U / (e2e_ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(4 * (vin.numel() + sin.numel())),
               "d2h_bytes_per_step": int(4 * (yout.numel() + xout.numel())),
               "pipelining": "none: copies and projections in order on one stream per rank; bytes of rank 0"}
    fwd = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    back = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    coll = float(np.mean([e[2].elapsed_time(e[3]) for e in ev]))
    total, fwd, back, coll = aggregate_over_ranks([start.elapsed_time(end), fwd, back, coll], world, dev)
    ms_per_step = total / args.steps
    if rank != 0:
        return 0
    n_vox_local = int(np.prod(vol.shape))
    B_local = algorithmic_bytes(U / world, n_vox_local, g.n_rays / world)
    peak, peak_kind = measured_hbm_peak()
    dom_ms = max(fwd, back)
    fwd_kernel, back_kernel = kernel_names(info) if info else ("forward_kernel", "back_scatter_kernel")
    line = {
        "metric": METRIC, "value": 2 * U / (ms_per_step * 1e-3) / 1e9, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": scaling, "vs_baseline": None, "dtype": "f32 (fp64 ray setup)", "data": "synthetic",
        "config": dict(workload_config(wl), split=args.split, parallelism=f"{args.split} x{world}"),
        "updates_per_direction": U,
        "per_rank_max": {"forward_ms": fwd, "back_kernel_ms": back, "collective_ms": coll,
                         "rank0_shard": shard,
                         "collective_bytes_per_rank": int(4 * g.n_vox * (world - 1) / world)
                         if args.split == "views" else 0},
        "roofline": {"kernel": back_kernel if back >= fwd else fwd_kernel, "bound": "hbm",
                     "achieved": B_local / (dom_ms * 1e-3) / 1e9, "peak": peak,
                     "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": B_local / (dom_ms * 1e-3) / 1e9 / peak, "traffic": None,
                     "algorithmic_bytes_per_launch": B_local},
        "clocks": clk, "e2e": e2e,
        "gpu_launches": args.steps * (launches_per_step(info) if info else 0),
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--views", type=int, default=0,
                    help="use this many evenly spaced views of the workload (0 = all); for profiling")
    ap.add_argument("--first", type=int, default=-1,
                    help="with --views: take that many consecutive views from this one instead")
    ap.add_argument("--variant", choices=sorted(VARIANTS), default="auto",
                    help="force an adjoint variant (default: the plan's automatic choice)")
    ap.add_argument("--slice-rows", type=int, default=0, choices=[0, 1, 2, 4, 8],
                    help="force the detector rows per shared (x, y) walk (default: automatic)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the geometry-gradient timing")
    ap.add_argument("--batch", type=int, default=0,
                    help="time the batched calls on this many members against single calls instead")
    ap.add_argument("--solver", choices=["cgls", "sirt"], default=None,
                    help="time solver iterations (against one forward + back) instead of the projector step")
    ap.add_argument("--split", choices=["views", "slices", "replicas"], default=None,
                    help="with several processes: view shards + reduce-scatter (default), z-slab shards "
                         "(slices that decouple), or independent replicas of the whole workload")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    split = args.split or ("views" if world > 1 else "replicas")
    args.split = split
    grouped = world > 1 or (split != "replicas" and "RANK" in os.environ)
    if grouped:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.solver:
            return run_solver(args, rank, world, local_rank)
        if args.batch > 0:
            return run_batch(args, rank, world, local_rank)
        if split != "replicas" and grouped:
            return run_sharded(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if grouped:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
