"""The benchmark's bookkeeping on the CPU: on two gloo ranks every rank sees
the slowest rank's timings and the whole-job throughput counts all ranks'
work over that time; the digest that keys the committed DRAM-traffic
capture ignores comments only; each plan's kernels, launch count and
traffic model."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [100.0 + 50.0 * rank, 30.0 + rank, 70.0 - rank]
        got = bench.aggregate_over_ranks(mine, world)
        out[rank] = (got, bench.throughput(2_000_000_000, world, got[0]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_work():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        times, value = out[rank]
        assert times == [150.0, 31.0, 70.0]
        # two ranks x 2e9 updates in 150 ms
        assert value == pytest.approx(2 * 2e9 / 0.150 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.aggregate_over_ranks([1.5, 2.0], 1) == [1.5, 2.0]
    assert bench.throughput(1e9, 1, 1000.0) == pytest.approx(1.0)


def test_code_digest_ignores_comments_and_whitespace_only(tmp_path, monkeypatch):
    """The committed DRAM-traffic capture stays valid across comment edits of
    the kernel sources and is voided by any change of code."""
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    a = tmp_path / "a.cu"
    a.write_text("// header\\nint f(int x) {\\n  return x + 1;  /* add one */\\n}\\n")
    d0 = bench.code_digest(["a.cu"])
    a.write_text("// a longer header\\n/* block\\n comment */\\nint f(int x)   {\\n\\n  return x + 1;\\n}\\n")
    assert bench.code_digest(["a.cu"]) == d0
    a.write_text("int f(int x) {\\n  return x + 2;\\n}\\n")
    assert bench.code_digest(["a.cu"]) != d0



def test_committed_kernel_counters_match_the_sources():
    """Every entry of profiles/kernel_counters.json was captured on the kernel
    code as it stands (the digest of its sources matches), so the bench line's
    traffic and issue-rate fraction come from the current kernels."""
    import json
    import os

    import bench
    path = os.path.join(bench.ROOT, "profiles", "kernel_counters.json")
    kernels = json.load(open(path))["kernels"]
    assert {"forward_rows4_kernel", "back_scatter_rows4_kernel", "forward_kernel", "back_scatter_kernel"} <= set(kernels)
    for name, per_workload in kernels.items():
        for wl, k in per_workload.items():
            assert bench.code_digest(k["sources"]) == k["code_sha256"], (name, wl)
            assert bench.kernel_counters(name, int(wl)) is not None
            assert k["updates"] > 0 and k["warp_instructions"] > 0
    f = bench.issue_fraction("forward_rows4_kernel", 4, 3.0e12, 1965.0, 148)
    assert 0.5 < f["frac"] < 1.0 and 0.2 < f["warp_instructions_per_update"] < 0.4
    assert bench.measured_traffic("back_scatter_rows4_kernel", 4, 900) > 1e9


def test_kernel_bookkeeping_of_each_plan():
    """The bench names the kernels of the plan it timed, counts the library's
    launches per step, and scales the gather adjoint's committed DRAM bytes
    by the view count except its output volume, written once."""
    import bench
    gather = {"slice_rows": 4, "interleaved_slices": 1, "adjoint_variant": 4, "n_transposed_views": 450}
    assert bench.kernel_names(gather) == ("forward_rows4_kernel", "back_gather_kernel")
    assert bench.launches_per_step(gather) == 4        # interleave + forward, slice sums + gather
    scatter = dict(gather, adjoint_variant=3)
    assert bench.kernel_names(scatter) == ("forward_rows4_kernel", "back_scatter_rows4_kernel")
    assert bench.launches_per_step(scatter) == 4       # interleave + forward, adjoint + deinterleave
    cone = {"slice_rows": 1, "interleaved_slices": 0, "adjoint_variant": 3, "n_transposed_views": 7}
    assert bench.kernel_names(cone) == ("forward_kernel", "back_scatter_kernel")
    assert bench.launches_per_step(cone) == 4          # transposes on both sides
    k = bench.kernel_counters("back_gather_kernel", 4)
    assert k is not None and 0 < k["fixed_dram_bytes"] < k["dram_bytes"]
    assert bench.measured_traffic("back_gather_kernel", 4, k["views"]) == k["dram_bytes"]
    full = bench.measured_traffic("back_gather_kernel", 4, 15 * k["views"])
    assert full == k["fixed_dram_bytes"] + 15 * (k["dram_bytes"] - k["fixed_dram_bytes"])
