"""The benchmark's multi-rank bookkeeping on two gloo ranks (CPU): every
rank sees the slowest rank's timings and the whole-job throughput counts all
ranks' work over that time."""
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
