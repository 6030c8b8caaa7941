"""The multi-rank aggregation of bench.py (max-over-ranks timing, summed
executed pairs) with world size 2 over gloo on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r: call times (graph, e2e, attention, dense, direct) and pairs (exec, sparse)
        times = torch.tensor([20.0 + rank, 39.0 - rank, 9.7 + 0.1 * rank, 32.5, 21.7 + rank],
                             dtype=torch.float64)
        pairs = torch.tensor([1.7e10 + rank, 1.5e10 + 2 * rank], dtype=torch.float64)
        bench.reduce_over_ranks(dist, times, pairs)
        out[rank] = times.tolist() + pairs.tolist()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_slowest_time_and_summed_pairs():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    want = [21.0, 39.0, 9.8, 32.5, 22.7, 2 * 1.7e10 + 1, 2 * 1.5e10 + 2]
    for r in range(world):
        assert out[r] == pytest.approx(want)
    import bench
    # the job value divides the summed pairs by the slowest rank's time
    assert bench.job_tflops(128, out[0][5], out[0][0]) == pytest.approx(
        4.0 * 128 * (2 * 1.7e10 + 1) / 21.0e-3 / 1e12)


def test_one_rank_is_left_unchanged():
    import bench
    times = torch.tensor([1.0, 2.0])
    pairs = torch.tensor([3.0])
    bench.reduce_over_ranks(None, times, pairs)
    assert times.tolist() == [1.0, 2.0] and pairs.tolist() == [3.0]
