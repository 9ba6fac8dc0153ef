"""bench.py's multi-rank bookkeeping on CPU: two gloo ranks with different local times must both
report the slowest rank's time per step and the whole-job throughput (world x one call's useful
FLOPs per step)."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_total_ms = [100.0, 130.0][rank]  # 10 steps; rank 1 is the slower one
        ms, value = bench.whole_job(local_total_ms, 10, 4.0e12, world, device="cpu")
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_whole_job_takes_slowest_rank_and_sums_work():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, value = out[rank]
        assert ms == pytest.approx(13.0)
        assert value == pytest.approx(4.0e12 * 2 / 13.0e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    ms, value = bench.whole_job(80.0, 10, 4.0e12, 1, device="cpu")
    assert ms == pytest.approx(8.0) and value == pytest.approx(500.0)
