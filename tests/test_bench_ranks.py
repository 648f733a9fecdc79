"""The bench's multi-rank arithmetic on two gloo ranks (CPU): every rank
learns the slowest rank's time per step, and the whole-job throughput counts
both ranks' work over that time.  (On the GPU the same helpers run over NCCL,
one process per GPU, each rank an independent replica of the step.)"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = (ms, bench.aggregate_tflops(world, 3.6e12, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, times = 2, [3.5, 4.25]
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world, start_method="spawn")
    for rank in range(world):
        ms, v = out[rank]
        assert ms == max(times)
        assert v == pytest.approx(world * 3.6e12 / (max(times) * 1e-3) / 1e12)


def test_single_process_is_unchanged():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.aggregate_tflops(1, 3.6e12, 3.6) == pytest.approx(1000.0)
