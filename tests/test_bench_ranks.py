"""The multi-GPU bench path on CPU: two gloo ranks combine their step times as the
benchmark does (slowest rank decides the step time, the value counts every rank's work)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 3.5][rank]  # the second rank is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.whole_job_tflops(world, 1e12, ms)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step_and_count_all_work():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value = res[rank]
        assert ms == 3.5
        assert value == pytest.approx(world * 1e12 / 3.5e-3 / 1e12)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.whole_job_tflops(1, 2e12, 2.0) == pytest.approx(1000.0)
