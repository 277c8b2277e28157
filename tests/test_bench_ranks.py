"""The multi-rank host logic of bench.py on CPU: two `gloo` ranks (world size 2) agree on the
job's time as the maximum of their local times, and the whole-job value counts every rank's
steps. (On a GPU machine the same functions run over NCCL; every run here has one GPU.)"""
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


def _rank_main(rank, world, port, local_times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(dist, world, local_times[rank], "cpu")
        out[rank] = t
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    world = 2
    local_times = [0.25, 0.75]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), local_times, out), nprocs=world, join=True)
    assert out[0] == out[1] == max(local_times)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(None, 1, 0.5, "cpu") == 0.5


def test_whole_job_value_counts_every_rank():
    # 2 ranks x 10 steps x 30 MB in 0.75 s (the slower rank's time)
    assert bench.whole_job_gbs(2, 10, 30e6, 0.75) == pytest.approx(0.8)
    assert bench.whole_job_gbs(1, 10, 30e6, 0.75) == pytest.approx(0.4)
