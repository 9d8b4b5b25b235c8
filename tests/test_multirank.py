"""The multi-rank (N > 1) path of the benchmark on CPU with the gloo backend:
every rank runs an independent replica, the slowest rank's time is taken
(max over ranks) and the whole-job value counts the work of all ranks."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports (r+1) ms for the step and (10 - r) ms for a second timer
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    manager = mp.get_context("spawn").Manager()      # no fork of this multi-threaded process
    out = manager.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: [2.0, 10.0], 1: [2.0, 10.0]}


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 1.0]) == [3.5, 1.0]


def test_whole_job_value_counts_all_ranks():
    # 8 replicas of 70.4 TFLOP each, slowest rank 10 ms: 56.3 PFLOP/s of dense-equivalent work
    assert bench.whole_job_tflops(70.4e12, 8, 10.0) == pytest.approx(56320.0)
    assert bench.whole_job_tflops(70.4e12, 1, 10.0) == pytest.approx(7040.0)
