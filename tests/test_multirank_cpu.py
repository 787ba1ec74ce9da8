"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
replica; the job's time is the max over ranks and the value is the whole
job's work over that time (weak scaling).  No GPU, no data-path collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        local_ms = 10.0 + 5.0 * rank                  # rank 1 is the slower one
        ms = bench.reduce_max(torch, dist, local_ms, torch.device("cpu"))
        value = bench.job_throughput(ws, 100, 5_732_352, ms)
        out[rank] = (ms, value)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_max_timing_and_weak_scaling_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1]                       # every rank agrees on the job's numbers
    ms, value = out[0]
    assert ms == 15.0                             # the slowest rank's time
    assert value == pytest.approx(2 * 100 * 5_732_352 / 15e-3)


def test_single_rank_identity():
    assert bench.reduce_max(torch, None, 3.5, None) == 3.5
    assert bench.job_throughput(1, 10, 1.0, 1000.0) == 10.0
