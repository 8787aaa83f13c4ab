"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each
timing its own workload instance; the job time is the max over ranks and
the value aggregates the executed FLOPs of all ranks (weak scaling)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [12.5, 30.0][rank]
    got = bench.max_over_ranks(ms, world, torch.device("cpu"))
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == 30.0 and out[1] == 30.0


def test_aggregate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.aggregate_tflops(78.8e12, 1, 160.0)
    four = bench.aggregate_tflops(78.8e12, 4, 160.0)
    assert abs(four - 4 * one) < 1e-9
    assert abs(one - 78.8 / 0.160) < 1e-9
