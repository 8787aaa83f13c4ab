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


@pytest.mark.parametrize("Hq,Hkv,world", [(40, 40, 8), (28, 4, 2), (28, 4, 4), (48, 48, 2)])
def test_head_partition_covers_every_head_once(Hq, Hkv, world):
    sys.path.insert(0, ROOT)
    import bench
    seen_q, seen_kv = [], []
    for r in range(world):
        hq0, hq1, hkv0, hkv1 = bench.head_partition(Hq, Hkv, r, world)
        seen_q += list(range(hq0, hq1))
        seen_kv += list(range(hkv0, hkv1))
        grp = Hq // Hkv
        assert all(h // grp in range(hkv0, hkv1) for h in range(hq0, hq1))     # GQA groups stay whole
    assert seen_q == list(range(Hq)) and seen_kv == list(range(Hkv))


def test_head_partition_rejects_uneven():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(ValueError):
        bench.head_partition(28, 4, 0, 8)


def _gather_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    full = torch.arange(2 * 6 * 5 * 3, dtype=torch.float32).view(2, 6, 5, 3)
    hq0, hq1, _, _ = bench.head_partition(6, 6, rank, world)
    got = bench.gather_heads(full[:, hq0:hq1].contiguous(), world)
    out[rank] = bool(torch.equal(got, full))
    dist.barrier()
    dist.destroy_process_group()


def test_gather_heads_reassembles_the_output_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_gather_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0] and out[1]
