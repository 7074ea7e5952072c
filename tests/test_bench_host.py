"""Host logic of the benchmark's multi-process ("replicas only") mode, on
CPU: two gloo ranks, as torchrun would launch them.  Each rank times its own
replica; the reported time is the maximum over ranks, and every rank takes the
same collective steps."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime as dt
    import bench
    tdist.init_process_group("gloo", rank=rank, world_size=world,
                             timeout=dt.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, got))
    finally:
        tdist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res == {0: 2.5, 1: 2.5}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1, None) == 3.25
    bench.barrier(1)


def test_algorithmic_bytes_gate_shape():
    import bench
    # 8192 x 28672 asymmetric at M = 1: codes + fp16 scales + fp16 zeros + x + y
    assert bench.algorithmic_bytes(1, 8192, 28672, False) == 124_870_656
    assert bench.algorithmic_bytes(1, 4096, 4096, True) == 8_675_328
