"""Multi-rank host logic of bench.py on CPU: gloo, world size 2.

Beyond one GPU the decode step runs as independent replicas (no collective on
the data path); the only cross-rank steps are the timing reduction (the max
over ranks) and the whole-job throughput.  These run here with the gloo
backend on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # ranks report different elapsed times; every rank must get the max
        elapsed = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        value = bench.job_throughput(world, 4, 8, elapsed)
        out[rank] = (elapsed, value)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_world2():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        elapsed, value = out[r]
        assert elapsed == 15.0
        # 2 replicas x batch 4 x 8 steps in 15 ms
        assert value == pytest.approx(2 * 4 * 8 / 0.015)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(1, 1, 64, 320.0) == pytest.approx(200.0)
