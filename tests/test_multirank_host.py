"""The multi-rank bench path on CPU: two gloo ranks on 127.0.0.1 time different local
durations and must both report the whole-job throughput of the slower one."""
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


def _rank(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        value, ms = bench.job_throughput(local_ms[rank], 85 * 10, world, torch.device("cpu"))
        out[rank] = (value, ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    world, port = 2, _free_port()
    local_ms = [120.0, 150.0]
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, local_ms, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        value, ms = res[r]
        assert ms == pytest.approx(150.0)
        # 850 tokens per rank, two ranks, 0.15 s for the job
        assert value == pytest.approx(2 * 850 / 0.150)


def test_single_rank_is_local_time():
    value, ms = bench.job_throughput(50.0, 100, 1, torch.device("cpu"))
    assert ms == 50.0 and value == pytest.approx(2000.0)
