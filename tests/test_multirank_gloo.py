"""The N > 1 bench path on CPU: two gloo ranks reduce their step times with
bench.reduce_max (max over ranks) and report the whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        ms = bench.reduce_max(local_ms, world)
        value = bench.job_throughput(world, 1.0e12, ms)
        bench.barrier(world)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_job_rate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        ms, value = res[rank]
        assert ms == pytest.approx(15.0)                      # the slower rank's time
        assert value == pytest.approx(2 * 1.0e12 / 15.0e-3)  # both ranks' work over it


def test_single_rank_shortcuts():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_throughput(1, 10.0, 1000.0) == pytest.approx(10.0)
