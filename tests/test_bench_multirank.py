"""Host logic of bench.py's N>1 path on CPU: two gloo ranks agree on the
slowest rank's time, and the reported value counts every rank's units."""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        t_ms = 10.0 + 5.0 * rank  # rank 1 is slower
        t_max = bench.max_over_ranks(torch, world, t_ms, device="cpu")
        v = bench.job_throughput(1e6, 100, world, t_max)
        out[rank] = (t_max, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_job_value():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 ranks x 100 steps x 1e6 units over 15 ms
    assert res[0][1] == pytest.approx(2 * 100 * 1e6 / 0.015)
    assert res[0][1] == res[1][1]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(torch, 1, 3.5, device="cpu") == 3.5
    assert bench.job_throughput(2.0, 10, 1, 1000.0) == pytest.approx(20.0)
