"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each timing its
own replica, agree on the max over ranks (the job's time is its slowest
rank's), and the tokens counted are all ranks' tokens."""
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


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (10 + r) ms of device time and (20 + 3 r) ms end to end
        dev_ms, e2e_ms = bench.max_over_ranks([10.0 + rank, 20.0 + 3 * rank], world, torch.device("cpu"))
        out[rank] = (dev_ms, e2e_ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        got = dict(out)
    assert got[0] == got[1] == (11.0, 23.0)
    # whole-job throughput: every rank's tokens over the slowest rank's time
    steps, T = 64, 1
    value = steps * T * world / (got[0][0] / 1e3)
    assert value == pytest.approx(2 * 64 / 0.011)


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1, torch.device("cpu")) == [3.0, 4.0]
