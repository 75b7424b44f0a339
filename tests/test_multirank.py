"""The multi-rank path of bench.py on CPU: two gloo ranks run the same
collective steps, and the timing aggregation takes the slowest rank."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        # per-rank device times: rank r took 10 + 5 r ms per step
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        e = bench.max_over_ranks(3.0 * (world - rank), world, torch.device("cpu"))
        dist.barrier()
        out[rank] = (t, e, bench.job_rate(65536, world, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        got = dict(out)
    for rank in range(world):
        t, e, rate = got[rank]
        assert t == 15.0          # the slowest rank's time, on every rank
        assert e == 6.0
        assert rate == pytest.approx(2 * 65536 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.job_rate(100, 1, 10.0) == pytest.approx(1e4)
