"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each timing
its own replica, reduce to the slowest rank's time, and the whole-job rate is
units of all ranks over that time (replicas only; no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r pretends its replica took 10 + r ms per step and 20 + 3 r ms e2e
        total, e2e = bench.max_over_ranks([10.0 + rank, 20.0 + 3 * rank])
        out[rank] = (total, e2e, bench.whole_job_rate(world, 526422120, total) / 1e9)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    # the manager process is spawned too: a fork of this (threaded) process may deadlock
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][:2] == (11.0, 23.0) and res[1][:2] == (11.0, 23.0)
    # 2 replicas x 526.4 MB in 11 ms
    assert abs(res[0][2] - 2 * 526422120 / 11e-3 / 1e9) < 1e-6


def test_single_rank_identity():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_rate(1, 100.0, 1.0) == 100000.0
