"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each timing its
own replica, agree on the slowest rank's time and on the whole-job
throughput (the decode step does not shard, so ranks are replicas and the
only exchange is this max)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms_local = 10.0 * (rank + 1)  # rank 1 is the slower replica
        out[rank] = bench.job_throughput(world, 1, 100, ms_local)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    with mp.get_context("spawn").Manager() as m:  # no fork of this multi-threaded process
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        ms, ms_per_step, value = res[r]
        assert ms == pytest.approx(20.0)
        assert ms_per_step == pytest.approx(0.2)
        assert value == pytest.approx(world * 1 * 100 / 0.020)  # tokens of both replicas over the slowest time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.job_throughput(1, 1, 10, 5.0) == (5.0, 0.5, 10 / 0.005)
