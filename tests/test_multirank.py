"""Host logic of the multi-GPU bench path, on CPU with the gloo backend and two
ranks: every rank runs its own replica, the time is the maximum over ranks,
and the job value counts the work of all replicas."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        got = bench.max_over_ranks(ms, torch.device("cpu"))
        value = bench.job_value(world, steps=4, work_per_step=1e12, max_ms=got)
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_time_is_max_and_value_counts_all_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, got, value in res:
        assert got == 15.0                          # slowest rank
        assert value == pytest.approx(2 * 4 * 1e12 / 0.015)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_value(1, 10, 2e12, 1000.0) == pytest.approx(2e13)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    args = argparse.Namespace(steps=1, warmup=3)
    assert bench.run_reference(args, rank=1, world=2) is None
    assert capsys.readouterr().out == ""
