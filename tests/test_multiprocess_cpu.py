"""The multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

On GPUs every rank runs its own copy of the workload (heads are independent,
no collective on the data path); the only cross-rank steps are the barrier and
the max-over-ranks time, which these tests exercise without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                    # rank 1 is the slow one
        bench.barrier(torch, world)
        m = bench.max_over_ranks(torch, world, local_ms)
        value = bench.job_throughput(65536, 3, world, m)
        q.put((rank, m, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, value in got:
        assert m == 15.0                                   # the slowest rank's time
        assert value == pytest.approx(65536 * 3 * 2 / 0.015)   # all ranks' tokens


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.job_throughput(1000, 4, 1, 2000.0) == pytest.approx(2000.0)
