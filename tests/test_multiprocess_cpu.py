"""Multi-rank host logic on CPU: gloo ranks on 127.0.0.1.

bench.py: on GPUs rank r owns heads [H r, H (r + 1)) of a job of H x world
heads (heads are independent, no collective on the data path); the only
cross-rank steps are the barrier and the max-over-ranks time.  The sequence split (seqsplit.py)
has one real exchange, the all-gather of segment states and their prefix sum.
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


# ------------------------------------------------ sequence split (row f4) ----
# The exchange logic of symmetric_taylor_self_b200.seqsplit on gloo CPU ranks:
# the per-rank steps run on the float64 oracle (a reference implementation of
# the same four methods), the all-gather and the prefix order are the product
# code's.

class _OracleImpl:
    """Per-rank steps on the oracle: states are float64 CPU tensors."""

    def zero_state(self, B, H, d_K, d_V, P, device):
        import math
        F = math.comb(d_K + P - 1, P - 1)
        return {"S": torch.zeros(B, H, F, d_V, dtype=torch.float64),
                "Z": torch.zeros(B, H, F, dtype=torch.float64), "tokens": 0}

    def _run(self, q, k, v, P, st):
        import oracle
        B, H, n, _ = q.shape
        y = torch.zeros(B, H, n, v.shape[-1], dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                yy, _, S, Z = oracle.scan(q[b, h], k[b, h], v[b, h], P, S=st["S"][b, h].numpy(),
                                          Z=st["Z"][b, h].numpy())
                y[b, h] = torch.from_numpy(yy)
                st["S"][b, h] = torch.from_numpy(S)
                st["Z"][b, h] = torch.from_numpy(Z)
        st["tokens"] += n
        return y

    def segment_state(self, q, k, v, P):
        st = self.zero_state(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], P, None)
        self._run(q, k, v, P, st)
        return st

    def accumulate(self, st, S, Z, tokens):
        st["S"] += S
        st["Z"] += Z
        st["tokens"] += tokens

    def prefill(self, q, k, v, P, st):
        return self._run(q, k, v, P, st)

    @staticmethod
    def tensors(st):
        return st["S"], st["Z"]


def _split_worker(rank, world, port, lens, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from symmetric_taylor_self_b200 import seqsplit
    from symmetric_taylor_self_b200 import workloads as wl

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        qa, ka, va = wl.random_inputs(1, 2, sum(lens), 4, 3, seed=77)
        t0 = sum(lens[:rank])
        sl = slice(t0, t0 + lens[rank])
        y, st = seqsplit.prefill_sequence_split(qa[:, :, sl], ka[:, :, sl], va[:, :, sl], P=3,
                                                impl=_OracleImpl())
        q.put((rank, y.numpy(), st["S"].numpy(), st["Z"].numpy(), st["tokens"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [(40, 40), (23, 50, 31)])
def test_sequence_split_exchange_gloo(lens):
    """G ranks, each with one segment (lengths may differ): the concatenated
    outputs and the last rank's state equal one prefill of the whole sequence."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle
    from symmetric_taylor_self_b200 import workloads as wl

    world = len(lens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, lens, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, y, S, Z, tokens = q.get(timeout=120)
        got[r] = (y, S, Z, tokens)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    qa, ka, va = wl.random_inputs(1, 2, sum(lens), 4, 3, seed=77)
    y_all = np.concatenate([got[r][0] for r in range(world)], axis=2)
    for h in range(2):
        yr, _, Sr, Zr = oracle.scan(qa[0, h], ka[0, h], va[0, h], 3)
        np.testing.assert_allclose(y_all[0, h], yr, rtol=1e-10, atol=1e-12)
        _, S_last, Z_last, tokens = got[world - 1]
        np.testing.assert_allclose(S_last[0, h], Sr, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(Z_last[0, h], Zr, rtol=1e-10, atol=1e-12)
        assert tokens == sum(lens)


def test_reference_arm_json_line(monkeypatch, capsys):
    """The oracle arm on rank 0 prints one JSON line with the contract's keys."""
    import json

    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                                      "--cpu-seconds", "1"])
    assert bench.main() == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_sequence_split_single_rank_without_process_group():
    """Without a process group the split runs as one rank: no exchange, an empty
    prefix, and the outputs of one prefill."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle
    from symmetric_taylor_self_b200 import seqsplit
    from symmetric_taylor_self_b200 import workloads as wl

    q, k, v = wl.random_inputs(1, 2, 37, 3, 2, seed=91)
    y, st = seqsplit.prefill_sequence_split(q, k, v, P=4, impl=_OracleImpl())
    assert st["tokens"] == 37
    for h in range(2):
        yr, _, Sr, Zr = oracle.scan(q[0, h], k[0, h], v[0, h], 4)
        np.testing.assert_allclose(y[0, h].numpy(), yr, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(st["S"][0, h].numpy(), Sr, rtol=1e-12, atol=1e-12)


def test_rank_head_shards_partition_one_job():
    """The shards the ranks draw (workloads.make_inputs with h0, H_total) are the
    heads of one larger job: concatenated in rank order they equal the inputs of
    the same workload with H x world heads."""
    import dataclasses
    sys.path.insert(0, ROOT)
    from symmetric_taylor_self_b200 import workloads as wl
    w = dataclasses.replace(wl.WORKLOADS["prefill_d16"], N=256)
    world = 3
    shards = [wl.make_inputs(w, h0=r * w.H, H_total=w.H * world)[0] for r in range(world)]
    big = dataclasses.replace(w, H=w.H * world)
    whole = wl.make_inputs(big)[0]
    for i in range(3):
        assert torch.equal(torch.cat([sh[i] for sh in shards], dim=1), whole[i])
    assert not torch.equal(shards[0][0], shards[1][0])
