"""The multi-rank bookkeeping of bench.py on CPU: two gloo ranks, each a
replica with its own device time. Both must see the slowest rank's time, and
the job's throughput counts the tokens of every rank over that time. The
reference arm does its work on rank 0 alone."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

N_TOKENS, STEPS = 32768, 20
LOCAL_MS = (410.0, 437.5)  # rank 1 is the slower replica


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        ms = bench.max_over_ranks(LOCAL_MS[rank], dist, "cpu")
        out[rank] = (ms, bench.replicas_throughput(N_TOKENS, STEPS, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    slow = max(LOCAL_MS)
    want = 2 * N_TOKENS * STEPS / (slow / 1000.0)
    for r in range(2):
        ms, value = res[r]
        assert ms == slow
        assert value == pytest.approx(want, rel=1e-12)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.replicas_throughput(1000, 4, 1, 2.0) == pytest.approx(2e6)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup = 1, 0

    assert bench.run_reference(Args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
