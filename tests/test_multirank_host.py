"""Host logic of the multi-process benchmark path on CPU: two `gloo` ranks.

The linear layer does not shard: N GPUs run N independent replicas with no data-path
collective. What the N > 1 path adds is host logic only. The timed region is bracketed by
barriers, the time reported is the slowest rank's, and the whole-job value counts every rank's
units. The reference arm's ranks other than 0 exit without work. These tests run that logic
with world size 2 on the `gloo` backend.
"""
import datetime
import multiprocessing as mp
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, seconds, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench as b
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b.barrier(world)
        t = b.barrier_max(seconds[rank], world)
        b.barrier(world)
        q.put((rank, t, b.job_rate(1000.0, 10, world, t)))
    finally:
        dist.destroy_process_group()


def _run_ranks(seconds):
    world = len(seconds)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, seconds, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            rank, t, rate = q.get(timeout=120)
            out[rank] = (t, rate)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
                p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return out


def test_two_ranks_report_the_slowest_time_and_the_summed_work():
    out = _run_ranks([0.5, 2.0])  # rank 1 is the slower one
    assert sorted(out) == [0, 1]
    for rank in (0, 1):
        t, rate = out[rank]
        assert t == 2.0
        # 1000 units per step per rank, 10 steps, 2 ranks, over the slowest rank's 2 s
        assert rate == pytest.approx(1000.0 * 10 * 2 / 2.0)


def test_job_rate_is_weak_scaling():
    one = bench.job_rate(15_427_259 * 21, 10, 1, 0.09)
    assert bench.job_rate(15_427_259 * 21, 10, 2, 0.09) == pytest.approx(2 * one)
    assert bench.job_rate(15_427_259 * 21, 10, 8, 0.18) == pytest.approx(4 * one)


def test_barrier_max_is_identity_on_one_rank():
    assert bench.barrier_max(1.25, 1) == 1.25
    bench.barrier(1)  # no process group needed


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    class NoWork:
        def __init__(self):
            raise AssertionError("a rank other than 0 started the oracle")

    monkeypatch.setattr(bench, "CpuSample", NoWork)
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(types.SimpleNamespace(steps=2, warmup=3)) is None
    assert capsys.readouterr().out == ""
