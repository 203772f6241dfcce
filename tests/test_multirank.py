"""The benchmark's multi-rank path on the CPU: two gloo ranks, no GPU.

Under torchrun every rank runs its own batch (no collective on the data
path); the only cross-rank steps are the timing reduction (the slowest
rank's time) and rank 0's report.  These tests run those steps as two
spawned processes over gloo on 127.0.0.1, and check that a rank that leaves
early ends the other rank's collective with an error instead of a hang.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _max_worker(rank, world, port, q):
    _init(rank, world, port, 60)
    cpu = torch.device("cpu")
    first = bench.max_over_ranks([3.0, 7.5][rank], world, cpu)
    # a second reduction in the same order: the ranks stay in step
    second = bench.max_over_ranks([9.25, 1.0][rank], world, cpu)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, first, second))


def _leaver_worker(rank, world, port, q):
    _init(rank, world, port, 10)
    dist.barrier()
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()  # the message is sent before the process goes
        os._exit(0)      # leaves between steps, with nothing in flight
    try:
        bench.max_over_ranks(1.0, world, torch.device("cpu"))
        q.put((rank, "no error"))
    except Exception as e:  # gloo reports the closed peer or the timeout
        q.put((rank, "error:" + type(e).__name__))


def _run(worker, world=2, timeout=90):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=timeout) for _ in range(world)]
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return dict((r, v) for r, *v in out)


def test_every_rank_gets_the_slowest_time():
    got = _run(_max_worker)
    assert got[0] == got[1] == [7.5, 9.25]


def test_job_rate_counts_all_ranks_over_the_slowest():
    # 2 ranks x 4 steps x 1e9 bytes in 8 ms (the slower rank) = 1e12 bytes/s
    assert bench.job_rate(1e9, 4, 2, 8.0) == pytest.approx(1e12)
    assert bench.job_rate(5.0, 3, 1, 1000.0) == pytest.approx(15.0)
    assert bench.max_over_ranks(4.5, 1, torch.device("cpu")) == 4.5   # no collective at N=1


def test_a_rank_that_leaves_ends_the_others_collective():
    got = _run(_leaver_worker, timeout=120)
    assert got[1] == ["left"]
    assert got[0][0].startswith("error:"), got[0]


def test_reference_arm_prints_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1"])
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args: called.append(args) or {})
    bench.main()
    assert capsys.readouterr().out == "" and not called
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("LOCAL_RANK", "0")
    bench.main()
    assert capsys.readouterr().out.strip() == "{}" and len(called) == 1
