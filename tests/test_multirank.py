"""The benchmark's multi-rank plumbing on CPU: two gloo ranks.

bench.py runs one independent replica of the workload per GPU (the unit, one
matrix, is independent; there is no data-path collective) and reports the
whole-job throughput over the slowest rank's device time.  Here two CPU
processes exercise the same helpers with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.rank_env()
        ms = 10.0 + 5.0 * rank               # rank-dependent "device time"
        got = bench.max_over_ranks(ms, torch.device("cpu"))
        thr = bench.job_throughput(72, w, 20, got)
        out.put((r, w, lr, got, thr))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, (r, w, lr, got, thr) in enumerate(res):
        assert (r, w, lr) == (rank, 2, rank)
        assert got == 15.0                   # the slowest rank's time
        assert thr == pytest.approx(72 * 2 * 20 / 0.015)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_throughput(72, 1, 10, 1000.0) == pytest.approx(720.0)


def test_reference_arm_other_ranks_do_nothing(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 2, 3, 2

    bench.run_reference(A())
    assert capsys.readouterr().out == ""
