"""The N > 1 host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The gmm has no exchange step, so N GPUs run N independent replicas; what is
shared across ranks is the timing: every rank takes the slowest rank's time
and the whole-job throughput counts every rank's FLOPs.  The reference arm
runs on rank 0 only.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world)
        q.put((rank, ms, bench.job_tflops(1e12, world, 4, ms)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
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
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 4 steps x 1 TFLOP in 15 ms
    assert all(abs(r[2] - 2 * 4 * 1e12 / 0.015 / 1e12) < 1e-9 for r in res)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tflops(2e12, 1, 10, 1000.0) == pytest.approx(20.0)


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload, steps, warmup = "tiny", 1, 0
    bench.run_reference(A)
    assert capsys.readouterr().out == ""
