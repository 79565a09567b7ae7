"""The bench's multi-rank logic on CPU with two gloo ranks: every rank runs a
replica, the job time is the slowest rank's (all-reduce MAX), the whole-job
throughput counts every rank's work, and only rank 0 runs the reference arm."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [2.0, 3.5][rank]
        ms = bench._max_over_ranks(dist, my_ms, torch.device("cpu"))
        value = bench.replica_throughput(1e12, world, ms)
        q.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 3.5                                 # the slowest rank sets the job time
        assert value == pytest.approx(2 * 1e12 / 3.5e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench._max_over_ranks(None, 1.25, torch.device("cpu")) == 1.25
    assert bench.replica_throughput(2e12, 1, 2.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup = "longformer_tiny", 1, 0
    bench.run_reference(A())
    assert capsys.readouterr().out == ""
