"""The bench's multi-rank logic on CPU with two gloo ranks: every rank runs a
replica, the job time is the slowest rank's (all-reduce MAX), the whole-job
throughput counts every rank's work, and only rank 0 runs the reference arm."""
import json
import os
import socket
import subprocess
import sys

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


def test_launch_decision_for_gpus_flag():
    assert bench.launch_decision(1, {}) == "run"
    assert bench.launch_decision(2, {}) == "relaunch"
    assert bench.launch_decision(2, {"WORLD_SIZE": "2"}) == "run"
    assert bench.launch_decision(2, {"WORLD_SIZE": "4"}) == "error"
    assert bench.launch_decision(1, {"WORLD_SIZE": "2"}) == "error"


def test_torchrun_command_one_rank_per_gpu_on_localhost():
    cmd = bench.torchrun_command(4, ["--gpus", "4", "--steps", "3"], 29511, 900)
    assert cmd[:4] == ["timeout", "-k", "60", "900"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29511"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
    assert os.path.basename(cmd[-5]) == "bench.py"


def test_bench_gpus_two_relaunches_two_ranks_on_cpu():
    """`bench.py --gpus 2` started without torchrun starts two ranks itself; the
    reference arm (CPU oracle, rank 0 only) then reports the job's two GPUs."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--workload", "longformer_tiny", "--steps", "1", "--warmup", "0",
                        "--ref-budget", "0.2"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                               # rank 0 alone prints
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2


def test_bench_rejects_a_rank_count_that_differs_from_gpus():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0
