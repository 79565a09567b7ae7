#!/usr/bin/env python
"""Benchmark of banded sparse self-attention on B200.

One step = one forward of the whole hot path over one batch of the synthetic
workload (window, global rows/columns, side keys -- whatever the workload has).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0).  `value` is useful in-band TFLOP/s (4*D per attended
pair, all attention patterns of the workload) measured on the device with CUDA
events, inputs resident in HBM, L2 flushed before every timed step; `e2e` is the
same metric through the public API with pinned host buffers and the host<->device
copies inside the timed region.  Under torchrun every rank runs its own replica
of the workload (no collective on the data path: the (batch, head) units are
independent) and the slowest rank's time is reported ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "in-band attention TFLOP/s and % of B200 BF16 tensor peak at n=16K/32K, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2**20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def _kernel_hash():
    h = hashlib.sha256()
    for name in ("band_tc.cu", "ptx.cuh", "swa_kernels.h", "softmax_math.cuh", "side_mean.cuh"):
        with open(os.path.join(ROOT, "sliding_window_global_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per launch of the band kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(workload)
    if not e or e.get("kernel_hash") != _kernel_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def launch_decision(gpus: int, env) -> str:
    """How to run for --gpus N: "run" (this process is the whole job, or one rank of
    a torchrun job of N ranks), "relaunch" (N > 1 without torchrun: start N ranks
    with torchrun), or "error" (torchrun started a different number of ranks)."""
    if "WORLD_SIZE" in env:
        return "run" if int(env["WORLD_SIZE"]) == gpus else "error"
    return "relaunch" if gpus > 1 else "run"


def torchrun_command(gpus: int, argv, port: int, timeout_s: int):
    """One rank per GPU on this node, rendezvous on 127.0.0.1, bounded by timeout."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return ["timeout", "-k", "60", str(timeout_s), *cmd]


def _free_port() -> int:
    import socket
    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        return sck.getsockname()[1]


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), ws
    return None, 0, 1


def _max_over_ranks(dist, x: float, device) -> float:
    """Slowest rank's time: every rank takes part (a host-side all-reduce of one scalar)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(flop_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job useful TFLOP/s: every rank runs one replica of the workload (weak
    scaling), and the job takes as long as the slowest rank."""
    return flop_per_rank * world / (ms_max * 1e-3) / 1e12


def prepare(w, device):
    """Device-resident inputs of one workload, built with the library's own kernels
    (side keys: block means on the device; side and local bias: host bucket
    expansion)."""
    from sliding_window_global_b200.profile_case import device_inputs
    return device_inputs(w, device)


def local_radius(w) -> int:
    from sliding_window_global_b200.profile_case import local_radius as radius
    return radius(w)


def count_flops(w, host):
    from sliding_window_global_b200 import flops
    gl = host["global_idx"].numpy() if host["global_idx"] is not None else None
    vl = host["valid_len"].numpy() if host["valid_len"] is not None else None
    rb = host["rand_blocks"].numpy() if host.get("rand_blocks") is not None else None
    pairs = flops.attended_pairs(w.seq_len, w.window, w.dilation, w.causal, gl, vl, w.batch,
                                 w.num_side, rb)
    return pairs, flops.useful_flops(pairs, w.head_dim)


def time_device(w, plan, dev, steps, warmup, device):
    """Per-step CUDA-event time of one forward, L2 flushed before each step."""
    import torch
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    from sliding_window_global_b200.profile_case import forward_kwargs
    kw = forward_kwargs(w, dev)
    out = torch.empty((w.batch, w.q_heads, w.seq_len, w.head_dim), dtype=w.torch_dtype, device=device)
    lse = torch.empty((w.batch, w.q_heads, w.seq_len), dtype=torch.float32, device=device)
    for _ in range(warmup):
        flush.fill_(1.0)
        plan.forward(dev["q"], dev["k"], dev["v"], out=out, lse=lse, **kw)
    torch.cuda.synchronize()
    if plan.check() != 0:
        raise RuntimeError("device error word set during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    for s in range(steps):
        flush.fill_(float(s))
        starts[s].record()
        plan.forward(dev["q"], dev["k"], dev["v"], out=out, lse=lse, **kw)
        ends[s].record()
        launches += plan.last_launches
    torch.cuda.synchronize()
    if plan.check() != 0:
        raise RuntimeError("device error word set during timing")
    ms = [starts[s].elapsed_time(ends[s]) for s in range(steps)]
    return sum(ms) / steps, launches


def time_backward(w, plan, dev, steps, warmup, device):
    """Per-step CUDA-event time of one backward (dq, dk, dv, and the side keys' gradients
    when the workload has side keys) from the forward's out and lse and a seeded
    upstream gradient, with every term of the workload's pattern, L2 flushed before
    each step."""
    import torch
    from sliding_window_global_b200.profile_case import forward_kwargs
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    out, lse = plan.forward(dev["q"], dev["k"], dev["v"], **forward_kwargs(w, dev))
    g = torch.Generator(device=device).manual_seed(11)
    dout = torch.randn(out.shape, generator=g, device=device).to(out.dtype)
    kw = forward_kwargs(w, dev)
    grads = plan.backward(dev["q"], dev["k"], dev["v"], out, lse, dout, **kw)
    for _ in range(warmup):
        flush.fill_(1.0)
        plan.backward(dev["q"], dev["k"], dev["v"], out, lse, dout, dq=grads[0], dk=grads[1],
                      dv=grads[2], **kw)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    for s in range(steps):
        flush.fill_(float(s))
        starts[s].record()
        plan.backward(dev["q"], dev["k"], dev["v"], out, lse, dout, dq=grads[0], dk=grads[1],
                      dv=grads[2], **kw)
        ends[s].record()
        launches += plan.last_launches
    torch.cuda.synchronize()
    if plan.check() != 0:
        raise RuntimeError("device error word set during the backward")
    return sum(starts[s].elapsed_time(ends[s]) for s in range(steps)) / steps, launches


def time_e2e(w, plan, host, steps, warmup, device):
    """Same metric through the public API with pinned host buffers: every step copies
    its inputs host->device, runs the forward (which builds the side keys from k and
    v on the device) and reads the output and lse back.  Steps are pipelined over two buffer sets on
    three streams (copy-in, compute, copy-out), so the host->device copy of one step
    overlaps the forward and the device->host copy of the previous one; the time is
    taken with CUDA events from the first copy-in to the last copy-out."""
    import torch

    names = [k for k in ("q", "k", "v", "global_idx", "valid_len", "bias", "local_bias",
                         "rand_blocks") if host.get(k) is not None]
    pinned = {k: host[k].contiguous().pin_memory() for k in names}
    h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in names)
    oshape = (w.batch, w.q_heads, w.seq_len, w.head_dim)
    lshape = (w.batch, w.q_heads, w.seq_len)
    nbuf = 2
    dev = [{k: torch.empty_like(pinned[k], device=device) for k in names} for _ in range(nbuf)]
    outs = [(torch.empty(oshape, dtype=w.torch_dtype, device=device),
             torch.empty(lshape, dtype=torch.float32, device=device)) for _ in range(nbuf)]
    host_out = [(torch.empty(oshape, dtype=w.torch_dtype).pin_memory(),
                 torch.empty(lshape, dtype=torch.float32).pin_memory()) for _ in range(nbuf)]
    d2h = host_out[0][0].numel() * host_out[0][0].element_size() + host_out[0][1].numel() * 4
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_comp = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]
    used = [False] * nbuf

    def step(i):
        b = i % nbuf
        d, (o, lse), (ho, hl) = dev[b], outs[b], host_out[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_comp[b])           # the forward that read these inputs is done
            for k in names:
                d[k].copy_(pinned[k], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if used[b]:
                s_comp.wait_event(ev_out[b])          # out of this slot has been read back
            # Transient-Global side keys: block means of k and v, built inside the forward
            plan.forward(d["q"], d["k"], d["v"], window=list(w.window), dilation=list(w.dilation),
                         causal=w.causal, global_idx=d.get("global_idx"),
                         bias=d.get("bias"), valid_len=d.get("valid_len"), out=o, lse=lse,
                         local_bias=d.get("local_bias"), rand_blocks=d.get("rand_blocks"),
                         side_from_kv=bool(w.side_block), stream=s_comp)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(max(1, warmup)):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_comp.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(steps):
        step(i)
    s_in.wait_stream(s_out)
    t1.record(s_in)
    torch.cuda.synchronize()
    if plan.check() != 0:
        raise RuntimeError("device error word set during the end-to-end run")
    return t0.elapsed_time(t1) / steps, h2d, d2h


def cpu_baseline(w, host, budget_s=12.0):
    """The fp64 oracle as it stands, on a bounded sample of query rows of the same
    workload, on all host cores; throughput in useful TFLOP/s."""
    import numpy as np
    import torch

    import oracle
    inp = dict(host)
    if w.side_block:   # the oracle makes its own side keys from the same k/v
        inp["side_k"] = torch.from_numpy(oracle.side_aggregate(host["k"], w.side_block, host["valid_len"]))
        inp["side_v"] = torch.from_numpy(oracle.side_aggregate(host["v"], w.side_block, host["valid_len"]))
    if host.get("local_table") is not None:
        inp["local_bias"] = oracle.expand_local_bias(host["local_table"], local_radius(w))
    prob = oracle.Problem(inp["q"], inp["k"], inp["v"], window=np.array(w.window),
                          dilation=np.array(w.dilation), causal=w.causal,
                          global_idx=inp["global_idx"], side_k=inp.get("side_k"),
                          side_v=inp.get("side_v"), side_block=w.side_block or 16,
                          bias=inp.get("bias"), valid_len=inp["valid_len"], scale=inp["scale"],
                          local_bias=inp.get("local_bias"), rand_blocks=inp.get("rand_blocks"),
                          rand_block=128)
    rng = np.random.default_rng(0)
    total_rows = w.batch * w.q_heads * w.seq_len
    rows = np.sort(rng.choice(total_rows, min(total_rows, 2000), replace=False))
    t = time.perf_counter()
    _, _, cnt = prob.forward(rows)
    dt = time.perf_counter() - t
    # scale the sample to fill the budget
    m = int(min(total_rows, max(len(rows), len(rows) * budget_s / max(dt, 1e-3))))
    rows = np.sort(rng.choice(total_rows, m, replace=False))
    t = time.perf_counter()
    _, _, cnt = prob.forward(rows)
    dt = time.perf_counter() - t
    flop = 4 * w.head_dim * int(cnt.sum())
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{m} of {total_rows} query rows (uniform, seeded), {dt:.1f} s, fp64 C + OpenMP"}


def run_ours(args):
    import torch

    from sliding_window_global_b200 import Plan, workloads
    dist, rank, world = _dist()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    peaks, peak_src = _peaks()

    def one(name, with_extras):
        w = workloads.WORKLOADS[name]
        host, dev = prepare(w, device)
        pairs, flop = count_flops(w, host)
        S = w.num_side
        plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, w.torch_dtype,
                    max_global=w.num_global, num_side=S, side_block=w.side_block or 16)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            ms, launches = time_device(w, plan, dev, args.steps, args.warmup, device)
        ms = _max_over_ranks(dist, ms, device)
        clocks = clk.summary()
        tflops = replica_throughput(flop, world, ms)
        res = {"workload": name, "ms_per_step": ms, "value": tflops, "pairs": pairs,
               "useful_gflop_per_step": flop / 1e9, "gpu_launches": launches, "clocks": clocks,
               "w": w}
        if with_extras:
            e2e_ms, h2d, d2h = time_e2e(w, plan, host, max(3, args.steps // 4), 2, device)
            e2e_ms = _max_over_ranks(dist, e2e_ms, device)
            res["e2e"] = {"value": replica_throughput(flop, world, e2e_ms), "unit": "TFLOP/s",
                          "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
            peak = peaks["bf16_tflops"]
            # dominant kernel = the band kernel; for these workloads it is the only launch
            achieved = flop / (ms * 1e-3) / 1e12
            res["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peak,
                               "unit": "TFLOP/s", "frac": achieved / peak,
                               "traffic": _traffic(name),
                               "peak_source": f"{peak_src} bf16_tflops (burst, cuBLAS)",
                               "kernel": "attn_tc_kernel<D,0> (band)",
                               "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak)}
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(w, host)
            if not args.no_backward and not w.num_global and not w.num_side and not w.local_bias \
                    and not w.num_rand:
                bms, blaunch = time_backward(w, plan, dev, args.steps, args.warmup, device)
                bms = _max_over_ranks(dist, bms, device)
                # useful backward work: five products per attended pair (S, dP, dV, dK, dQ)
                bflop = 2.5 * flop
                res["backward"] = {"workload": name, "value": replica_throughput(bflop, world, bms),
                                   "unit": "TFLOP/s", "ms_per_step": bms,
                                   "useful_gflop_per_step": bflop / 1e9, "gpu_launches": blaunch,
                                   "frac_of_peak": bflop / (bms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                   "kernels": "bwd_delta + bwd_dq_kernel<D> + bwd_dkv_kernel<D>"}
        elif not args.no_backward:
            # secondary workloads: the backward of their full pattern
            bms, blaunch = time_backward(w, plan, dev, args.steps, args.warmup, device)
            bms = _max_over_ranks(dist, bms, device)
            bflop = 2.5 * flop
            res["backward"] = {"value": replica_throughput(bflop, world, bms), "unit": "TFLOP/s",
                               "ms_per_step": bms, "gpu_launches": blaunch}
        plan.close()
        del dev
        torch.cuda.empty_cache()
        return res

    main = one(args.workload, True)
    secs = []
    for name in (args.secondary or "").split(","):
        if name and name != "none" and name != args.workload:
            secs.append(one(name, False))
    if rank == 0:
        w = main.pop("w")
        line = {
            "metric": METRIC, "value": main["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads,
                       "kv_heads": w.kv_heads, "seq_len": w.seq_len, "head_dim": w.head_dim,
                       "window": sorted(set(w.window)), "dilation": sorted(set(w.dilation)),
                       "causal": w.causal, "num_global": w.num_global, "num_side": w.num_side,
                       "padding": w.padding, "useful_gflop_per_step": main["useful_gflop_per_step"],
                       "attended_pairs": main["pairs"],
                       "l2": "L2 flushed (252 MB write) before every timed step",
                       "parallelism": f"replicas x{world}"},
            "roofline": main["roofline"], "e2e": main["e2e"], "gpu_launches": main["gpu_launches"],
            "clocks": main["clocks"],
        }
        if "backward" in main:
            line["backward"] = main["backward"]
        if "cpu_baseline" in main:
            line["cpu_baseline"] = main["cpu_baseline"]
        if secs:
            line["secondary"] = []
            for sec in secs:
                sw = sec.pop("w")
                entry = {
                    "workload": sw.name, "value": sec["value"], "unit": "TFLOP/s",
                    "ms_per_step": sec["ms_per_step"],
                    "frac_of_peak": sec["value"] / world / peaks["bf16_tflops"],
                    "useful_gflop_per_step": sec["useful_gflop_per_step"],
                    "gpu_launches": sec["gpu_launches"], "clocks": sec["clocks"]}
                if "backward" in sec:
                    entry["backward"] = sec["backward"]
                line["secondary"].append(entry)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """Reference arm: the fp64 oracle (this method has no runnable upstream code), on
    the host cores, each step a bounded sample of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    from sliding_window_global_b200 import workloads
    w = workloads.WORKLOADS[args.workload]
    host = workloads.make_inputs(w)
    if w.side_block and host["bias_table"] is not None:
        import torch

        import oracle
        nblk = (w.seq_len + w.side_block - 1) // w.side_block
        host["bias"] = torch.from_numpy(oracle.expand_side_bias(host["bias_table"], w.num_side, nblk))
    per_step = args.ref_budget or max(1.0, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    base = None
    for s in range(args.warmup + args.steps):
        r = cpu_baseline(w, host, budget_s=per_step)
        if s >= args.warmup:
            vals.append(r["value"])
            base = r
    v = float(np.mean(vals))
    line = {"metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads,
                       "kv_heads": w.kv_heads, "seq_len": w.seq_len, "head_dim": w.head_dim},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="swan_swa")
    ap.add_argument("--secondary", default="longt5_tglobal,longformer_base,dilated,longt5_local,bigbird_itc",
                    help="comma-separated workloads timed after the main one (device time only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass timing")
    ap.add_argument("--ref-budget", type=float, default=None,
                    help="reference arm: seconds of oracle work per step (default: fit a few minutes)")
    args = ap.parse_args()
    how = launch_decision(args.gpus, os.environ)
    if how == "error":
        print(f"bench.py: --gpus {args.gpus} but torchrun started WORLD_SIZE="
              f"{os.environ.get('WORLD_SIZE')} ranks", file=sys.stderr)
        sys.exit(2)
    if how == "relaunch":
        # N GPUs were asked for without torchrun: start one rank per GPU ourselves
        cmd = torchrun_command(args.gpus, sys.argv[1:], _free_port(), 1800)
        sys.exit(subprocess.call(cmd))
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
