"""Run one workload's forward pass a few times on its seeded device inputs, for
profilers (ncu) and quick timing.  No parity checks; use the tests for those.

    python -m sliding_window_global_b200.profile_case WORKLOAD [--seq-len N] [--batch B] [--reps R]
        [--backward]

The inputs, kernels and launch configuration are those of the bench's timed step
(``device_inputs`` builds the bench's inputs too).
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

from . import Plan, bucket_local_bias, expand_side_bias, side_aggregate, workloads


def local_radius(w) -> int:
    """Radius of the local-bias table: the largest window offset, max min(r*d, n-1)."""
    return max(min(r * d, w.seq_len - 1) for r, d in zip(w.window, w.dilation))


def device_inputs(w, device):
    """Seeded inputs of workload ``w`` (``workloads.make_inputs``) on the device; side
    keys are built by the library's block-mean kernel, the side- and local-bias
    tables by its host bucket expansions.  Returns (host dict, device dict)."""
    inp = workloads.make_inputs(w)
    host = dict(inp)
    dev = {}
    for k in ("q", "k", "v", "global_idx", "valid_len", "rand_blocks"):
        dev[k] = inp[k].to(device) if inp[k] is not None else None
    if w.side_block:
        dev["side_k"] = side_aggregate(dev["k"], w.side_block, dev["valid_len"])
        dev["side_v"] = side_aggregate(dev["v"], w.side_block, dev["valid_len"])
        if inp["bias_table"] is not None:
            nblk = (w.seq_len + w.side_block - 1) // w.side_block
            host["bias"] = expand_side_bias(inp["bias_table"], w.num_side, nblk)
            dev["bias"] = host["bias"].to(device)
    if inp.get("local_table") is not None:
        host["local_bias"] = bucket_local_bias(inp["local_table"], local_radius(w))
        dev["local_bias"] = host["local_bias"].to(device)
    torch.cuda.synchronize(device)
    return host, dev


def forward_kwargs(w, dev) -> dict:
    """Keyword arguments of ``Plan.forward`` for workload ``w``'s device inputs."""
    return dict(window=list(w.window), dilation=list(w.dilation), causal=w.causal,
                global_idx=dev["global_idx"], side_k=dev.get("side_k"), side_v=dev.get("side_v"),
                bias=dev.get("bias"), valid_len=dev["valid_len"], local_bias=dev.get("local_bias"),
                rand_blocks=dev.get("rand_blocks"))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--seq-len", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--backward", action="store_true",
                    help="after the forwards, run the backward pass --reps times")
    a = ap.parse_args(argv)
    w = workloads.WORKLOADS[a.workload]
    if a.seq_len:
        w = dataclasses.replace(w, seq_len=a.seq_len)
    if a.batch:
        w = dataclasses.replace(w, batch=a.batch)
    device = torch.device("cuda", 0)
    _, dev = device_inputs(w, device)
    plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, w.torch_dtype,
                max_global=w.num_global, num_side=w.num_side, side_block=w.side_block or 16)
    for _ in range(a.reps):
        out, _ = plan.forward(dev["q"], dev["k"], dev["v"], **forward_kwargs(w, dev))
    if a.backward:
        out, lse = plan.forward(dev["q"], dev["k"], dev["v"], **forward_kwargs(w, dev))
        dout = torch.randn(out.shape, device=out.device, generator=torch.Generator("cuda").manual_seed(1))
        dout = dout.to(out.dtype)
        for _ in range(a.reps):
            plan.backward(dev["q"], dev["k"], dev["v"], out, lse, dout, window=list(w.window),
                          dilation=list(w.dilation), causal=w.causal, valid_len=dev["valid_len"])
    torch.cuda.synchronize()
    status = plan.check()
    print(f"{w.name} B={w.batch} n={w.seq_len}: status {status}, launches/forward "
          f"{plan.last_launches}, mean |out| {float(out.float().abs().mean()):.4f}")
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
