"""Run one workload's forward pass a few times on random device inputs, for
profilers (ncu) and quick timing.  No parity checks; use the tests for those.

    python -m sliding_window_global_b200.profile_case WORKLOAD [--seq-len N] [--batch B] [--reps R]

The kernels and launch configuration are those of the bench's timed step.
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

from . import Plan, expand_side_bias, side_aggregate, workloads


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--seq-len", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--reps", type=int, default=4)
    a = ap.parse_args(argv)
    w = workloads.WORKLOADS[a.workload]
    if a.seq_len:
        w = dataclasses.replace(w, seq_len=a.seq_len)
    if a.batch:
        w = dataclasses.replace(w, batch=a.batch)
    B, Hq, Hkv, n, D = w.batch, w.q_heads, w.kv_heads, w.seq_len, w.head_dim
    g = torch.Generator("cuda").manual_seed(0)
    q = torch.randn((B, Hq, n, D), device="cuda", generator=g).to(w.torch_dtype)
    k = torch.randn((B, Hkv, n, D), device="cuda", generator=g).to(w.torch_dtype)
    v = torch.randn((B, Hkv, n, D), device="cuda", generator=g).to(w.torch_dtype)
    kw = {}
    if w.side_block:
        kw["side_k"] = side_aggregate(k, w.side_block)
        kw["side_v"] = side_aggregate(v, w.side_block)
        if w.side_bias:
            nblk = (n + w.side_block - 1) // w.side_block
            kw["bias"] = expand_side_bias(torch.randn(Hq, 32), w.num_side, nblk).cuda()
    gl = (torch.arange(w.num_global, dtype=torch.int32, device="cuda").repeat(B, 1)
          if w.num_global else None)
    vl = torch.full((B,), w.valid_len, dtype=torch.int32, device="cuda") if w.padding else None
    plan = Plan(B, n, Hq, Hkv, D, w.torch_dtype, max_global=w.num_global, num_side=w.num_side,
                side_block=w.side_block or 16)
    for _ in range(a.reps):
        out, _ = plan.forward(q, k, v, window=list(w.window), dilation=list(w.dilation),
                              causal=w.causal, global_idx=gl, valid_len=vl, **kw)
    torch.cuda.synchronize()
    status = plan.check()
    print(f"{w.name} B={B} n={n}: status {status}, launches/forward {plan.last_launches}, "
          f"mean |out| {float(out.float().abs().mean()):.4f}")
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
