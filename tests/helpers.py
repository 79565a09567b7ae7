"""Shared helpers of the parity tests: build problems from a workload, run the
CUDA path through the C ABI binding, run the fp64 oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sliding_window_global_b200 import workloads

# Tolerances (fp32: max-abs 1e-4; bf16: max-abs 2e-2 and mean-abs 5e-3 over valid rows).
TOL = {
    "fp32": dict(max_abs=1e-4, mean_abs=1e-4, lse=1e-5),
    "bf16": dict(max_abs=2e-2, mean_abs=5e-3, lse=1e-3),
}


def host_problem(w: workloads.Workload, inp: dict | None = None):
    """Inputs of one workload plus the side keys / bias table both sides consume.

    Side keys/values are the oracle's block means rounded to the workload dtype and
    the side-bias table is the oracle's expansion of the seeded bucket table: these
    are inputs of the attention, made once on the host and fed to both sides."""
    inp = dict(inp) if inp is not None else workloads.make_inputs(w)
    if w.side_block:
        vl = inp["valid_len"]
        sk = oracle.side_aggregate(inp["k"], w.side_block, vl)
        sv = oracle.side_aggregate(inp["v"], w.side_block, vl)
        inp["side_k"] = torch.from_numpy(sk).to(w.torch_dtype)
        inp["side_v"] = torch.from_numpy(sv).to(w.torch_dtype)
        if inp.get("bias_table") is not None:
            nblk = (w.seq_len + w.side_block - 1) // w.side_block
            inp["bias"] = torch.from_numpy(oracle.expand_side_bias(inp["bias_table"], w.num_side, nblk))
    if inp.get("local_table") is not None:
        R = local_radius(w)
        inp["local_bias"] = torch.from_numpy(oracle.expand_local_bias(inp["local_table"], R))
    return inp


def local_radius(w) -> int:
    """Smallest table radius covering every window offset: max over heads of
    min(r * d, n - 1)."""
    return max(min(r * d, w.seq_len - 1) for r, d in zip(w.window, w.dilation))


def oracle_problem(w, inp):
    return oracle.Problem(inp["q"], inp["k"], inp["v"], window=inp["window"].numpy(),
                          dilation=inp["dilation"].numpy(), causal=inp["causal"],
                          global_idx=inp["global_idx"], side_k=inp.get("side_k"),
                          side_v=inp.get("side_v"), side_block=w.side_block or 16,
                          bias=inp.get("bias"), valid_len=inp["valid_len"], scale=inp["scale"],
                          local_bias=inp.get("local_bias"), rand_blocks=inp.get("rand_blocks"),
                          rand_block=128)


def to_dev(inp, device="cuda"):
    out = {}
    for k, v in inp.items():
        if isinstance(v, torch.Tensor) and k not in ("window", "dilation", "bias_table", "local_table"):
            out[k] = v.to(device).contiguous()
        else:
            out[k] = v
    return out


def run_gpu(w, dinp, plan=None, debug=False):
    from sliding_window_global_b200 import Plan
    g = 0 if dinp["global_idx"] is None else int(dinp["global_idx"].shape[-1])
    S = 0 if dinp.get("side_k") is None else int(dinp["side_k"].shape[2])
    if plan is None:
        plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, w.torch_dtype,
                    max_global=g, num_side=S, side_block=w.side_block or 16, debug=debug)
    out, lse = plan.forward(dinp["q"], dinp["k"], dinp["v"], window=dinp["window"],
                            dilation=dinp["dilation"], causal=dinp["causal"],
                            global_idx=dinp["global_idx"], side_k=dinp.get("side_k"),
                            side_v=dinp.get("side_v"), bias=dinp.get("bias"),
                            valid_len=dinp["valid_len"], local_bias=dinp.get("local_bias"),
                            rand_blocks=dinp.get("rand_blocks"))
    torch.cuda.synchronize()
    return out, lse, plan


def compare(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_ref: np.ndarray, lse_ref: np.ndarray,
            dtype: str, what: str = ""):
    """Element-wise comparison on valid rows; padded rows must be exactly 0 / -inf."""
    tol = TOL[dtype]
    valid = ~np.isneginf(lse_ref)
    pad = ~valid
    assert np.all(out_gpu[pad] == 0.0), f"{what}: padded rows not zero"
    assert np.all(np.isneginf(lse_gpu[pad])), f"{what}: padded lse not -inf"
    assert np.all(np.isfinite(out_gpu[valid])), f"{what}: non-finite outputs"
    diff = np.abs(out_gpu[valid].astype(np.float64) - out_ref[valid])
    max_abs = float(diff.max()) if diff.size else 0.0
    mean_abs = float(diff.mean()) if diff.size else 0.0
    lse_err = float(np.abs(lse_gpu[valid] - lse_ref[valid]).max()) if valid.any() else 0.0
    assert max_abs <= tol["max_abs"], f"{what}: max-abs {max_abs:.3e} > {tol['max_abs']}"
    assert mean_abs <= tol["mean_abs"], f"{what}: mean-abs {mean_abs:.3e} > {tol['mean_abs']}"
    assert lse_err <= tol["lse"], f"{what}: lse err {lse_err:.3e} > {tol['lse']}"
    return dict(max_abs=max_abs, mean_abs=mean_abs, lse=lse_err)


def sample_rows(w, inp, count: int, seed: int = 0):
    """Flat row ids (b*Hq+h)*n+i: every head, the first/last tiles, all global rows,
    padding boundary rows, plus seeded random rows."""
    rng = np.random.default_rng(seed)
    B, H, n = w.batch, w.q_heads, w.seq_len
    picks = set()
    edge = [0, 1, 63, 64, 127, 128, 129, n // 2, n - 129, n - 128, n - 1]
    V = w.valid_len
    edge += [V - 2, V - 1, V, V + 1]
    gl = inp["global_idx"]
    for b in range(B):
        for h in range(H):
            for i in edge:
                if 0 <= i < n:
                    picks.add((b * H + h) * n + i)
            if gl is not None:
                for i in gl[b].tolist():
                    picks.add((b * H + h) * n + i)
    extra = rng.integers(0, B * H * n, size=count)
    picks.update(int(x) for x in extra)
    return np.array(sorted(picks), dtype=np.int64)
