"""GPU parity of the backward pass (swa_backward through the C ABI) against the
fp64 oracle's gradients on the same seeded inputs.

The device forward supplies out and lse (as a training step would); the oracle
recomputes its own in fp64.  Tolerance, from the arithmetic: P and dS enter the
tensor-core products rounded to bf16 (relative 2^-9 each), out and dout are bf16
(Delta = rowsum(dout * out) inherits out's rounding), accumulation is fp32.
Summed over a row's keys these give relative errors of a few 1e-3 of the
gradient's scale, so each gradient is compared against its own magnitude: the
max error within 2e-2 of max |grad| and the mean error within 1e-2 of mean |grad|,
magnitudes floored at 1e-3 (a gradient that is exactly 0 in exact arithmetic,
e.g. dq with a one-key window, comes out at rounding level, ~1e-6).
"""
import dataclasses

import numpy as np
import pytest
import torch

from sliding_window_global_b200 import Plan, workloads
from tests import helpers

pytestmark = pytest.mark.gpu

REL_MAX, REL_MEAN = 2e-2, 1e-2


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _small(base, **kw):
    return dataclasses.replace(workloads.SMALL[base], **kw)


CASES = [
    ("causal_gqa_d128", _small("swan_swa")),
    ("noncausal_d64_pad", _small("longt5_tglobal", side_block=0, side_bias=False, padding=51)),
    ("dilated_heads", _small("dilated", num_global=0, global_mode="none")),
    ("causal_dilated_d128", _small("swan_swa", dilation=(1, 1, 1, 1, 2, 2, 2, 2), window=(40,) * 8)),
    ("window_covers_seq", _small("longformer_base", window=(5000,) * 4, num_global=0,
                                 global_mode="none", seq_len=300)),
    ("r0", _small("longformer_base", window=(0,) * 4, num_global=0, global_mode="none")),
    ("tiny_ragged", _small("dilated", seq_len=77, batch=2, num_global=0, global_mode="none",
                           window=(9,) * 4, dilation=(1, 2, 1, 3))),
    ("gqa_d64_ragged", _small("swan_swa", head_dim=64, seq_len=333, window=(90,) * 8,
                              causal=False)),
]


def run_backward(w, seed=77):
    inp = helpers.host_problem(w)
    dinp = helpers.to_dev(inp)
    out, lse, plan = helpers.run_gpu(w, dinp)
    g = torch.Generator("cpu").manual_seed(seed)
    dout = torch.randn(out.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = plan.backward(dinp["q"], dinp["k"], dinp["v"], out, lse, dout.cuda(),
                               window=dinp["window"], dilation=dinp["dilation"],
                               causal=dinp["causal"], valid_len=dinp["valid_len"])
    torch.cuda.synchronize()
    assert plan.check() == 0
    assert plan.last_launches == 3
    ref = helpers.oracle_problem(w, inp).backward(dout)
    return (dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()), ref


def compare_grads(got, ref, what):
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(a)), f"{what} {name}: non-finite"
        err = np.abs(a.astype(np.float64) - b)
        scale_max = max(float(np.abs(b).max()), 1e-3)
        scale_mean = max(float(np.abs(b).mean()), 1e-3)
        print(f"{what} {name}: max err {err.max():.2e} (scale {scale_max:.2e}), "
              f"mean err {err.mean():.2e} (scale {scale_mean:.2e})")
        assert err.max() <= REL_MAX * scale_max, f"{what} {name}: max err {err.max():.3e} vs {scale_max:.3e}"
        assert err.mean() <= REL_MEAN * scale_mean, f"{what} {name}: mean err {err.mean():.3e} vs {scale_mean:.3e}"


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(name, w):
    _need_gpu()
    got, ref = run_backward(w)
    compare_grads(got, ref, name)


def test_backward_padded_rows_and_keys_are_zero():
    _need_gpu()
    w = _small("longt5_tglobal", side_block=0, side_bias=False, padding=200)
    (dq, dk, dv), _ = run_backward(w)
    V = w.valid_len
    assert np.all(dq[:, :, V:] == 0) and np.all(dk[:, :, V:] == 0) and np.all(dv[:, :, V:] == 0)


# The full pattern: global rows and columns (BigBird §3.2.3), side keys with their
# bias (LongT5 guide, Transient-Global), the local relative bias (LongT5 guide,
# 相对位置编码) and random blocks (BigBird §3.2.2), each against the oracle's backward.
FULL_CASES = [
    ("globals_padding", workloads.SMALL["longformer_base"]),
    ("globals_dilated", workloads.SMALL["dilated"]),
    ("side_keys_bias", workloads.SMALL["longt5_tglobal"]),
    ("local_bias_padding", workloads.SMALL["longt5_local"]),
    ("random_globals_padding", workloads.SMALL["bigbird_itc"]),
    ("side_globals_local", _small("longt5_tglobal", num_global=9, global_mode="random", local_bias=True,
                                  padding=30)),
    ("globals_gqa_d128", _small("swan_swa", causal=False, num_global=7, global_mode="random",
                                window=(60,) * 8, padding=13)),
    ("random_d128_gqa", _small("swan_swa", causal=False, num_rand=2, window=(100,) * 8, seq_len=1100)),
]


def run_full_backward(w, seed=78):
    inp = helpers.host_problem(w)
    dinp = helpers.to_dev(inp)
    out, lse, plan = helpers.run_gpu(w, dinp)
    g = torch.Generator("cpu").manual_seed(seed)
    dout = torch.randn(out.shape, generator=g).to(torch.bfloat16)
    grads = plan.backward(dinp["q"], dinp["k"], dinp["v"], out, lse, dout.cuda(),
                          window=dinp["window"], dilation=dinp["dilation"], causal=dinp["causal"],
                          valid_len=dinp["valid_len"], global_idx=dinp["global_idx"],
                          side_k=dinp.get("side_k"), side_v=dinp.get("side_v"), bias=dinp.get("bias"),
                          local_bias=dinp.get("local_bias"), rand_blocks=dinp.get("rand_blocks"))
    torch.cuda.synchronize()
    assert plan.check() == 0
    ref = helpers.oracle_problem(w, inp).backward(dout)
    return [x.cpu().numpy() for x in grads], ref


@pytest.mark.parametrize("name,w", FULL_CASES, ids=[c[0] for c in FULL_CASES])
def test_full_pattern_backward_matches_oracle(name, w):
    _need_gpu()
    got, ref = run_full_backward(w)
    assert len(got) == len(ref)
    compare_grads(got[:3], ref[:3], name)
    if len(ref) == 5:
        compare_side_grads(got[3:], ref[3:], name)


def compare_side_grads(got, ref, what):
    for name, a, b in zip(("dside_k", "dside_v"), got, ref):
        assert np.all(np.isfinite(a)), f"{what} {name}: non-finite"
        err = np.abs(a.astype(np.float64) - b)
        scale_max = max(float(np.abs(b).max()), 1e-3)
        scale_mean = max(float(np.abs(b).mean()), 1e-3)
        print(f"{what} {name}: max err {err.max():.2e} (scale {scale_max:.2e})")
        assert err.max() <= REL_MAX * scale_max and err.mean() <= REL_MEAN * scale_mean, what + " " + name


def test_backward_unsupported_cases():
    _need_gpu()
    from sliding_window_global_b200 import SwaError
    # side keys in the plan but not passed to the backward
    w = workloads.SMALL["longt5_tglobal"]
    inp = helpers.to_dev(helpers.host_problem(w))
    out, lse, plan = helpers.run_gpu(w, inp)
    with pytest.raises(SwaError) as e:
        plan.backward(inp["q"], inp["k"], inp["v"], out, lse, out, window=inp["window"])
    assert e.value.status == 1
    # query heads of one KV head with different windows
    w = _small("swan_swa", window=(100, 50, 100, 100, 100, 100, 100, 100))
    inp = helpers.to_dev(helpers.host_problem(w))
    out, lse, plan = helpers.run_gpu(w, inp)
    with pytest.raises(SwaError) as e:
        plan.backward(inp["q"], inp["k"], inp["v"], out, lse, out, window=inp["window"], causal=True)
    assert e.value.status == 2
