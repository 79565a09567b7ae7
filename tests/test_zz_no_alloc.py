"""GPU test of swa_forward_noalloc, the allocation-free entry point.

Some callers cannot allocate memory when they run the attention: code under a
fixed memory budget or inside a framework that owns all device memory,
real-time loops where an allocation (and the synchronisation a device
allocation can bring) is not allowed, and plug-ins that cannot keep a plan
object alive between calls.  swa_forward_noalloc serves them: it takes the plan
descriptor directly and keeps its scratch in a static device array.

This test calls it through the C ABI (ctypes, no Python wrapper) and checks its
output against the plan-based swa_forward on the same inputs, with the parity
tolerance of the bf16 tests, on two calls in a row with different inputs (so
stale scratch from the first call would show in the second).  It lives in a file
of its own that pytest collects last, and needs nothing set up by other tests.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from sliding_window_global_b200 import Plan, load_library, workloads
from sliding_window_global_b200.swa import PlanDesc
from tests import helpers

pytestmark = pytest.mark.gpu

SWA_OK, SWA_ERR_UNSUPPORTED, SWA_ERR_DEVICE_CHECK = 0, 2, 6
SWA_DEBUG_CHECKS = 1


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(w, dinp, out, lse, max_global, flags=0):
    lib = load_library()
    S = 0 if dinp.get("side_k") is None else int(dinp["side_k"].shape[2])
    desc = PlanDesc(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim,
                    0 if w.dtype == "bf16" else 1, max_global, S, w.side_block if S else 0, 0.0, flags)
    H = w.q_heads
    win = (ctypes.c_int32 * H)(*[int(x) for x in dinp["window"].tolist()])
    dil = (ctypes.c_int32 * H)(*[int(x) for x in dinp["dilation"].tolist()])
    g = 0 if dinp["global_idx"] is None else int(dinp["global_idx"].shape[-1])
    st = lib.swa_forward_noalloc(ctypes.byref(desc), _ptr(dinp["q"]), _ptr(dinp["k"]), _ptr(dinp["v"]),
                                 _ptr(dinp["global_idx"]), g, _ptr(dinp.get("side_k")),
                                 _ptr(dinp.get("side_v")), _ptr(dinp.get("bias")), win, dil,
                                 int(bool(dinp["causal"])), _ptr(dinp["valid_len"]), _ptr(out), _ptr(lse),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _compare(w, a_out, a_lse, b_out, b_lse):
    tol = helpers.TOL[w.dtype]
    lb, la = b_lse.cpu().numpy(), a_lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lb), np.isneginf(la))
    valid = ~np.isneginf(lb)
    d = np.abs(a_out.float().cpu().numpy()[valid] - b_out.float().cpu().numpy()[valid])
    assert d.max() <= tol["max_abs"] and d.mean() <= tol["mean_abs"]
    assert np.abs(la[valid] - lb[valid]).max() <= tol["lse"]
    assert torch.equal(a_out[~torch.from_numpy(valid)], b_out[~torch.from_numpy(valid)])


CASES = [
    # global tokens and padding: the gathered rows and split partials live in the scratch
    ("globals", workloads.SMALL["longformer_base"], 3001),
    ("dilated_globals", workloads.SMALL["dilated"], 3002),
    ("gqa_causal", workloads.SMALL["swan_swa"], 3003),
    ("fp32", workloads.SMALL["longformer_tiny"], 3004),
    # global tokens together with side keys and their bias: one more split (the side
    # keys') in the scratch layout
    ("globals_side_bias", dataclasses.replace(workloads.SMALL["longt5_tglobal"], name="tglobal_globals",
                                              num_global=12, global_mode="leading"), 3005),
    # 1000 global slots at D=128: the full set of global-row splits would exceed the
    # scratch array, so the entry point uses fewer splits than the plan-based path
    ("globals_near_limit", dataclasses.replace(workloads.SMALL["longformer_base"], name="many_globals",
                                               q_heads=2, kv_heads=2, head_dim=128, seq_len=2048,
                                               num_global=1000, window=(64, 64), dilation=(1, 1),
                                               padding=0), 3006),
]


@pytest.mark.parametrize("name,w,seed2", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_plan_forward_twice(name, w, seed2):
    _need_gpu()
    for seed in (w.seed, seed2):                       # two calls in a row, different inputs
        inp = helpers.host_problem(w, workloads.make_inputs(w, seed=seed))
        dinp = helpers.to_dev(inp)
        ref_out, ref_lse, _ = helpers.run_gpu(w, dinp)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _noalloc(w, dinp, out, lse, max_global=w.num_global)
        torch.cuda.synchronize()
        assert st == SWA_OK
        _compare(w, out, lse, ref_out, ref_lse)


def test_noalloc_rejects_problems_beyond_the_scratch_limit():
    _need_gpu()
    # 4 x 32 heads x 1024 global slots x D=128: the gathered rows alone exceed 16 MiB
    w = dataclasses.replace(workloads.SMALL["longformer_base"], batch=4, q_heads=32, kv_heads=32,
                            head_dim=128, seq_len=2048, num_global=1024, window=(8,) * 32,
                            dilation=(1,) * 32, padding=0)
    inp = workloads.make_inputs(w)
    dinp = helpers.to_dev(inp)
    out = torch.zeros((w.batch, w.q_heads, w.seq_len, w.head_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.batch, w.q_heads, w.seq_len), dtype=torch.float32, device="cuda")
    assert _noalloc(w, dinp, out, lse, max_global=w.num_global) == SWA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 0).all())                     # nothing was launched


def test_noalloc_debug_mode_reports_device_checks():
    """With SWA_DEBUG_CHECKS the allocation-free entry point synchronises and returns
    what the device error word says: a global index list that breaks its
    precondition (not increasing, beyond the sequence, negative) gives
    SWA_ERR_DEVICE_CHECK before any kernel that indexes with it runs, so out stays
    untouched; the next call with a valid list returns SWA_OK (the word was cleared)
    and matches the plan-based forward."""
    _need_gpu()
    w = workloads.SMALL["longformer_base"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    n = w.seq_len
    out = torch.full((w.batch, w.q_heads, n, w.head_dim), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.batch, w.q_heads, n), dtype=torch.float32, device="cuda")
    for bad in ([3, 2, 5, 9], [2, 3, 5, n + 40], [-1, 3, 5, 9]):
        d = dict(dinp, global_idx=torch.tensor([bad], dtype=torch.int32, device="cuda"))
        st = _noalloc(w, d, out, lse, max_global=4, flags=SWA_DEBUG_CHECKS)
        torch.cuda.synchronize()
        assert st == SWA_ERR_DEVICE_CHECK, bad
        assert bool((out == 7.0).all()), bad
    good = torch.tensor([[2, 3, 5, 9]], dtype=torch.int32, device="cuda")
    d = dict(dinp, global_idx=good)
    assert _noalloc(w, d, out, lse, max_global=4, flags=SWA_DEBUG_CHECKS) == SWA_OK
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = helpers.run_gpu(w, d)
    _compare(w, out, lse, ref_out, ref_lse)
