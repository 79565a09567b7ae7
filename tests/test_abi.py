"""C-ABI checks that need no GPU: the library loads and exports every function
include/swa.h declares; host-side validation returns statuses; the host helpers
(relative bucket, side-bias expansion) agree exactly with the oracle's own."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from sliding_window_global_b200 import swa as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sliding_window_global_b200 import build
    build.build()
    return binding.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(swa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert len(declared) >= 10
    assert sorted(binding.EXPORTS) == declared
    for name in declared:
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert lib.swa_status_string(code).decode() == name
    assert lib.swa_status_string(99).decode() == "SWA_ERR_UNKNOWN"


def _desc(**kw):
    base = dict(batch=1, seq_len=256, num_q_heads=4, num_kv_heads=2, head_dim=64, dtype=0,
                max_global=0, num_side=0, side_block=0, scale=0.0, flags=0)
    base.update(kw)
    return binding.PlanDesc(**base)


@pytest.mark.parametrize("bad", [dict(batch=0), dict(seq_len=0), dict(num_q_heads=3),
                                 dict(num_kv_heads=0), dict(dtype=7), dict(max_global=-1),
                                 dict(max_global=300), dict(num_side=4, side_block=0),
                                 dict(scale=-1.0), dict(flags=8), dict(head_dim=0)])
def test_plan_create_rejects_bad_descriptors(lib, bad):
    h = ctypes.c_void_p()
    d = _desc(**bad)
    assert lib.swa_plan_create(ctypes.byref(h), ctypes.byref(d)) == 1
    assert not h.value


_BAD_DESCRIPTORS = [
    (dict(batch=0), 1), (dict(seq_len=0), 1), (dict(num_q_heads=3), 1), (dict(num_kv_heads=0), 1),
    (dict(dtype=7), 1), (dict(max_global=-1), 1), (dict(max_global=300), 1),
    (dict(num_side=4, side_block=0), 1), (dict(scale=-1.0), 1), (dict(flags=8), 1),
    (dict(head_dim=0), 1), (dict(head_dim=96), 2), (dict(num_q_heads=256, num_kv_heads=1), 2),
    (dict(batch=2**31 - 1), 2),
]


@pytest.mark.parametrize("bad,status", _BAD_DESCRIPTORS)
def test_both_forward_entry_points_validate_descriptors_alike(lib, bad, status):
    """swa_plan_create and swa_forward_noalloc share one descriptor validator: the same
    bad descriptor gives the same status from both, before any device work."""
    h = ctypes.c_void_p()
    d = _desc(**bad)
    assert lib.swa_plan_create(ctypes.byref(h), ctypes.byref(d)) == status
    win = (ctypes.c_int32 * max(1, d.num_q_heads))()
    st = lib.swa_forward_noalloc(ctypes.byref(d), None, None, None, None, 0, None, None, None, win,
                                 None, 0, None, None, None, None)
    assert st == status


def test_plan_create_unsupported_head_dim(lib):
    h = ctypes.c_void_p()
    d = _desc(head_dim=96)
    assert lib.swa_plan_create(ctypes.byref(h), ctypes.byref(d)) == 2
    d = _desc(num_q_heads=256, num_kv_heads=1)
    assert lib.swa_plan_create(ctypes.byref(h), ctypes.byref(d)) == 2


def test_null_arguments(lib):
    d = _desc()
    assert lib.swa_plan_create(None, ctypes.byref(d)) == 1
    h = ctypes.c_void_p()
    assert lib.swa_plan_create(ctypes.byref(h), None) == 1
    assert lib.swa_forward(None, *([None] * 4), 0, None, None, None, None, None, 0, None, None,
                           None, None) == 1
    assert lib.swa_plan_destroy(None) == 0
    assert lib.swa_plan_check(None, None) == 1
    assert lib.swa_plan_workspace_bytes(None) == 0
    assert lib.swa_side_aggregate(None, None, 1, 1, 16, 64, 16, None, 0, None) == 1
    assert lib.swa_expand_side_bias(0, 1, 1, None, None) == 1


def test_relative_bucket_matches_oracle(lib):
    for delta in range(-3000, 3001):
        assert lib.swa_relative_bucket(delta) == oracle.relative_bucket(delta)


def test_expand_side_bias_matches_oracle(lib):
    gen = torch.Generator("cpu").manual_seed(4)
    table = torch.randn((12, 32), generator=gen)
    for S, nblk in [(1024, 1024), (100, 37), (5, 1), (1, 9)]:
        ours = binding.expand_side_bias(table, S, nblk).numpy()
        ref = oracle.expand_side_bias(table, S, nblk)
        assert np.array_equal(ours, ref)


def test_bucket_local_bias_matches_oracle(lib):
    gen = torch.Generator("cpu").manual_seed(6)
    table = torch.randn((12, 32), generator=gen)
    for R in (0, 1, 7, 127, 511, 2000):
        ours = binding.bucket_local_bias(table, R).numpy()
        ref = oracle.expand_local_bias(table, R)
        assert ours.shape == (12, 2 * R + 1)
        assert np.array_equal(ours, ref)
    assert lib.swa_bucket_local_bias(0, 1, None, None) == 1
    assert lib.swa_bucket_local_bias(1, -1, None, None) == 1


def test_forward_ex_null_arguments(lib):
    assert lib.swa_forward_ex(None, None, None) == 1
    args = binding.ForwardArgs()
    assert lib.swa_forward_ex(None, ctypes.byref(args), None) == 1


def test_backward_null_arguments(lib):
    assert lib.swa_backward(None, None, None) == 1
    args = binding.BackwardArgs()
    assert lib.swa_backward(None, ctypes.byref(args), None) == 1


def test_exp2_selftest_rejects_bad_arguments(lib):
    assert lib.swa_selftest_exp2_poly(None, None, -1, None) == 1
    assert lib.swa_selftest_exp2_poly(None, None, 4, None) == 1


def test_selftest_rejects_bad_limits(lib):
    assert lib.swa_selftest_wait_timeout(None, 1000, None) == 1
