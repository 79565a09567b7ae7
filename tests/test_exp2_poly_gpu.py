"""Direct pin of the FMA-pipe exponential of the band kernel's softmax.

Part of the exponentials of the softmax (p = 2^(s - m), scores in log2 units) are
evaluated with a degree-3 polynomial on the FMA pipe instead of the MUFU unit.
Inside the attention parity tests a few times its stated error would still pass the
bf16 tolerance, so this test holds the device function itself to its bound on a
dense grid, against 2^x in fp64 and against CUDA's exp2f."""
import numpy as np
import pytest
import torch

from sliding_window_global_b200.swa import selftest_exp2_poly

pytestmark = pytest.mark.gpu

REL_BOUND = 1.02e-4          # stated in softmax_math.cuh and include/swa.h


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_exp2_poly_relative_error_bound_on_a_dense_grid():
    _need_gpu()
    # every float32 step is too many; 2^22 points over [-125.5, 8] plus the
    # neighbourhood of each integer (where the rounding to i switches)
    grid = np.linspace(-125.5, 8.0, 1 << 22, dtype=np.float64)
    ints = np.arange(-125, 9, dtype=np.float64)
    near = (ints[:, None] + np.array([-0.5, -0.5 + 1e-6, -1e-6, 0.0, 1e-6, 0.5 - 1e-6])[None, :]).ravel()
    x = np.concatenate([grid, near[(near >= -125.5) & (near <= 8.0)]]).astype(np.float32)
    y = selftest_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= REL_BOUND, (rel.max(), x[rel.argmax()])
    # and against CUDA's own exp2f on the device
    cu = torch.exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    assert np.abs(y / cu - 1.0).max() <= REL_BOUND + 2e-7


def test_exp2_poly_underflow_and_masked_scores():
    _need_gpu()
    x = np.array([-np.inf, -1e30, -1000.0, -128.0, -127.0], dtype=np.float32)
    y = selftest_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.all(y == 0.0) and not np.any(np.signbit(y))      # exactly +0
    tail = np.linspace(-127.0, -125.5, 4097, dtype=np.float32)
    yt = selftest_exp2_poly(torch.from_numpy(tail).cuda()).cpu().numpy()
    assert np.all(np.isfinite(yt)) and np.all(yt >= 0.0) and np.all(yt <= 2.0 ** -125)


def test_exp2_poly_exact_at_zero_and_odd_length():
    _need_gpu()
    x = np.array([0.0, 1.0, 7.0, -3.0, 2.5], dtype=np.float32)   # odd length: one pair is partial
    y = selftest_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy()
    assert y[0] == 1.0                                            # c0 = 1 exactly
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) <= REL_BOUND)
