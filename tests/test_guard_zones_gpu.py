"""Out-of-bounds and missing writes of the forward and backward, caught without a sanitizer.

The forward writes into caller buffers that sit inside larger allocations: a guard
zone of canary values before and after ``out`` and ``lse``, and ``out`` / ``lse``
themselves filled with NaN before the call.  After the call the canaries must be
untouched (no write past either end), no element of ``out`` or ``lse`` may still be
NaN (every row, padded ones included, was written), and the result must equal a
forward into fresh buffers bit for bit.  Every workload kind runs this: band with
global tokens and padding, dilation, side keys with bias, the causal GQA window,
the local bias, random blocks, and the fp32 path.
"""
import numpy as np
import pytest
import torch

from sliding_window_global_b200 import workloads
from tests import helpers

pytestmark = pytest.mark.gpu

GUARD = 4096                     # elements of canary on each side


def _guarded(shape, dtype, canary):
    """A NaN-filled tensor of `shape` inside a buffer with canary zones on both sides."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), canary, dtype=dtype, device="cuda")
    buf[GUARD:GUARD + n] = float("nan")
    return buf, buf[GUARD:GUARD + n].view(shape)


@pytest.mark.parametrize("name", list(workloads.SMALL))
def test_forward_writes_exactly_its_outputs(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = workloads.SMALL[name]
    inp = workloads.make_inputs(w)
    dinp = helpers.to_dev(inp)
    ref_out, ref_lse, plan = helpers.run_gpu(w, dinp)

    canary_out = 12345.0 if w.torch_dtype == torch.float32 else 1280.0    # exact in bf16
    obuf, out = _guarded(ref_out.shape, ref_out.dtype, canary_out)
    lbuf, lse = _guarded(ref_lse.shape, torch.float32, -4321.0)
    plan.forward(dinp["q"], dinp["k"], dinp["v"], window=dinp["window"], dilation=dinp["dilation"],
                 causal=dinp["causal"], global_idx=dinp["global_idx"], side_k=dinp.get("side_k"),
                 side_v=dinp.get("side_v"), bias=dinp.get("bias"), valid_len=dinp["valid_len"],
                 local_bias=dinp.get("local_bias"), rand_blocks=dinp.get("rand_blocks"), out=out, lse=lse)
    torch.cuda.synchronize()
    assert plan.check() == 0

    for buf, canary, what in ((obuf, canary_out, "out"), (lbuf, -4321.0, "lse")):
        head, tail = buf[:GUARD], buf[-GUARD:]
        assert torch.all(head == canary), f"{name}: write before {what}"
        assert torch.all(tail == canary), f"{name}: write after {what}"
    assert not torch.isnan(out).any(), f"{name}: rows of out left unwritten"
    assert not torch.isnan(lse).any(), f"{name}: rows of lse left unwritten"
    assert torch.equal(out, ref_out), f"{name}: out differs from a forward into fresh buffers"
    assert torch.equal(lse, ref_lse), f"{name}: lse differs from a forward into fresh buffers"


GRAD_CASES = ["swan_swa", "longformer_base", "dilated", "longt5_tglobal", "longt5_local", "bigbird_itc"]


@pytest.mark.parametrize("name", GRAD_CASES)
def test_backward_writes_exactly_its_gradients(name):
    """The same for dq, dk, dv (and dside_k, dside_v): canaries intact, no NaN left
    (padded rows and keys get zeros), equal to a backward into fresh buffers."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = workloads.SMALL[name]
    inp = helpers.host_problem(w)
    dinp = helpers.to_dev(inp)
    out, lse, plan = helpers.run_gpu(w, dinp)
    g = torch.Generator("cpu").manual_seed(91)
    dout = torch.randn(out.shape, generator=g).to(torch.bfloat16).cuda()
    kw = dict(window=dinp["window"], dilation=dinp["dilation"], causal=dinp["causal"],
              valid_len=dinp["valid_len"], global_idx=dinp["global_idx"], side_k=dinp.get("side_k"),
              side_v=dinp.get("side_v"), bias=dinp.get("bias"), local_bias=dinp.get("local_bias"),
              rand_blocks=dinp.get("rand_blocks"))
    ref = plan.backward(dinp["q"], dinp["k"], dinp["v"], out, lse, dout, **kw)
    torch.cuda.synchronize()
    assert plan.check() == 0
    bufs = [_guarded(r.shape, torch.float32, 7777.0) for r in ref[:3]]
    got = plan.backward(dinp["q"], dinp["k"], dinp["v"], out, lse, dout, dq=bufs[0][1], dk=bufs[1][1],
                        dv=bufs[2][1], **kw)
    torch.cuda.synchronize()
    assert plan.check() == 0
    for (buf, view), r, what in zip(bufs, ref[:3], ("dq", "dk", "dv")):
        assert torch.all(buf[:GUARD] == 7777.0), f"{name}: write before {what}"
        assert torch.all(buf[-GUARD:] == 7777.0), f"{name}: write after {what}"
        assert not torch.isnan(view).any(), f"{name}: rows of {what} left unwritten"
        assert torch.equal(view, r), f"{name}: {what} differs from a backward into fresh buffers"
    for a, r in zip(got[3:], ref[3:]):
        assert not torch.isnan(a).any() and torch.equal(a, r), f"{name}: side-key gradients differ"
