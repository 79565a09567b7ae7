"""ctypes binding of libswa.so (the C ABI declared in include/swa.h).

Argument marshalling only: every step of the attention runs in the library's
CUDA kernels.  There is no fallback -- if the library cannot be loaded, or a
tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libswa.so")
_lock = threading.Lock()
_lib = None

STATUS = {
    0: "SWA_OK", 1: "SWA_ERR_INVALID_ARG", 2: "SWA_ERR_UNSUPPORTED", 3: "SWA_ERR_CUDA",
    4: "SWA_ERR_OOM", 5: "SWA_ERR_TIMEOUT", 6: "SWA_ERR_DEVICE_CHECK",
}
SWA_BF16, SWA_FP32 = 0, 1
SWA_DEBUG_CHECKS = 1

# Every symbol include/swa.h declares.
EXPORTS = (
    "swa_plan_create", "swa_forward", "swa_plan_check", "swa_plan_destroy",
    "swa_plan_workspace_bytes", "swa_plan_last_launches", "swa_status_string",
    "swa_side_aggregate", "swa_relative_bucket", "swa_expand_side_bias", "swa_forward_noalloc",
    "swa_forward_ex", "swa_bucket_local_bias", "swa_backward", "swa_selftest_wait_timeout",
    "swa_selftest_exp2_poly",
)


class SwaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class PlanDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("seq_len", ctypes.c_int), ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int),
        ("max_global", ctypes.c_int), ("num_side", ctypes.c_int), ("side_block", ctypes.c_int),
        ("scale", ctypes.c_float), ("flags", ctypes.c_uint),
    ]


class ForwardArgs(ctypes.Structure):
    """swa_forward_args of include/swa.h."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("global_idx", ctypes.c_void_p), ("num_global", ctypes.c_int),
        ("side_k", ctypes.c_void_p), ("side_v", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("window", ctypes.c_void_p), ("dilation", ctypes.c_void_p), ("causal", ctypes.c_int),
        ("valid_len", ctypes.c_void_p), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("local_bias", ctypes.c_void_p), ("local_radius", ctypes.c_int),
        ("rand_blocks", ctypes.c_void_p), ("num_rand", ctypes.c_int),
        ("side_from_kv", ctypes.c_int),
    ]


class BackwardArgs(ctypes.Structure):
    """swa_backward_args of include/swa.h."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("window", ctypes.c_void_p), ("dilation", ctypes.c_void_p), ("causal", ctypes.c_int),
        ("valid_len", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
        ("dv", ctypes.c_void_p),
        ("global_idx", ctypes.c_void_p), ("num_global", ctypes.c_int),
        ("side_k", ctypes.c_void_p), ("side_v", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("local_bias", ctypes.c_void_p), ("local_radius", ctypes.c_int),
        ("rand_blocks", ctypes.c_void_p), ("num_rand", ctypes.c_int),
        ("dside_k", ctypes.c_void_p), ("dside_v", ctypes.c_void_p),
    ]


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libswa.so from the package directory (raise if it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libswa.so not built at {_LIB_PATH}; run __graft_entry__.build()")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.swa_plan_create.argtypes = [ctypes.POINTER(P), ctypes.POINTER(PlanDesc)]
        lib.swa_plan_create.restype = I
        lib.swa_forward.argtypes = [P, P, P, P, P, I, P, P, P, P, P, I, P, P, P, P]
        lib.swa_forward.restype = I
        lib.swa_plan_check.argtypes = [P, P]
        lib.swa_plan_check.restype = I
        lib.swa_plan_destroy.argtypes = [P]
        lib.swa_plan_destroy.restype = I
        lib.swa_plan_workspace_bytes.argtypes = [P]
        lib.swa_plan_workspace_bytes.restype = U64
        lib.swa_plan_last_launches.argtypes = [P]
        lib.swa_plan_last_launches.restype = I
        lib.swa_status_string.argtypes = [I]
        lib.swa_status_string.restype = ctypes.c_char_p
        lib.swa_side_aggregate.argtypes = [P, P, I, I, I, I, I, P, I, P]
        lib.swa_side_aggregate.restype = I
        lib.swa_relative_bucket.argtypes = [I]
        lib.swa_relative_bucket.restype = I
        lib.swa_expand_side_bias.argtypes = [I, I, I, P, P]
        lib.swa_expand_side_bias.restype = I
        lib.swa_forward_noalloc.argtypes = [ctypes.POINTER(PlanDesc), P, P, P, P, I, P, P, P, P, P, I,
                                            P, P, P, P]
        lib.swa_forward_noalloc.restype = I
        lib.swa_forward_ex.argtypes = [P, ctypes.POINTER(ForwardArgs), P]
        lib.swa_forward_ex.restype = I
        lib.swa_bucket_local_bias.argtypes = [I, I, P, P]
        lib.swa_bucket_local_bias.restype = I
        lib.swa_backward.argtypes = [P, ctypes.POINTER(BackwardArgs), P]
        lib.swa_backward.restype = I
        lib.swa_selftest_wait_timeout.argtypes = [P, ctypes.c_uint64, P]
        lib.swa_selftest_wait_timeout.restype = I
        lib.swa_selftest_exp2_poly.argtypes = [P, P, I, P]
        lib.swa_selftest_exp2_poly.restype = I
        _lib = lib
        return lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return SWA_BF16
    if t == torch.float32:
        return SWA_FP32
    raise TypeError(f"unsupported dtype {t}; use bfloat16 or float32")


def _dev_ptr(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _host_i32(x, H: int, name: str):
    if x is None:
        return None, None
    if isinstance(x, int):
        vals = [x] * H
    elif isinstance(x, torch.Tensor):
        vals = [int(v) for v in x.detach().cpu().reshape(-1).tolist()]
    else:
        vals = [int(v) for v in x]
    if len(vals) == 1:
        vals = vals * H
    if len(vals) != H:
        raise ValueError(f"{name} needs {H} per-head values, got {len(vals)}")
    arr = (ctypes.c_int32 * H)(*vals)
    return arr, vals


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Plan:
    """One problem shape: owns the device workspace of a libswa plan."""

    def __init__(self, batch: int, seq_len: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, dtype: torch.dtype = torch.bfloat16, *, max_global: int = 0,
                 num_side: int = 0, side_block: int = 16, scale: float = 0.0, debug: bool = False):
        self._lib = load_library()
        self.desc = PlanDesc(batch, seq_len, num_q_heads, num_kv_heads, head_dim, _dtype_code(dtype),
                             max_global, num_side, side_block if num_side else 0, float(scale),
                             SWA_DEBUG_CHECKS if debug else 0)
        self.dtype = dtype
        h = ctypes.c_void_p()
        st = self._lib.swa_plan_create(ctypes.byref(h), ctypes.byref(self.desc))
        if st != 0:
            raise SwaError(st, "swa_plan_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    @property
    def workspace_bytes(self) -> int:
        return int(self._lib.swa_plan_workspace_bytes(self._h))

    @property
    def last_launches(self) -> int:
        return int(self._lib.swa_plan_last_launches(self._h))

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, window,
                dilation=None, causal: bool = False, global_idx: Optional[torch.Tensor] = None,
                side_k: Optional[torch.Tensor] = None, side_v: Optional[torch.Tensor] = None,
                bias: Optional[torch.Tensor] = None, valid_len: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                return_lse: bool = True, local_bias: Optional[torch.Tensor] = None,
                rand_blocks: Optional[torch.Tensor] = None, side_from_kv: bool = False,
                stream=None):
        """``local_bias``: optional [Hq, 2R+1] fp32 device table of the LongT5 local
        relative-position bias (window keys of non-global rows, column (j - i) + R).
        ``rand_blocks``: optional int32 device tensor [B, Hq, ceil(n/128), r] of
        BigBird random key blocks (128 keys each) per query block.
        ``side_from_kv``: build the Transient-Global side keys / values from k and v
        on the device (block means of ``side_block`` tokens) instead of taking them."""
        d = self.desc
        H = d.num_q_heads
        if out is None:
            out = torch.empty((d.batch, H, d.seq_len, d.head_dim), dtype=self.dtype, device=q.device)
        if lse is None and return_lse:
            lse = torch.empty((d.batch, H, d.seq_len), dtype=torch.float32, device=q.device)
        w_arr, _ = _host_i32(window, H, "window")
        d_arr, _ = _host_i32(dilation, H, "dilation")
        g = 0 if global_idx is None else int(global_idx.shape[-1])
        if local_bias is not None or rand_blocks is not None or side_from_kv:
            width = 1 if local_bias is None else int(local_bias.shape[-1])
            if local_bias is not None and (local_bias.dim() != 2 or local_bias.shape[0] != H
                                           or width % 2 == 0):
                raise ValueError("local_bias must be [Hq, 2R+1]")
            nrand = 0
            if rand_blocks is not None:
                nqb = (d.seq_len + 127) // 128
                if rand_blocks.dim() != 4 or tuple(rand_blocks.shape[:3]) != (d.batch, H, nqb):
                    raise ValueError("rand_blocks must be [B, Hq, ceil(n/128), r]")
                nrand = int(rand_blocks.shape[-1])
            a = ForwardArgs(
                _dev_ptr(q, "q", self.dtype), _dev_ptr(k, "k", self.dtype), _dev_ptr(v, "v", self.dtype),
                _dev_ptr(global_idx, "global_idx", torch.int32), g,
                _dev_ptr(side_k, "side_k", self.dtype), _dev_ptr(side_v, "side_v", self.dtype),
                _dev_ptr(bias, "bias", torch.float32), ctypes.cast(w_arr, ctypes.c_void_p),
                None if d_arr is None else ctypes.cast(d_arr, ctypes.c_void_p), int(bool(causal)),
                _dev_ptr(valid_len, "valid_len", torch.int32), _dev_ptr(out, "out", self.dtype),
                _dev_ptr(lse, "lse", torch.float32), _dev_ptr(local_bias, "local_bias", torch.float32),
                (width - 1) // 2, _dev_ptr(rand_blocks, "rand_blocks", torch.int32), nrand,
                int(bool(side_from_kv)))
            st = self._lib.swa_forward_ex(self._h, ctypes.byref(a), _stream_handle(stream))
            if st != 0:
                raise SwaError(st, "swa_forward_ex")
            return out, lse
        st = self._lib.swa_forward(
            self._h, _dev_ptr(q, "q", self.dtype), _dev_ptr(k, "k", self.dtype),
            _dev_ptr(v, "v", self.dtype), _dev_ptr(global_idx, "global_idx", torch.int32), g,
            _dev_ptr(side_k, "side_k", self.dtype), _dev_ptr(side_v, "side_v", self.dtype),
            _dev_ptr(bias, "bias", torch.float32), w_arr, d_arr, int(bool(causal)),
            _dev_ptr(valid_len, "valid_len", torch.int32), _dev_ptr(out, "out", self.dtype),
            _dev_ptr(lse, "lse", torch.float32), _stream_handle(stream))
        if st != 0:
            raise SwaError(st, "swa_forward")
        return out, lse

    def backward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                 lse: torch.Tensor, dout: torch.Tensor, *, window, dilation=None,
                 causal: bool = False, valid_len: Optional[torch.Tensor] = None,
                 dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                 dv: Optional[torch.Tensor] = None, global_idx: Optional[torch.Tensor] = None,
                 side_k: Optional[torch.Tensor] = None, side_v: Optional[torch.Tensor] = None,
                 bias: Optional[torch.Tensor] = None, local_bias: Optional[torch.Tensor] = None,
                 rand_blocks: Optional[torch.Tensor] = None, stream=None):
        """Gradients, fp32, for the upstream gradient ``dout``; ``out`` and ``lse`` are the
        forward's results, and the optional terms those the forward ran with.  Returns
        (dq, dk, dv), plus (dside_k, dside_v) when the plan has side keys."""
        d = self.desc
        H, Hkv = d.num_q_heads, d.num_kv_heads
        shape_q = (d.batch, H, d.seq_len, d.head_dim)
        shape_k = (d.batch, Hkv, d.seq_len, d.head_dim)
        if dq is None:
            dq = torch.empty(shape_q, dtype=torch.float32, device=q.device)
        if dk is None:
            dk = torch.empty(shape_k, dtype=torch.float32, device=q.device)
        if dv is None:
            dv = torch.empty(shape_k, dtype=torch.float32, device=q.device)
        w_arr, _ = _host_i32(window, H, "window")
        d_arr, _ = _host_i32(dilation, H, "dilation")
        dsk = dsv = None
        if d.num_side > 0:
            shape_s = (d.batch, Hkv, d.num_side, d.head_dim)
            dsk = torch.empty(shape_s, dtype=torch.float32, device=q.device)
            dsv = torch.empty(shape_s, dtype=torch.float32, device=q.device)
        g = 0 if global_idx is None else int(global_idx.shape[-1])
        width = 1 if local_bias is None else int(local_bias.shape[-1])
        nrand = 0 if rand_blocks is None else int(rand_blocks.shape[-1])
        a = BackwardArgs(
            _dev_ptr(q, "q", self.dtype), _dev_ptr(k, "k", self.dtype), _dev_ptr(v, "v", self.dtype),
            _dev_ptr(out, "out", self.dtype), _dev_ptr(lse, "lse", torch.float32),
            _dev_ptr(dout, "dout", self.dtype), ctypes.cast(w_arr, ctypes.c_void_p),
            None if d_arr is None else ctypes.cast(d_arr, ctypes.c_void_p), int(bool(causal)),
            _dev_ptr(valid_len, "valid_len", torch.int32), _dev_ptr(dq, "dq", torch.float32),
            _dev_ptr(dk, "dk", torch.float32), _dev_ptr(dv, "dv", torch.float32),
            _dev_ptr(global_idx, "global_idx", torch.int32), g,
            _dev_ptr(side_k, "side_k", self.dtype), _dev_ptr(side_v, "side_v", self.dtype),
            _dev_ptr(bias, "bias", torch.float32), _dev_ptr(local_bias, "local_bias", torch.float32),
            (width - 1) // 2, _dev_ptr(rand_blocks, "rand_blocks", torch.int32), nrand,
            _dev_ptr(dsk, "dside_k", torch.float32), _dev_ptr(dsv, "dside_v", torch.float32))
        st = self._lib.swa_backward(self._h, ctypes.byref(a), _stream_handle(stream))
        if st != 0:
            raise SwaError(st, "swa_backward")
        if dsk is not None:
            return dq, dk, dv, dsk, dsv
        return dq, dk, dv

    def selftest_wait_timeout(self, limit_ns: int, stream=None) -> None:
        """Enqueue the failure-path self test: a bounded wait that expires after
        ``limit_ns`` and sets the timeout bit that ``check()`` then reports."""
        st = self._lib.swa_selftest_wait_timeout(self._h, int(limit_ns), _stream_handle(stream))
        if st != 0:
            raise SwaError(st, "swa_selftest_wait_timeout")

    def check(self, stream=None) -> int:
        """Synchronise and return the status of the device error word (0 = OK)."""
        return int(self._lib.swa_plan_check(self._h, _stream_handle(stream)))

    def close(self):
        if getattr(self, "_h", None):
            self._lib.swa_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_plans = {}


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, window, dilation=None,
            causal: bool = False, global_idx=None, side_k=None, side_v=None, bias=None,
            valid_len=None, side_block: int = 16, scale: float = 0.0, return_lse: bool = True,
            local_bias=None, rand_blocks=None):
    """Banded sparse attention of q [B,Hq,n,D] over k/v [B,Hkv,n,D] (CUDA tensors).

    Returns ``(out, lse)``: out like q, lse fp32 [B,Hq,n] (natural log).  Plans are
    cached by problem shape."""
    B, Hq, n, D = q.shape
    Hkv = k.shape[1]
    S = 0 if side_k is None else int(side_k.shape[2])
    g = 0 if global_idx is None else int(global_idx.shape[-1])
    key = (q.device.index, B, n, Hq, Hkv, D, q.dtype, g, S, side_block if S else 0, float(scale))
    plan = _plans.get(key)
    if plan is None:
        plan = Plan(B, n, Hq, Hkv, D, q.dtype, max_global=g, num_side=S, side_block=side_block,
                    scale=scale)
        _plans[key] = plan
    return plan.forward(q, k, v, window=window, dilation=dilation, causal=causal,
                        global_idx=global_idx, side_k=side_k, side_v=side_v, bias=bias,
                        valid_len=valid_len, return_lse=return_lse, local_bias=local_bias,
                        rand_blocks=rand_blocks)


def side_aggregate(x: torch.Tensor, block: int, valid_len: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Transient-Global block means [B,H,n,D] -> [B,H,n//block,D] on the device."""
    lib = load_library()
    B, H, n, D = x.shape
    out = torch.empty((B, H, n // block, D), dtype=x.dtype, device=x.device)
    st = lib.swa_side_aggregate(_dev_ptr(x, "x"), _dev_ptr(out, "out"), B, H, n, D, block,
                                _dev_ptr(valid_len, "valid_len", torch.int32), _dtype_code(x.dtype),
                                _stream_handle(stream))
    if st != 0:
        raise SwaError(st, "swa_side_aggregate")
    return out


def selftest_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The band kernel's FMA-pipe 2^x evaluated on a CUDA fp32 tensor (a self test)."""
    lib = load_library()
    x = x.contiguous()
    y = torch.empty_like(x)
    st = lib.swa_selftest_exp2_poly(_dev_ptr(x, "x", torch.float32), _dev_ptr(y, "y", torch.float32),
                                    int(x.numel()), _stream_handle(stream))
    if st != 0:
        raise SwaError(st, "swa_selftest_exp2_poly")
    return y


def relative_bucket(delta: int) -> int:
    return int(load_library().swa_relative_bucket(int(delta)))


def expand_side_bias(table: torch.Tensor, num_side: int, nblk: int) -> torch.Tensor:
    """[Hq,32] fp32 bucket table (host) -> [Hq, num_side + nblk - 1] fp32 (host)."""
    lib = load_library()
    t = table.detach().to("cpu", torch.float32).contiguous()
    Hq = t.shape[0]
    out = torch.empty((Hq, num_side + nblk - 1), dtype=torch.float32)
    st = lib.swa_expand_side_bias(Hq, num_side, nblk, ctypes.c_void_p(t.data_ptr()),
                                  ctypes.c_void_p(out.data_ptr()))
    if st != 0:
        raise SwaError(st, "swa_expand_side_bias")
    return out


def bucket_local_bias(table: torch.Tensor, radius: int) -> torch.Tensor:
    """[Hq,32] fp32 bucket table (host) -> [Hq, 2*radius + 1] local-bias table (host),
    column c holding the bucket of the offset c - radius."""
    lib = load_library()
    t = table.detach().to("cpu", torch.float32).contiguous()
    Hq = t.shape[0]
    out = torch.empty((Hq, 2 * radius + 1), dtype=torch.float32)
    st = lib.swa_bucket_local_bias(Hq, int(radius), ctypes.c_void_p(t.data_ptr()),
                                   ctypes.c_void_p(out.data_ptr()))
    if st != 0:
        raise SwaError(st, "swa_bucket_local_bias")
    return out
