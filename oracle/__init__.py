"""fp64 CPU oracle for banded sparse self-attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (the CUDA library and its Python binding) never imports, links or runs it,
and the two share no code: the oracle is plain C (``swa_oracle.c``) compiled
with gcc and OpenMP, reached through ctypes from here.

What it computes, and from which passage of the pages, is stated function by
function in ``swa_oracle.c``.  Every function is pinned by the ``-m "not gpu"``
tests in ``tests/test_oracle_pins.py`` (brute force, worked example, closed
cases, the bucket threshold table).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class _Extras(ctypes.Structure):
    """oracle_extras of swa_oracle.c."""
    _fields_ = [("local_bias", ctypes.c_void_p), ("local_radius", ctypes.c_int),
                ("rand_blocks", ctypes.c_void_p), ("num_rand", ctypes.c_int),
                ("rand_block", ctypes.c_int)]


def _extras(local_bias=None, local_radius=0, rand_blocks=None, rand_block=128):
    ex = _Extras()
    ex.local_bias = None if local_bias is None else local_bias.ctypes.data
    ex.local_radius = int(local_radius)
    if rand_blocks is not None and rand_blocks.shape[-1] > 0:
        ex.rand_blocks = rand_blocks.ctypes.data
        ex.num_rand = int(rand_blocks.shape[-1])
        ex.rand_block = int(rand_block)
    return ex


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_forward.argtypes = [I, I, I, I, I, P, P, P, P, I, P, P, I, I, P, P, P, I, P,
                                           D, P, I64, P, P, P]
            lib.oracle_forward.restype = I
            lib.oracle_dense_bruteforce.argtypes = [I, I, I, I, I, P, P, P, P, I, P, P, I, I, P, P,
                                                    P, I, P, D, P, P]
            lib.oracle_dense_bruteforce.restype = I
            EX = ctypes.POINTER(_Extras)
            lib.oracle_forward_ex.argtypes = lib.oracle_forward.argtypes + [EX]
            lib.oracle_forward_ex.restype = I
            lib.oracle_dense_bruteforce_ex.argtypes = lib.oracle_dense_bruteforce.argtypes + [EX]
            lib.oracle_dense_bruteforce_ex.restype = I
            lib.oracle_key_counts.argtypes = [I, I, I, P, I, I, P, P, I, P, P]
            lib.oracle_key_counts.restype = I
            lib.oracle_key_list.argtypes = [I, I, I, P, I, P, P, I, P, I, I, I, P]
            lib.oracle_key_list.restype = I
            lib.oracle_key_counts_ex.argtypes = lib.oracle_key_counts.argtypes + [EX]
            lib.oracle_key_counts_ex.restype = I
            lib.oracle_key_list_ex.argtypes = lib.oracle_key_list.argtypes + [EX]
            lib.oracle_key_list_ex.restype = I
            lib.oracle_relative_bucket.argtypes = [I]
            lib.oracle_relative_bucket.restype = I
            lib.oracle_expand_side_bias.argtypes = [I, I, I, P, P]
            lib.oracle_expand_side_bias.restype = I
            lib.oracle_side_aggregate.argtypes = [I, I, I, I, I, P, P, P]
            lib.oracle_side_aggregate.restype = I
            lib.oracle_backward.argtypes = [I, I, I, I, I, P, P, P, P, P, I, P, P, I, P, D, EX, P, P, P]
            lib.oracle_backward.restype = I
            lib.oracle_backward_ex.argtypes = [I, I, I, I, I, P, P, P, P, P, I, P, P, I, I, P, P, P, I,
                                               P, D, EX, P, P, P, P, P]
            lib.oracle_backward_ex.restype = I
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = I
            _lib = lib
    return _lib


def _f32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly (bf16/fp32 -> fp32)
        import torch
        x = x.detach().to("cpu", torch.float32).numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _i32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _per_head(x, Hq):
    a = np.asarray(x, dtype=np.int32).reshape(-1)
    if a.size == 1:
        a = np.full(Hq, int(a[0]), dtype=np.int32)
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


class Problem:
    """One attention problem, widened to fp32 host arrays (exact for bf16/fp32)."""

    def __init__(self, q, k, v, *, window, dilation=1, causal=False, global_idx=None,
                 side_k=None, side_v=None, side_block=16, bias=None, valid_len=None, scale=None,
                 local_bias=None, rand_blocks=None, rand_block=128):
        """``local_bias``: optional [Hq, 2R+1] table added to window keys of non-global
        rows at column (j - i) + R (R inferred from the table width).
        ``rand_blocks``: optional int [B, Hq, ceil(n / rand_block), r] random key
        blocks of each query block (non-global rows attend their keys too)."""
        self.q, self.k, self.v = _f32(q), _f32(k), _f32(v)
        self.B, self.Hq, self.n, self.D = self.q.shape
        self.Hkv = self.k.shape[1]
        self.window = _per_head(window, self.Hq)
        self.dilation = _per_head(dilation, self.Hq)
        self.causal = int(bool(causal))
        self.global_idx = _i32(global_idx)
        self.g = 0 if self.global_idx is None else int(self.global_idx.shape[-1])
        if self.g == 0:
            self.global_idx = None
        self.side_k, self.side_v = _f32(side_k), _f32(side_v)
        self.S = 0 if self.side_k is None else int(self.side_k.shape[2])
        self.side_block = int(side_block) if self.S else 0
        self.bias = _f32(bias)
        self.valid_len = _i32(valid_len)
        self.scale = float(scale) if scale is not None else 1.0 / np.sqrt(self.D)
        self.local_bias = _f32(local_bias)
        self.local_radius = 0
        if self.local_bias is not None:
            width = self.local_bias.shape[-1]
            if self.local_bias.shape != (self.Hq, width) or width % 2 == 0:
                raise ValueError("local_bias must be [Hq, 2R+1]")
            self.local_radius = (width - 1) // 2
        self.rand_blocks = _i32(rand_blocks)
        self.rand_block = int(rand_block)
        if self.rand_blocks is not None:
            nqb = (self.n + self.rand_block - 1) // self.rand_block
            if self.rand_blocks.ndim != 4 or self.rand_blocks.shape[:3] != (self.B, self.Hq, nqb):
                raise ValueError("rand_blocks must be [B, Hq, ceil(n / rand_block), r]")

    def _ex(self):
        self._exk = _extras(self.local_bias, self.local_radius, self.rand_blocks, self.rand_block)
        return ctypes.byref(self._exk)

    def _common(self):
        return (self.B, self.Hq, self.Hkv, self.n, self.D, _ptr(self.q), _ptr(self.k), _ptr(self.v),
                _ptr(self.global_idx), self.g, _ptr(self.side_k), _ptr(self.side_v), self.S,
                self.side_block, _ptr(self.bias), _ptr(self.window), _ptr(self.dilation),
                self.causal, _ptr(self.valid_len), self.scale)

    def forward(self, rows=None):
        """fp64 (out, lse, count).  ``rows``: flat row ids (b*Hq+h)*n+i, or None for all.

        Without ``rows`` the results are shaped [B,Hq,n,D] / [B,Hq,n]; with rows they
        are [len(rows), D] / [len(rows)].
        """
        lib = _load()
        if rows is None:
            total = self.B * self.Hq * self.n
            rp = None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            total = rows.size
            rp = _ptr(rows)
        out = np.empty((total, self.D), dtype=np.float64)
        lse = np.empty(total, dtype=np.float64)
        cnt = np.empty(total, dtype=np.int64)
        _check(lib.oracle_forward_ex(*self._common(), rp, total, _ptr(out), _ptr(lse), _ptr(cnt),
                                     self._ex()), "forward")
        if rows is None:
            return (out.reshape(self.B, self.Hq, self.n, self.D), lse.reshape(self.B, self.Hq, self.n),
                    cnt.reshape(self.B, self.Hq, self.n))
        return out, lse, cnt

    def backward(self, dout):
        """fp64 gradients for the upstream gradient ``dout`` (like q): (dq, dk, dv), plus
        (dside_k, dside_v) when the problem has side keys (a 5-tuple then)."""
        lib = _load()
        do = _f32(dout)
        dq = np.empty((self.B, self.Hq, self.n, self.D), dtype=np.float64)
        dk = np.empty((self.B, self.Hkv, self.n, self.D), dtype=np.float64)
        dv = np.empty((self.B, self.Hkv, self.n, self.D), dtype=np.float64)
        dsk = dsv = None
        if self.S:
            dsk = np.empty((self.B, self.Hkv, self.S, self.D), dtype=np.float64)
            dsv = np.empty((self.B, self.Hkv, self.S, self.D), dtype=np.float64)
        _check(lib.oracle_backward_ex(self.B, self.Hq, self.Hkv, self.n, self.D, _ptr(self.q),
                                      _ptr(self.k), _ptr(self.v), _ptr(do), _ptr(self.global_idx),
                                      self.g, _ptr(self.side_k), _ptr(self.side_v), self.S,
                                      self.side_block, _ptr(self.bias), _ptr(self.window),
                                      _ptr(self.dilation), self.causal, _ptr(self.valid_len),
                                      self.scale, self._ex(), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsk),
                                      _ptr(dsv)), "backward")
        if self.S:
            return dq, dk, dv, dsk, dsv
        return dq, dk, dv

    def dense_bruteforce(self):
        lib = _load()
        out = np.empty((self.B, self.Hq, self.n, self.D), dtype=np.float64)
        lse = np.empty((self.B, self.Hq, self.n), dtype=np.float64)
        _check(lib.oracle_dense_bruteforce_ex(*self._common(), _ptr(out), _ptr(lse), self._ex()),
               "dense")
        return out, lse


def key_counts(B, Hq, n, *, window, dilation=1, causal=False, global_idx=None, S=0,
               valid_len=None, rand_blocks=None, rand_block=128):
    """|K(i)| + S per row, [B,Hq,n] int64 (0 for padded rows)."""
    lib = _load()
    gi = _i32(global_idx)
    g = 0 if gi is None else int(gi.shape[-1])
    vl = _i32(valid_len)
    rb = _i32(rand_blocks)
    cnt = np.empty((B, Hq, n), dtype=np.int64)
    ex = _extras(rand_blocks=rb, rand_block=rand_block)
    _check(lib.oracle_key_counts_ex(B, Hq, n, _ptr(gi) if g else None, g, S,
                                    _ptr(_per_head(window, Hq)), _ptr(_per_head(dilation, Hq)),
                                    int(bool(causal)), _ptr(vl), _ptr(cnt), ctypes.byref(ex)),
           "key_counts")
    return cnt


def key_list(B, Hq, n, b, h, i, *, window, dilation=1, causal=False, global_idx=None,
             valid_len=None, rand_blocks=None, rand_block=128):
    """The explicit key set K(i) (ascending, no side keys) of one row."""
    lib = _load()
    gi = _i32(global_idx)
    g = 0 if gi is None else int(gi.shape[-1])
    vl = _i32(valid_len)
    rb = _i32(rand_blocks)
    keys = np.empty(max(n, 1), dtype=np.int32)
    w, d = _per_head(window, Hq), _per_head(dilation, Hq)
    ex = _extras(rand_blocks=rb, rand_block=rand_block)
    nk = lib.oracle_key_list_ex(B, Hq, n, _ptr(gi) if g else None, g, _ptr(w), _ptr(d),
                                int(bool(causal)), _ptr(vl), b, h, i, _ptr(keys), ctypes.byref(ex))
    if nk < 0:
        raise MemoryError("oracle key_list")
    return keys[:nk].copy()


def relative_bucket(delta: int) -> int:
    return int(_load().oracle_relative_bucket(int(delta)))


def expand_side_bias(table, S: int, nblk: int):
    """[Hq,32] bucket table -> [Hq, S + nblk - 1] fp32 side-bias table."""
    t = _f32(table)
    Hq = t.shape[0]
    out = np.empty((Hq, S + nblk - 1), dtype=np.float32)
    _check(_load().oracle_expand_side_bias(Hq, S, nblk, _ptr(t), _ptr(out)), "expand_side_bias")
    return out


def expand_local_bias(table, radius: int):
    """[Hq,32] bucket table -> [Hq, 2*radius + 1] fp32 local-bias table: column c
    holds the T5 bucket of the token offset c - radius (memory minus query
    position; LongT5 guide, 相对位置编码 section)."""
    t = _f32(table)
    cols = [relative_bucket(c - radius) for c in range(2 * radius + 1)]
    return np.ascontiguousarray(t[:, cols], dtype=np.float32)


def side_aggregate(x, block: int, valid_len=None):
    """Block means [B,H,n,D] -> [B,H,n//block,D] (fp64)."""
    a = _f32(x)
    B, H, n, D = a.shape
    vl = _i32(valid_len)
    out = np.empty((B, H, n // block, D), dtype=np.float64)
    _check(_load().oracle_side_aggregate(B, H, n, D, block, _ptr(a), _ptr(vl), _ptr(out)),
           "side_aggregate")
    return out


def num_threads() -> int:
    return int(_load().oracle_num_threads())
