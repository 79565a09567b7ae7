"""Banded sparse self-attention for NVIDIA B200 (sm_100a).

Sliding-window attention with optional dilation and causal mask, global tokens
(global rows and columns), LongT5-style appended side keys with an additive
bucketed bias, a LongT5 local relative-position bias on window keys, and grouped
KV heads -- computed by the hand-written CUDA kernels
of ``libswa.so`` behind the C ABI in ``include/swa.h``.  This Python layer only
marshals arguments: PyTorch provides device memory and streams.
"""
from .swa import (  # noqa: F401
    Plan,
    SwaError,
    bucket_local_bias,
    expand_side_bias,
    forward,
    lib_path,
    load_library,
    relative_bucket,
    side_aggregate,
)
