"""Seeded synthetic workloads for banded sparse self-attention.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the fp64 oracle and the CUDA path can consume the
same tensors.  The five named workloads follow the shapes of the pages' use
cases:

* ``longformer_tiny``  -- tiny Longformer-pattern check (fp32, one global token)
* ``longformer_base``  -- Longformer-base shape: 12 heads, n=4096, r=256,
  64 leading global (question) tokens, the last 300 positions padding
* ``dilated``          -- 2 x 12 heads, n=8192, r=256, dilation 2 on the last two
  heads, 8 seeded random global tokens per batch
* ``longt5_tglobal``   -- LongT5 Transient-Global pattern: n=16384, r=127 plus
  1024 side keys (block means of 16 tokens) with a 32-bucket side bias
* ``swan_swa``         -- SWAN-GPT SWA-RoPE layer: 32 query / 8 KV heads, n=32768,
  D=128, causal window of 512 keys, q and k rotated by RoPE (base 10000)
* ``longt5_local``     -- LongT5 Local attention: n=16384, 12 heads, r=127 with the
  local relative-position bias (a 32-bucket table per head over the token offset)
* ``bigbird_itc``      -- BigBird-ITC pattern: n=4096, 12 heads, r=191 (three
  128-key blocks), the first 128 tokens global, 3 random key blocks of 128 per
  query block

Inputs are N(0,1) from ``torch.Generator('cpu').manual_seed(seed)`` drawn in
the order q, k, v, global positions, side-bias table, local-bias table, random
key blocks, then rounded to the dtype.  Random blocks of query block q are drawn
without replacement from the blocks other than q-1, q, q+1 and the global
blocks, per (batch, head, query block).  Side keys/values (block means) and the expanded bias
tables are NOT made here: each side (oracle and CUDA library) derives them with
its own code.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    seq_len: int
    head_dim: int
    dtype: str                      # "fp32" | "bf16"
    window: tuple                   # one-sided radius r per query head
    dilation: tuple                 # per query head
    causal: bool = False
    num_global: int = 0
    global_mode: str = "none"       # "none" | "leading" | "random"
    padding: int = 0                # trailing padded positions (valid_len = n - padding)
    side_block: int = 0             # k of the Transient-Global blocks (0: no side keys)
    side_bias: bool = False         # seeded 32-bucket side-bias table
    local_bias: bool = False        # seeded 32-bucket local relative-position bias table
    num_rand: int = 0               # random key blocks of 128 per query block
    rope: bool = False              # rotate q and k with RoPE (base 10000, all dims)
    seed: int = 0

    def __post_init__(self):
        if len(self.window) != self.q_heads or len(self.dilation) != self.q_heads:
            raise ValueError(f"{self.name}: window/dilation need one value per query head")
        if self.q_heads % self.kv_heads:
            raise ValueError(f"{self.name}: q_heads must be a multiple of kv_heads")

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    @property
    def num_side(self) -> int:
        return self.seq_len // self.side_block if self.side_block else 0

    @property
    def valid_len(self) -> int:
        return self.seq_len - self.padding

    def describe(self) -> dict:
        d = dataclasses.asdict(self)
        d["window"] = sorted(set(self.window))
        d["dilation"] = sorted(set(self.dilation))
        return d


def _heads(val, H):
    return tuple([val] * H) if isinstance(val, int) else tuple(val)


WORKLOADS = {
    "longformer_tiny": Workload("longformer_tiny", 1, 2, 2, 256, 64, "fp32", _heads(32, 2),
                                _heads(1, 2), num_global=1, global_mode="leading", seed=1001),
    "longformer_base": Workload("longformer_base", 1, 12, 12, 4096, 64, "bf16", _heads(256, 12),
                                _heads(1, 12), num_global=64, global_mode="leading", padding=300,
                                seed=1002),
    "dilated": Workload("dilated", 2, 12, 12, 8192, 64, "bf16", _heads(256, 12),
                        tuple([1] * 10 + [2] * 2), num_global=8, global_mode="random", seed=1003),
    "longt5_tglobal": Workload("longt5_tglobal", 1, 12, 12, 16384, 64, "bf16", _heads(127, 12),
                               _heads(1, 12), side_block=16, side_bias=True, seed=1004),
    "swan_swa": Workload("swan_swa", 1, 32, 8, 32768, 128, "bf16", _heads(511, 32), _heads(1, 32),
                         causal=True, rope=True, seed=1005),
    "longt5_local": Workload("longt5_local", 1, 12, 12, 16384, 64, "bf16", _heads(127, 12),
                             _heads(1, 12), local_bias=True, seed=1006),
    "bigbird_itc": Workload("bigbird_itc", 1, 12, 12, 4096, 64, "bf16", _heads(191, 12),
                            _heads(1, 12), num_global=128, global_mode="leading", num_rand=3,
                            seed=1007),
}

# Reduced versions with the same structure (several tiles and a ragged tail) that the
# fp64 oracle finishes in seconds.
SMALL = {
    "longformer_tiny": WORKLOADS["longformer_tiny"],
    "longformer_base": dataclasses.replace(WORKLOADS["longformer_base"], name="longformer_base_small",
                                           seq_len=1000, window=_heads(100, 4), dilation=_heads(1, 4),
                                           num_global=16, padding=77, q_heads=4, kv_heads=4,
                                           seed=2002),
    "dilated": dataclasses.replace(WORKLOADS["dilated"], name="dilated_small", seq_len=1111,
                                   q_heads=4, kv_heads=4, window=_heads(70, 4),
                                   dilation=(1, 1, 2, 3), num_global=5, seed=2003),
    "longt5_tglobal": dataclasses.replace(WORKLOADS["longt5_tglobal"], name="longt5_tglobal_small",
                                          seq_len=1024, q_heads=3, kv_heads=3, window=_heads(127, 3),
                                          dilation=_heads(1, 3), seed=2004),
    "swan_swa": dataclasses.replace(WORKLOADS["swan_swa"], name="swan_swa_small", seq_len=1200,
                                    q_heads=8, kv_heads=2, window=_heads(300, 8),
                                    dilation=_heads(1, 8), seed=2005),
    "longt5_local": dataclasses.replace(WORKLOADS["longt5_local"], name="longt5_local_small",
                                        seq_len=1100, q_heads=3, kv_heads=3, window=_heads(127, 3),
                                        dilation=_heads(1, 3), padding=45, seed=2006),
    "bigbird_itc": dataclasses.replace(WORKLOADS["bigbird_itc"], name="bigbird_itc_small",
                                       seq_len=1300, q_heads=4, kv_heads=4, window=_heads(100, 4),
                                       dilation=_heads(1, 4),
                                       num_global=20, padding=37, seed=2007),
}


def _rope_(x: torch.Tensor, positions: torch.Tensor) -> torch.Tensor:
    """Input recipe of the SWA-RoPE workload: rotate interleaved pairs (2m, 2m+1) by
    angle pos * 10000^(-2m/D), in fp64, one head at a time.  Returns fp64."""
    D = x.shape[-1]
    theta = torch.pow(torch.tensor(10000.0, dtype=torch.float64),
                      -torch.arange(0, D, 2, dtype=torch.float64) / D)
    ang = positions.to(torch.float64)[:, None] * theta[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    out = torch.empty(x.shape, dtype=torch.float64)
    for b in range(x.shape[0]):
        for h in range(x.shape[1]):
            xx = x[b, h].to(torch.float64)
            x0, x1 = xx[:, 0::2], xx[:, 1::2]
            out[b, h, :, 0::2] = x0 * c - x1 * s
            out[b, h, :, 1::2] = x0 * s + x1 * c
    return out


def make_inputs(w: Workload, seed: Optional[int] = None) -> dict:
    """Draw one workload's tensors on the host (CPU), already rounded to ``w.dtype``."""
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    B, Hq, Hkv, n, D = w.batch, w.q_heads, w.kv_heads, w.seq_len, w.head_dim
    q = torch.randn((B, Hq, n, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, n, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, n, D), generator=g, dtype=torch.float32)
    global_idx = None
    if w.num_global:
        if w.global_mode == "leading":
            global_idx = torch.arange(w.num_global, dtype=torch.int32).repeat(B, 1)
        else:
            rows = []
            for _ in range(B):
                perm = torch.randperm(w.valid_len, generator=g)[: w.num_global]
                rows.append(torch.sort(perm).values)
            global_idx = torch.stack(rows).to(torch.int32)
    bias_table = None
    if w.side_bias:
        bias_table = torch.randn((Hq, 32), generator=g, dtype=torch.float32)
    local_table = None
    if w.local_bias:
        local_table = torch.randn((Hq, 32), generator=g, dtype=torch.float32)
    rand_blocks = None
    if w.num_rand:
        nqb = (n + 127) // 128
        gblocks = set()
        if global_idx is not None:
            gblocks = {int(x) // 128 for x in global_idx.reshape(-1).tolist()}
        rand_blocks = torch.empty((B, Hq, nqb, w.num_rand), dtype=torch.int32)
        for b in range(B):
            for h in range(Hq):
                for qb in range(nqb):
                    cand = [x for x in range(nqb) if abs(x - qb) > 1 and x not in gblocks]
                    if len(cand) < w.num_rand:
                        cand = list(range(nqb))
                    pick = torch.randperm(len(cand), generator=g)[: w.num_rand]
                    rand_blocks[b, h, qb] = torch.tensor([cand[int(t)] for t in pick], dtype=torch.int32)
    if w.rope:
        pos = torch.arange(n)
        q = _rope_(q, pos)
        k = _rope_(k, pos)
    dt = w.torch_dtype
    return dict(
        q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
        global_idx=global_idx,
        bias_table=bias_table,
        local_table=local_table,
        rand_blocks=rand_blocks,
        window=torch.tensor(w.window, dtype=torch.int32),
        dilation=torch.tensor(w.dilation, dtype=torch.int32),
        causal=w.causal,
        valid_len=(torch.full((B,), w.valid_len, dtype=torch.int32) if w.padding else None),
        side_block=w.side_block,
        num_side=w.num_side,
        scale=1.0 / math.sqrt(D),
    )
