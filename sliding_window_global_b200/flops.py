"""Useful work of one forward: attended (query, key) pairs and FLOPs.

useful FLOPs = 4 * D * sum over valid query rows of |K(i)| + S  (2*D for q.k and
2*D for p.v per attended pair).  Masked, padded and skipped work is excluded: this
is the method's algorithmic work, not the dense n^2 work it avoids.

Counted in closed form per row (vectorised over rows):
  window part |W(i)| = t_hi - t_lo + 1 with t_lo = max(-r, -floor(i/d)) and
  t_hi = 0 (causal) or min(r, floor((V-1-i)/d)); plus the global keys outside the
  window; plus the keys of the row's random key blocks that are neither global nor
  in the window (counted once each); a global query row instead counts every valid
  key; plus S side keys.
"""
from __future__ import annotations

import numpy as np


def _random_extra(i, V, r, d, causal, gl, blocks, bs):
    """Per row of one query block: keys of its random blocks outside W(i) and G."""
    keys = np.unique(np.concatenate([np.arange(b * bs, b * bs + bs) for b in blocks]))
    keys = keys[(keys >= 0) & (keys < V)]
    keys = np.setdiff1d(keys, gl, assume_unique=False)
    if keys.size == 0:
        return np.zeros(i.size, np.int64)
    diff = i[:, None] - keys[None, :]
    inwin = diff % d == 0
    inwin &= ((diff >= 0) & (diff <= r * d)) if causal else (np.abs(diff) <= r * d)
    return (~inwin).sum(1).astype(np.int64)


def attended_pairs(n: int, window, dilation, causal: bool, global_idx=None, valid_len=None,
                   batch: int = 1, num_side: int = 0, rand_blocks=None, rand_block: int = 128) -> int:
    window = np.asarray(window, dtype=np.int64).reshape(-1)
    dilation = np.asarray(dilation, dtype=np.int64).reshape(-1)
    if dilation.size == 1:
        dilation = np.full(window.size, int(dilation[0]), dtype=np.int64)
    total = 0
    for b in range(batch):
        V = int(valid_len[b]) if valid_len is not None else n
        V = min(V, n)
        i = np.arange(V, dtype=np.int64)
        gl = np.asarray(global_idx[b], dtype=np.int64) if global_idx is not None else np.zeros(0, np.int64)
        gl = gl[gl < V]
        isg = np.zeros(V, bool)
        isg[gl] = True
        for h, (r, d) in enumerate(zip(window.tolist(), dilation.tolist())):
            t_lo = np.maximum(-r, -(i // d))
            t_hi = np.zeros_like(i) if causal else np.minimum(r, (V - 1 - i) // d)
            cnt = t_hi - t_lo + 1
            if gl.size:
                diff = i[:, None] - gl[None, :]
                inwin = (diff % d == 0)
                if causal:
                    inwin &= (diff >= 0) & (diff <= r * d)
                else:
                    inwin &= np.abs(diff) <= r * d
                cnt = cnt + (~inwin).sum(1)
            if rand_blocks is not None and np.shape(rand_blocks)[-1] > 0:
                rb = np.asarray(rand_blocks[b][h], dtype=np.int64)
                for qb in range(rb.shape[0]):
                    rows = i[qb * rand_block: (qb + 1) * rand_block]
                    if rows.size:
                        cnt[rows] += _random_extra(rows, V, r, d, causal, gl, rb[qb], rand_block)
            if gl.size:
                cnt = np.where(isg, V, cnt)
            total += int(cnt.sum()) + V * num_side
    return total


def useful_flops(pairs: int, head_dim: int) -> int:
    return 4 * head_dim * pairs
