"""The bench's closed-form pair count against the oracle's explicit key sets."""
import numpy as np
import pytest

import oracle
from sliding_window_global_b200 import flops, workloads


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_pair_count_matches_oracle(name):
    w = workloads.WORKLOADS[name]
    need = (w.num_global and w.global_mode == "random") or w.num_rand
    inp = workloads.make_inputs(w) if need else None
    gl = inp["global_idx"].numpy() if inp is not None and inp["global_idx"] is not None else (
        np.tile(np.arange(w.num_global, dtype=np.int32), (w.batch, 1)) if w.num_global else None)
    rb = inp["rand_blocks"].numpy() if inp is not None and inp["rand_blocks"] is not None else None
    vl = np.full(w.batch, w.valid_len, np.int32) if w.padding else None
    ours = flops.attended_pairs(w.seq_len, w.window, w.dilation, w.causal, gl, vl, w.batch,
                                w.num_side, rb)
    ref = oracle.key_counts(w.batch, w.q_heads, w.seq_len, window=np.array(w.window),
                            dilation=np.array(w.dilation), causal=w.causal, global_idx=gl,
                            S=w.num_side, valid_len=vl, rand_blocks=rb).sum()
    assert ours == ref


def test_pair_count_small_grid():
    rng = np.random.default_rng(1)
    for _ in range(40):
        n = int(rng.integers(1, 90))
        H = int(rng.integers(1, 4))
        causal = bool(rng.integers(0, 2))
        window = rng.integers(0, 12, size=H)
        dil = rng.integers(1, 4, size=H)
        V = int(rng.integers(1, n + 1))
        g = 0 if causal else int(rng.integers(0, min(4, V) + 1))
        gl = np.sort(rng.choice(V, g, replace=False))[None].astype(np.int32) if g else None
        S = int(rng.integers(0, 3))
        ours = flops.attended_pairs(n, window, dil, causal, gl, np.array([V]), 1, S)
        ref = oracle.key_counts(1, H, n, window=window, dilation=dil, causal=causal, global_idx=gl,
                                S=S, valid_len=np.array([V], np.int32)).sum()
        assert ours == ref


def test_pair_count_with_random_blocks():
    rng = np.random.default_rng(3)
    for _ in range(25):
        n = int(rng.integers(1, 70))
        H = int(rng.integers(1, 3))
        bs = int(rng.integers(2, 9))
        nqb = (n + bs - 1) // bs
        r = int(rng.integers(1, 4))
        rb = rng.integers(0, nqb, size=(1, H, nqb, r)).astype(np.int32)
        window = rng.integers(0, 6, size=H)
        dil = rng.integers(1, 3, size=H)
        V = int(rng.integers(1, n + 1))
        g = int(rng.integers(0, min(3, V) + 1))
        gl = np.sort(rng.choice(V, g, replace=False))[None].astype(np.int32) if g else None
        ours = flops.attended_pairs(n, window, dil, False, gl, np.array([V]), 1, 0, rb, bs)
        ref = oracle.key_counts(1, H, n, window=window, dilation=dil, global_idx=gl,
                                valid_len=np.array([V], np.int32), rand_blocks=rb,
                                rand_block=bs).sum()
        assert ours == ref
