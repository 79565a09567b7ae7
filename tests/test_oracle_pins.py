"""Pins of the fp64 oracle against things other than itself (CPU only).

* brute force: an independent dense-mask statement of the same attention, on a
  grid of tiny problems (values <= 1e-12, supports exact via one-hot V);
* the worked window example of the BigBird notes (tests/golden);
* closed cases: window >= n is full (or causal) softmax attention from torch;
  global rows are full-attention rows; weights sum to one; outputs stay in the
  convex hull of the attended V rows; padded rows are exactly zero; q = 0 gives
  the plain mean over the key set (a cardinality check); dilation d equals d
  independent residue problems; GQA equals MHA with replicated K/V; side keys
  merge with the window part through the logsumexp identity;
* attended-pair counts against the closed forms of the LongT5 complexity
  statements O(l*r) and O(l*(r + l/k));
* the T5 bucket function against its threshold table and a float-log
  evaluation of the textbook formula.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng):
    return rng.standard_normal(shape).astype(np.float32)


def _problem(oracle_mod, rng, B, Hq, Hkv, n, D, r, d, causal, g, pad, S=0, kb=4, bias=False):
    q = _rand((B, Hq, n, D), rng)
    k = _rand((B, Hkv, n, D), rng)
    v = _rand((B, Hkv, n, D), rng)
    V = max(n - pad, 0)
    gi = None
    if g and V > 0:
        g = min(g, V)
        gi = np.stack([np.sort(rng.choice(V, g, replace=False)) for _ in range(B)]).astype(np.int32)
    sk = sv = bt = None
    if S:
        sk = _rand((B, Hkv, S, D), rng)
        sv = _rand((B, Hkv, S, D), rng)
        if bias:
            nblk = (n + kb - 1) // kb
            bt = _rand((Hq, S + nblk - 1), rng)
    vl = np.full(B, V, np.int32) if pad else None
    return oracle_mod.Problem(q, k, v, window=r, dilation=d, causal=causal, global_idx=gi,
                              side_k=sk, side_v=sv, side_block=kb, bias=bt, valid_len=vl)


def _assert_close_lse(a, b, tol):
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    m = ~np.isneginf(a)
    if m.any():
        assert np.max(np.abs(a[m] - b[m])) <= tol


def test_worked_window_example(oracle_mod):
    with open(os.path.join(GOLDEN, "bigbird_window_example.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for n, r, pos, attended in rows:
        n, r, pos = int(n), int(r), int(pos)
        expect = [int(x) - 1 for x in attended.split(",")]
        keys = oracle_mod.key_list(1, 1, n, 0, 0, pos - 1, window=r)
        assert keys.tolist() == expect


def test_oracle_matches_dense_bruteforce_grid(oracle_mod):
    rng = np.random.default_rng(7)
    cases = 0
    for n in (1, 2, 3, 5, 8, 13, 21, 33, 40):
        for r, d, causal, g, pad in itertools.product((0, 1, 2, 5), (1, 2, 3), (0, 1), (0, 1, 3),
                                                      (0, 1, 3)):
            if rng.random() > 0.22:   # a seeded third of the grid keeps the run short
                continue
            S = int(rng.integers(0, 3)) * 2
            G = int(rng.choice([1, 2]))
            p = _problem(oracle_mod, rng, 2, 2 * G, 2, n, 8, r, d, causal, g, pad, S=S, kb=4,
                         bias=bool(S and rng.random() < 0.7))
            o, lse, _ = p.forward()
            od, lsed = p.dense_bruteforce()
            assert np.max(np.abs(o - od)) <= 1e-12
            _assert_close_lse(lse, lsed, 1e-12)
            cases += 1
    assert cases > 150


def test_support_exact_onehot_v(oracle_mod):
    """V = identity rows -> o_i is the weight row; zero pattern must agree exactly."""
    rng = np.random.default_rng(11)
    for (n, r, d, causal, g, pad) in [(24, 2, 1, 0, 2, 3), (24, 3, 2, 0, 3, 0), (24, 4, 3, 1, 0, 2),
                                      (17, 1, 1, 1, 0, 0), (24, 0, 1, 0, 1, 5)]:
        p = _problem(oracle_mod, rng, 1, 2, 2, n, n, r, d, causal, g, pad)
        p.v = np.ascontiguousarray(np.broadcast_to(np.eye(n, dtype=np.float32), p.v.shape))
        o, _, cnt = p.forward()
        od, _ = p.dense_bruteforce()
        assert np.array_equal(o > 0, od > 0)
        assert np.array_equal((o > 0).sum(-1), cnt)   # no side keys: count = |K(i)|


def test_window_covering_sequence_is_full_attention(oracle_mod):
    rng = np.random.default_rng(3)
    n, D = 37, 16
    for causal in (0, 1):
        p = _problem(oracle_mod, rng, 2, 4, 2, n, D, n, 1, causal, 0, 0)
        o, _, _ = p.forward()
        q = torch.from_numpy(p.q).double()
        k = torch.from_numpy(p.k).double().repeat_interleave(2, dim=1)
        v = torch.from_numpy(p.v).double().repeat_interleave(2, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=bool(causal))
        assert np.max(np.abs(o - ref.numpy())) <= 1e-12
    # dilation with r*d >= n but d > 1 is not full attention: only the residue class
    p = _problem(oracle_mod, rng, 1, 1, 1, n, D, n, 2, 0, 0, 0)
    _, _, cnt = p.forward()
    assert cnt[0, 0, 0] == (n + 1) // 2


def test_global_rows_are_full_attention_rows(oracle_mod):
    rng = np.random.default_rng(5)
    n, D, pad = 50, 16, 6
    p = _problem(oracle_mod, rng, 2, 2, 2, n, D, 3, 2, 0, 4, pad)
    o, lse, _ = p.forward()
    V = n - pad
    q = torch.from_numpy(p.q).double()[..., :V, :]
    k = torch.from_numpy(p.k).double()[..., :V, :]
    v = torch.from_numpy(p.v).double()[..., :V, :]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    s = torch.einsum("bhid,bhjd->bhij", q, k) * p.scale
    ref_lse = torch.logsumexp(s, -1)
    for b in range(2):
        for i in p.global_idx[b]:
            assert np.max(np.abs(o[b, :, i] - ref.numpy()[b, :, i])) <= 1e-12
            assert np.max(np.abs(lse[b, :, i] - ref_lse.numpy()[b, :, i])) <= 1e-12


def test_weights_sum_to_one_and_convex_hull(oracle_mod):
    rng = np.random.default_rng(9)
    p = _problem(oracle_mod, rng, 2, 4, 2, 64, 16, 5, 2, 0, 3, 7, S=4, kb=8, bias=True)
    ones = p.v.copy()
    p.v = np.ones_like(p.v)
    sv = p.side_v
    p.side_v = np.ones_like(p.side_v)
    o, _, cnt = p.forward()
    valid = cnt > 0
    assert np.max(np.abs(o[valid] - 1.0)) <= 1e-13
    p.v, p.side_v = ones, sv
    o, _, _ = p.forward()
    for b, h, i in itertools.product(range(2), range(4), range(64)):
        if not valid[b, h, i]:
            continue
        keys = oracle_mod.key_list(2, 4, 64, b, h, i, window=p.window, dilation=p.dilation,
                                   global_idx=p.global_idx, valid_len=p.valid_len)
        rows = np.concatenate([p.v[b, h // 2, keys], p.side_v[b, h // 2]], 0)
        assert np.all(o[b, h, i] <= rows.max(0) + 1e-12)
        assert np.all(o[b, h, i] >= rows.min(0) - 1e-12)


def test_padded_rows_exact_zero(oracle_mod):
    rng = np.random.default_rng(13)
    p = _problem(oracle_mod, rng, 2, 2, 2, 30, 8, 3, 1, 0, 2, 9, S=2, kb=4, bias=True)
    o, lse, cnt = p.forward()
    assert np.all(o[:, :, 21:] == 0.0)
    assert np.all(np.isneginf(lse[:, :, 21:]))
    assert np.all(cnt[:, :, 21:] == 0)
    assert np.all(np.isfinite(o))
    assert np.all(np.isfinite(lse[:, :, :21]))


def test_zero_query_gives_mean_over_key_set(oracle_mod):
    rng = np.random.default_rng(17)
    p = _problem(oracle_mod, rng, 1, 2, 2, 40, 8, 4, 3, 0, 3, 2, S=3, kb=8)
    p.q = np.zeros_like(p.q)
    o, lse, cnt = p.forward()
    for h, i in itertools.product(range(2), range(38)):
        keys = oracle_mod.key_list(1, 2, 40, 0, h, i, window=p.window, dilation=p.dilation,
                                   global_idx=p.global_idx, valid_len=p.valid_len)
        rows = np.concatenate([p.v[0, h, keys], p.side_v[0, h]], 0).astype(np.float64)
        assert rows.shape[0] == cnt[0, h, i]
        assert np.max(np.abs(o[0, h, i] - rows.mean(0))) <= 1e-13
        assert abs(lse[0, h, i] - math.log(cnt[0, h, i])) <= 1e-13


def test_dilation_equals_residue_subproblems(oracle_mod):
    rng = np.random.default_rng(19)
    n, D, r = 41, 8, 3
    for d, causal in [(2, 0), (3, 0), (3, 1), (5, 0)]:
        p = _problem(oracle_mod, rng, 1, 1, 1, n, D, r, d, causal, 0, 0)
        o, lse, _ = p.forward()
        for c in range(d):
            idx = np.arange(c, n, d)
            sub = oracle_mod.Problem(p.q[:, :, idx], p.k[:, :, idx], p.v[:, :, idx], window=r,
                                     dilation=1, causal=causal, scale=p.scale)
            os_, ls_, _ = sub.forward()
            assert np.max(np.abs(o[:, :, idx] - os_)) <= 1e-14
            assert np.max(np.abs(lse[:, :, idx] - ls_)) <= 1e-14


def test_gqa_equals_replicated_mha(oracle_mod):
    rng = np.random.default_rng(23)
    p = _problem(oracle_mod, rng, 2, 6, 2, 29, 8, 2, 1, 0, 2, 3, S=2, kb=4, bias=True)
    o, lse, _ = p.forward()
    rep = oracle_mod.Problem(p.q, np.repeat(p.k, 3, axis=1), np.repeat(p.v, 3, axis=1),
                             window=p.window, dilation=p.dilation, global_idx=p.global_idx,
                             side_k=np.repeat(p.side_k, 3, axis=1), side_v=np.repeat(p.side_v, 3, axis=1),
                             side_block=4, bias=p.bias, valid_len=p.valid_len)
    o2, lse2, _ = rep.forward()
    assert np.max(np.abs(o - o2)) == 0.0
    _assert_close_lse(lse, lse2, 0.0)


def test_side_keys_merge_by_logsumexp(oracle_mod):
    """attn(K(i) U S) == lse-merge(attn(K(i)), attn(S)); the side part computed with
    torch over the bias column the LongT5 side bias names (memory block - query block)."""
    rng = np.random.default_rng(29)
    n, D, S, kb = 48, 8, 6, 8
    p = _problem(oracle_mod, rng, 1, 2, 2, n, D, 3, 1, 0, 0, 0, S=S, kb=kb, bias=True)
    o, lse, _ = p.forward()
    nos = oracle_mod.Problem(p.q, p.k, p.v, window=p.window, dilation=p.dilation)
    o1, l1, _ = nos.forward()
    q = torch.from_numpy(p.q).double()
    sk = torch.from_numpy(p.side_k).double()
    sv = torch.from_numpy(p.side_v).double()
    s = torch.einsum("bhid,bhsd->bhis", q, sk) * p.scale
    nblk = n // kb
    bias = torch.from_numpy(p.bias).double()
    i = torch.arange(n)[:, None]
    sig = torch.arange(S)[None, :]
    col = sig - i // kb + nblk - 1
    s = s + bias[:, col][None]
    l2 = torch.logsumexp(s, -1).numpy()
    o2 = torch.einsum("bhis,bhsd->bhid", torch.softmax(s, -1), sv).numpy()
    m = np.maximum(l1, l2)
    w1, w2 = np.exp(l1 - m), np.exp(l2 - m)
    merged = (o1 * w1[..., None] + o2 * w2[..., None]) / (w1 + w2)[..., None]
    assert np.max(np.abs(o - merged)) <= 1e-12
    assert np.max(np.abs(lse - (m + np.log(w1 + w2)))) <= 1e-12


def test_pair_counts_match_complexity_closed_forms(oracle_mod):
    # LongT5 Local: each token sees r on each side: sum |W(i)| = n(2r+1) - r(r+1) for n > r
    n, r = 1000, 127
    cnt = oracle_mod.key_counts(1, 1, n, window=r)
    assert cnt.sum() == n * (2 * r + 1) - r * (r + 1)
    # Transient-Global adds every one of the S = n/k block summaries to every row
    cnt = oracle_mod.key_counts(1, 1, n, window=r, S=n // 16)
    assert cnt.sum() == n * (2 * r + 1) - r * (r + 1) + n * (n // 16)
    # causal window of 512 keys (r = 511) including self
    n, r = 3000, 511
    cnt = oracle_mod.key_counts(1, 1, n, window=r, causal=True)
    assert cnt.sum() == n * (r + 1) - r * (r + 1) // 2
    assert cnt[0, 0, -1] == 512


def test_local_keys_inside_three_block_context(oracle_mod):
    """LongT5 local attention splits into blocks of block_len = r + 1 and attends inside
    the 3-block context (previous, own, next): every window key must lie there."""
    n, r = 1024, 127
    bl = r + 1
    for i in (0, 1, 127, 128, 500, 1023):
        keys = oracle_mod.key_list(1, 1, n, 0, 0, i, window=r)
        blk = i // bl
        assert keys.min() >= max(0, (blk - 1) * bl)
        assert keys.max() < min(n, (blk + 2) * bl)
        assert len(keys) <= 3 * bl


def test_bucket_threshold_table(oracle_mod):
    with open(os.path.join(GOLDEN, "t5_bucket_thresholds.txt")) as f:
        rows = [tuple(map(int, l.split())) for l in f if l.strip() and not l.startswith("#")]
    for a in range(8):
        assert oracle_mod.relative_bucket(-a) == a
        assert oracle_mod.relative_bucket(a) == (16 + a if a else 0)
    for bucket, first in rows:
        assert oracle_mod.relative_bucket(-first) == bucket
        assert oracle_mod.relative_bucket(-(first - 1)) == bucket - 1
        assert oracle_mod.relative_bucket(first) == bucket + 16
    for a in (128, 129, 1000, 100000):
        assert oracle_mod.relative_bucket(-a) == 15
        assert oracle_mod.relative_bucket(a) == 31


def test_bucket_matches_float_log_formula(oracle_mod):
    """Textbook T5 bucket with the log in fp32 (as the reference library evaluates it)."""
    a = np.arange(1, 2048, dtype=np.int64)
    af = a.astype(np.float32)
    large = 8 + (np.log(af / np.float32(8)) / np.float32(math.log(128 / 8)) * np.float32(8)).astype(np.int64)
    expect = np.where(a < 8, a, np.minimum(large, 15))
    got = np.array([oracle_mod.relative_bucket(-int(x)) for x in a])
    assert np.array_equal(got, expect)
    got_pos = np.array([oracle_mod.relative_bucket(int(x)) for x in a])
    assert np.array_equal(got_pos, expect + 16)


def test_expand_side_bias_columns(oracle_mod):
    table = np.arange(2 * 32, dtype=np.float32).reshape(2, 32)
    S, nblk = 5, 7
    out = oracle_mod.expand_side_bias(table, S, nblk)
    assert out.shape == (2, S + nblk - 1)
    # column c holds delta = c - (nblk - 1): delta 0 -> bucket 0, +1 -> 17, -1 -> 1
    assert out[1, nblk - 1] == 32 + 0
    assert out[1, nblk] == 32 + 17
    assert out[1, nblk - 2] == 32 + 1
    assert out[0, 0] == oracle_mod.relative_bucket(-(nblk - 1))


def test_side_aggregate_block_means(oracle_mod):
    rng = np.random.default_rng(31)
    x = _rand((2, 3, 64, 4), rng)
    out = oracle_mod.side_aggregate(x, 16)
    ref = x.astype(np.float64).reshape(2, 3, 4, 16, 4).mean(3)
    assert np.max(np.abs(out - ref)) <= 1e-15
    # padding tokens belong to no block; a trailing partial block joins the previous one
    ramp = np.broadcast_to(np.arange(70, dtype=np.float32)[None, None, :, None], (1, 1, 70, 2)).copy()
    out = oracle_mod.side_aggregate(ramp, 16, valid_len=np.array([60], np.int32))
    assert out.shape == (1, 1, 4, 2)
    assert out[0, 0, 0, 0] == 7.5
    assert out[0, 0, 3, 0] == np.mean(np.arange(48, 60))


# --- local relative-position bias on window keys (LongT5 guide, 相对位置编码) ----------


def _local_table(rng, Hq, R):
    return _rand((Hq, 2 * R + 1), rng)


def test_local_bias_matches_dense_bruteforce_grid(oracle_mod):
    """The per-row path (bias looked up per key of K(i)) against the dense-mask brute
    force (bias added on the band mask of non-global rows), globals, sides, dilation,
    causal and padding included."""
    rng = np.random.default_rng(41)
    cases = 0
    for n in (3, 8, 21, 40):
        for r, d, causal, g, pad in itertools.product((0, 1, 3), (1, 2), (0, 1), (0, 2), (0, 3)):
            if rng.random() > 0.5:
                continue
            S = int(rng.integers(0, 2)) * 3
            p = _problem(oracle_mod, rng, 2, 4, 2, n, 8, r, d, causal, g, pad, S=S, kb=4, bias=bool(S))
            R = min(r * d, n - 1) + int(rng.integers(0, 3))
            lt = _local_table(rng, 4, R)
            pb = oracle_mod.Problem(p.q, p.k, p.v, window=r, dilation=d, causal=causal,
                                    global_idx=p.global_idx, side_k=p.side_k, side_v=p.side_v,
                                    side_block=4, bias=p.bias, valid_len=p.valid_len, local_bias=lt)
            o, lse, _ = pb.forward()
            od, lsed = pb.dense_bruteforce()
            assert np.max(np.abs(o - od)) <= 1e-12
            _assert_close_lse(lse, lsed, 1e-12)
            cases += 1
    assert cases > 30


def test_constant_local_bias_is_a_softmax_shift(oracle_mod):
    """With no global or side keys every key is a window key, so a per-head constant
    bias c shifts all scores: o is unchanged and lse moves by exactly c."""
    rng = np.random.default_rng(43)
    p = _problem(oracle_mod, rng, 2, 3, 3, 37, 16, 4, 2, 0, 0, 5)
    c = np.array([0.5, -2.0, 3.25], np.float32)
    lt = np.repeat(c[:, None], 2 * 8 + 1, axis=1)
    pb = oracle_mod.Problem(p.q, p.k, p.v, window=4, dilation=2, valid_len=p.valid_len, local_bias=lt)
    o0, l0, _ = p.forward()
    o1, l1, _ = pb.forward()
    assert np.max(np.abs(o0 - o1)) <= 1e-12
    m = ~np.isneginf(l0)
    assert np.array_equal(np.isneginf(l1), ~m)          # padded rows stay empty
    assert np.max(np.abs(l1[m] - l0[m] - np.broadcast_to(c[None, :, None], l0.shape)[m])) <= 1e-12


def test_local_bias_offset_sign_closed_form(oracle_mod):
    """q = 0 and bias = alpha * (j - i): the weight of window key j is
    exp(alpha (j - i)) / sum over the window -- a closed form that fails if the
    table is read at (i - j) or off by one."""
    n, r, d, alpha = 30, 3, 2, 0.75   # alpha * integer is exact in fp32
    R = r * d
    q = np.zeros((1, 1, n, n), np.float32)
    k = np.ones((1, 1, n, n), np.float32)
    v = np.eye(n, dtype=np.float32)[None, None]
    lt = (alpha * (np.arange(2 * R + 1) - R)).astype(np.float32)[None]
    o, _, _ = oracle_mod.Problem(q, k, v, window=r, dilation=d, local_bias=lt).forward()
    for i in range(n):
        js = [i + d * t for t in range(-r, r + 1) if 0 <= i + d * t < n]
        w = np.exp(alpha * (np.array(js) - i))
        expect = np.zeros(n)
        expect[js] = w / w.sum()
        assert np.max(np.abs(o[0, 0, i] - expect)) <= 1e-14


def test_side_bias_direction_closed_form(oracle_mod):
    """q = 0, window radius 0, one-hot V over the sequence and the side rows, and a
    side-bias table that is a known function f of delta = memory block - query block
    (LongT5 guide, 相对位置编码: the side keys' bias is bucketed on the block
    distance, memory minus query).  Row i then has weight 1 on itself and
    exp(f(sigma - floor(i / k))) on side key sigma, normalised -- a closed form that
    fails if the table is read at the query-minus-memory distance or off by one."""
    n, k, S = 40, 4, 6
    nblk = -(-n // k)
    f = lambda dlt: 0.25 * dlt + 0.03125 * dlt * dlt          # asymmetric, exact in fp32
    D = n + S
    q = np.zeros((1, 1, n, D), np.float32)
    kk = np.ones((1, 1, n, D), np.float32)
    v = np.eye(n, D, dtype=np.float32)[None, None]
    side_k = np.ones((1, 1, S, D), np.float32)
    side_v = np.eye(S, D, k=n, dtype=np.float32)[None, None]
    # the table layout of the interface: column c holds delta = c - (nblk - 1)
    bias = np.array([[f(c - (nblk - 1)) for c in range(S + nblk - 1)]], np.float32)
    o, lse, _ = oracle_mod.Problem(q, kk, v, window=0, side_k=side_k, side_v=side_v, side_block=k,
                                   bias=bias).forward()
    for i in range(n):
        w_side = np.exp([f(sig - i // k) for sig in range(S)])
        z = 1.0 + w_side.sum()
        expect = np.zeros(D)
        expect[i] = 1.0 / z
        expect[n:] = w_side / z
        assert np.max(np.abs(o[0, 0, i] - expect)) <= 1e-14
        assert abs(lse[0, 0, i] - np.log(z)) <= 1e-13


def test_local_bias_skips_global_rows_and_out_of_window_global_keys(oracle_mod):
    """Table = -1e30 except offset 0: a non-global row keeps itself and the global
    keys outside its window (a global key inside the window is a window key and is
    suppressed too); a global row keeps plain full attention."""
    rng = np.random.default_rng(47)
    n, D, r = 40, 8, 3
    q, k, v = _rand((1, 1, n, D), rng), _rand((1, 1, n, D), rng), _rand((1, 1, n, D), rng)
    gi = np.array([[2, 5, 30]], np.int32)
    lt = np.full((1, 2 * r + 1), -1e30, np.float32)
    lt[0, r] = 0.0
    o, lse, _ = oracle_mod.Problem(q, k, v, window=r, global_idx=gi, local_bias=lt).forward()
    qd, kd, vd = (x[0, 0].astype(np.float64) for x in (q, k, v))
    for i in range(n):
        if i in gi[0]:
            keys = list(range(n))
        else:
            keys = [i] + [j for j in gi[0] if abs(j - i) > r]
        s = qd[i] @ kd[keys].T / np.sqrt(D)
        m = s.max()
        w = np.exp(s - m)
        assert np.max(np.abs(o[0, 0, i] - (w @ vd[keys]) / w.sum())) <= 1e-12
        assert abs(lse[0, 0, i] - (m + np.log(w.sum()))) <= 1e-12


def test_local_bias_table_must_cover_the_window(oracle_mod):
    rng = np.random.default_rng(49)
    p = _problem(oracle_mod, rng, 1, 1, 1, 20, 4, 3, 2, 0, 0, 0)
    short = oracle_mod.Problem(p.q, p.k, p.v, window=3, dilation=2, local_bias=_local_table(rng, 1, 5))
    with pytest.raises(RuntimeError):
        short.forward()
    # a radius past n - 1 is never needed
    big = oracle_mod.Problem(p.q[:, :, :4], p.k[:, :, :4], p.v[:, :, :4], window=50,
                             local_bias=_local_table(rng, 1, 3))
    big.forward()


def test_expand_local_bias_columns(oracle_mod):
    table = np.arange(2 * 32, dtype=np.float32).reshape(2, 32)
    R = 200
    out = oracle_mod.expand_local_bias(table, R)
    assert out.shape == (2, 2 * R + 1)
    # column c holds delta = c - R (memory minus query position): 0 -> bucket 0,
    # +1 -> 17 (the positive half starts at 16), -1 -> 1, |delta| >= 128 -> the last bucket
    assert out[1, R] == 32 + 0
    assert out[1, R + 1] == 32 + 17
    assert out[1, R - 1] == 32 + 1
    assert out[0, R + 7] == 16 + 7 and out[0, R + 8] == 16 + 8
    assert out[0, 0] == 15 and out[0, 2 * R] == 31


# --- BigBird random key blocks (精读笔记：Big Bird §3.2.2) ------------------------------


def _rand_blocks(rng, B, Hq, n, bs, r):
    nqb = (n + bs - 1) // bs
    return rng.integers(0, nqb, size=(B, Hq, nqb, r)).astype(np.int32)   # repeats allowed


def test_random_blocks_match_dense_bruteforce_grid(oracle_mod):
    """Per-row key sets with random blocks (repeats, overlaps with the window, globals
    and padding included) against the dense mask that adds them by block membership."""
    rng = np.random.default_rng(53)
    cases = 0
    for n in (5, 16, 29, 40):
        for r, d, g, pad, nr, bs in itertools.product((0, 1, 3), (1, 2), (0, 2), (0, 3), (1, 3),
                                                     (4, 7)):
            if rng.random() > 0.3:
                continue
            S = int(rng.integers(0, 2)) * 2
            p = _problem(oracle_mod, rng, 2, 2, 2, n, 8, r, d, 0, g, pad, S=S, kb=4, bias=bool(S))
            rb = _rand_blocks(rng, 2, 2, n, bs, nr)
            pr = oracle_mod.Problem(p.q, p.k, p.v, window=r, dilation=d, global_idx=p.global_idx,
                                    side_k=p.side_k, side_v=p.side_v, side_block=4, bias=p.bias,
                                    valid_len=p.valid_len, rand_blocks=rb, rand_block=bs)
            o, lse, _ = pr.forward()
            od, lsed = pr.dense_bruteforce()
            assert np.max(np.abs(o - od)) <= 1e-12
            _assert_close_lse(lse, lsed, 1e-12)
            cases += 1
    assert cases > 40


def test_random_block_key_list_is_the_set_union(oracle_mod):
    """K(i) = W(i) U G U (keys of the row's random blocks below V), as a set."""
    rng = np.random.default_rng(59)
    B, H, n, bs, nr, r = 2, 3, 50, 8, 3, 4
    V = 45
    gl = np.array([[3, 20], [0, 44]], np.int32)
    rb = _rand_blocks(rng, B, H, n, bs, nr)
    vl = np.array([V, V], np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(V):
                got = oracle_mod.key_list(B, H, n, b, h, i, window=r, global_idx=gl, valid_len=vl,
                                          rand_blocks=rb, rand_block=bs)
                if i in gl[b]:
                    want = set(range(V))
                else:
                    want = {j for j in range(i - r, i + r + 1) if 0 <= j < V} | set(gl[b].tolist())
                    for blk in rb[b, h, i // bs]:
                        want |= {j for j in range(blk * bs, blk * bs + bs) if j < V}
                assert got.tolist() == sorted(want)


def test_random_blocks_covering_everything_give_full_attention(oracle_mod):
    """When the random blocks of every query block cover the whole sequence, every row
    is a full-attention row (softmax over all valid keys, from torch)."""
    rng = np.random.default_rng(61)
    B, H, n, D, bs = 1, 2, 24, 8, 8
    q, k, v = (_rand((B, H, n, D), rng) for _ in range(3))
    rb = np.broadcast_to(np.arange(3, dtype=np.int32), (B, H, 3, 3)).copy()
    o, lse, cnt = oracle_mod.Problem(q, k, v, window=1, rand_blocks=rb, rand_block=bs).forward()
    s = torch.from_numpy(q).double() @ torch.from_numpy(k).double().transpose(-1, -2) / math.sqrt(D)
    ref = torch.softmax(s, -1) @ torch.from_numpy(v).double()
    assert np.max(np.abs(o - ref.numpy())) <= 1e-12
    assert np.all(cnt == n)


def test_random_blocks_zero_query_mean_over_key_set(oracle_mod):
    """q = 0: o_i is the plain mean of V over |W U G U R| keys (a cardinality check)."""
    rng = np.random.default_rng(67)
    B, H, n, D, bs, r = 1, 1, 40, 4, 8, 2
    q = np.zeros((B, H, n, D), np.float32)
    k, v = _rand((B, H, n, D), rng), _rand((B, H, n, D), rng)
    rb = _rand_blocks(rng, B, H, n, bs, 2)
    p = oracle_mod.Problem(q, k, v, window=r, rand_blocks=rb, rand_block=bs)
    o, _, cnt = p.forward()
    for i in range(n):
        keys = oracle_mod.key_list(B, H, n, 0, 0, i, window=r, rand_blocks=rb, rand_block=bs)
        assert len(keys) == cnt[0, 0, i]
        assert np.max(np.abs(o[0, 0, i] - v[0, 0, keys].astype(np.float64).mean(0))) <= 1e-12


# --- backward (gradients of softmax attention through the same key sets) ----------------


def _dense_mask(n, r, d, causal, gl, V):
    """The closed-form allowed matrix (band by dilation, causal, global rows/cols, padding)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    diff = i - j
    band = (diff % d == 0) & (((diff >= 0) & (diff <= r * d)) if causal else (np.abs(diff) <= r * d))
    isg = np.zeros(n, bool)
    if gl is not None:
        isg[gl] = True
    allow = band | isg[None, :] | isg[:, None]
    return allow & (i < V) & (j < V)


def test_backward_matches_torch_autograd_on_dense_masked_attention(oracle_mod):
    rng = np.random.default_rng(71)
    cases = 0
    for n, r, d, causal, g, pad, G in [(13, 2, 1, 0, 0, 0, 1), (20, 3, 2, 0, 2, 3, 2), (17, 4, 1, 1, 0, 2, 2),
                                       (24, 1, 3, 1, 0, 0, 1), (9, 20, 1, 0, 1, 0, 3), (30, 2, 2, 0, 3, 5, 1)]:
        B, Hkv, D = 2, 2, 8
        Hq = Hkv * G
        p = _problem(oracle_mod, rng, B, Hq, Hkv, n, D, r, d, causal, g, pad)
        dout = _rand((B, Hq, n, D), rng)
        dq, dk, dv = p.backward(dout)
        V = n - pad
        q = torch.from_numpy(p.q).double().requires_grad_()
        k = torch.from_numpy(p.k).double().requires_grad_()
        v = torch.from_numpy(p.v).double().requires_grad_()
        kk = k.repeat_interleave(G, dim=1)
        vv = v.repeat_interleave(G, dim=1)
        s = q @ kk.transpose(-1, -2) * p.scale
        outs = []
        for b in range(B):
            gl = p.global_idx[b] if p.global_idx is not None else None
            allow = torch.from_numpy(_dense_mask(n, r, d, causal, gl, V))
            sb = s[b].masked_fill(~allow, float("-inf"))
            w = torch.softmax(sb, -1).nan_to_num(0.0)          # padded rows: no keys, o = 0
            outs.append(w @ vv[b])
        o = torch.stack(outs)
        (o * torch.from_numpy(dout).double()).sum().backward()
        assert np.max(np.abs(dq - q.grad.numpy())) <= 1e-12
        assert np.max(np.abs(dk - k.grad.numpy())) <= 1e-12
        assert np.max(np.abs(dv - v.grad.numpy())) <= 1e-12
        cases += 1
    assert cases == 6


def test_backward_finite_differences(oracle_mod):
    """Central differences of L = sum(dout * o) through the oracle's forward, with the
    local bias and random blocks in play (the terms torch does not see above)."""
    rng = np.random.default_rng(73)
    B, H, n, D, r, bs = 1, 2, 20, 4, 2, 4
    q, k, v = (_rand((B, H, n, D), rng) for _ in range(3))
    dout = _rand((B, H, n, D), rng)
    gl = np.array([[5, 17]], np.int32)
    lt = _local_table(rng, H, r)
    rb = _rand_blocks(rng, B, H, n, bs, 2)
    kw = dict(window=r, global_idx=gl, local_bias=lt, rand_blocks=rb, rand_block=bs)
    dq, dk, dv = oracle_mod.Problem(q, k, v, **kw).backward(dout)

    def loss(qq, kk, vv):
        o, _, _ = oracle_mod.Problem(qq, kk, vv, **kw).forward()
        return float((o * dout.astype(np.float64)).sum())

    h = 2.0 ** -10
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += np.float32(h)
            minus[idx] -= np.float32(h)
            step = float(plus[idx]) - float(minus[idx])
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            a_p = [plus if x is arr else x for x in args]
            a_m = [minus if x is arr else x for x in args]
            fd = (loss(*a_p) - loss(*a_m)) / step
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx, fd, grad[idx])


def test_backward_with_side_keys_matches_torch_autograd(oracle_mod):
    """Side keys (and their additive bias) appended to every valid row: the oracle's
    gradients for q, k, v, side_k and side_v equal torch autograd through a dense
    masked attention over [K; side_k] and [V; side_v] (globals, padding, GQA, causal
    and dilation in play)."""
    rng = np.random.default_rng(79)
    for n, r, d, causal, g, pad, G, S, kb in [(16, 2, 1, 0, 0, 0, 1, 4, 4), (21, 3, 2, 0, 2, 3, 2, 5, 4),
                                              (18, 4, 1, 1, 0, 2, 2, 3, 6), (12, 1, 1, 0, 1, 0, 1, 6, 2)]:
        B, Hkv, D = 2, 2, 8
        Hq = Hkv * G
        p = _problem(oracle_mod, rng, B, Hq, Hkv, n, D, r, d, causal, g, pad, S=S, kb=kb, bias=True)
        dout = _rand((B, Hq, n, D), rng)
        dq, dk, dv, dsk, dsv = p.backward(dout)
        V = n - pad
        nblk = -(-n // kb)
        q = torch.from_numpy(p.q).double().requires_grad_()
        k = torch.from_numpy(p.k).double().requires_grad_()
        v = torch.from_numpy(p.v).double().requires_grad_()
        sk = torch.from_numpy(p.side_k).double().requires_grad_()
        sv = torch.from_numpy(p.side_v).double().requires_grad_()
        kk = torch.cat([k, sk], 2).repeat_interleave(G, dim=1)
        vv = torch.cat([v, sv], 2).repeat_interleave(G, dim=1)
        s = q @ kk.transpose(-1, -2) * p.scale
        # side-key bias: row i, side key sigma -> table column sigma - floor(i / kb) + nblk - 1
        col = (torch.arange(S)[None, :] - (torch.arange(n) // kb)[:, None]) + nblk - 1
        sb_bias = torch.from_numpy(p.bias).double()[:, col]               # [Hq, n, S]
        bias_full = torch.cat([torch.zeros(Hq, n, n, dtype=torch.float64), sb_bias], -1)
        outs = []
        for b in range(B):
            gl = p.global_idx[b] if p.global_idx is not None else None
            allow = np.concatenate([_dense_mask(n, r, d, causal, gl, V),
                                    np.repeat((np.arange(n) < V)[:, None], S, 1)], 1)
            sc = (s[b] + bias_full).masked_fill(~torch.from_numpy(allow), float("-inf"))
            w = torch.softmax(sc, -1).nan_to_num(0.0)
            outs.append(w @ vv[b])
        o = torch.stack(outs)
        (o * torch.from_numpy(dout).double()).sum().backward()
        for mine, ref in ((dq, q), (dk, k), (dv, v), (dsk, sk), (dsv, sv)):
            assert np.max(np.abs(mine - ref.grad.numpy())) <= 1e-12


def test_backward_with_side_keys_finite_differences(oracle_mod):
    """Central differences of L = sum(dout * o) through the oracle's forward, for every
    input the side-key backward differentiates (side keys, bias and globals in play)."""
    rng = np.random.default_rng(83)
    p = _problem(oracle_mod, rng, 1, 2, 1, 18, 4, 2, 1, 0, 2, 2, S=4, kb=4, bias=True)
    dout = _rand((1, 2, 18, 4), rng)
    grads = p.backward(dout)
    inputs = [p.q, p.k, p.v, p.side_k, p.side_v]
    kw = dict(window=p.window, dilation=p.dilation, global_idx=p.global_idx, side_block=p.side_block,
              bias=p.bias, valid_len=p.valid_len)

    def loss(arrs):
        o, _, _ = oracle_mod.Problem(arrs[0], arrs[1], arrs[2], side_k=arrs[3], side_v=arrs[4],
                                     **kw).forward()
        return float((o * dout.astype(np.float64)).sum())

    h = 2.0 ** -10
    for a_i, (arr, grad) in enumerate(zip(inputs, grads)):
        for _ in range(5):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = [x.copy() for x in inputs], [x.copy() for x in inputs]
            plus[a_i][idx] += np.float32(h)
            minus[a_i][idx] -= np.float32(h)
            step = float(plus[a_i][idx]) - float(minus[a_i][idx])
            fd = (loss(plus) - loss(minus)) / step
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (a_i, idx, fd, grad[idx])
