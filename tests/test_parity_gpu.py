"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

* every workload at a reduced size (several tiles and a ragged tail), full output;
* every workload at full size on sampled rows, plus whole-output properties;
* edge cases: r = 0, window covering the sequence, ragged n, one valid row, g > 128,
  side counts that are not a tile multiple, causal + dilation, GQA;
* exact support: with V = identity rows the output row is the weight row, so every
  key outside K(i) must come back exactly 0 and every key inside it positive.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from sliding_window_global_b200 import workloads
from tests import helpers

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_workload(w, seed_inp=None):
    inp = helpers.host_problem(w, seed_inp)
    dinp = helpers.to_dev(inp)
    out, lse, plan = helpers.run_gpu(w, dinp)
    assert plan.check() == 0
    ref_o, ref_l, _ = helpers.oracle_problem(w, inp).forward()
    return helpers.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, w.dtype, w.name)


@pytest.mark.parametrize("name", list(workloads.SMALL))
def test_small_workloads_full_output(name):
    _need_gpu()
    _check_workload(workloads.SMALL[name])


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_full_size_sampled_rows(name):
    _need_gpu()
    w = workloads.WORKLOADS[name]
    inp = helpers.host_problem(w)
    dinp = helpers.to_dev(inp)
    out, lse, plan = helpers.run_gpu(w, dinp)
    assert plan.check() == 0
    rows = helpers.sample_rows(w, inp, 1500 if w.seq_len * w.q_heads < 10**6 else 600)
    ref_o, ref_l, _ = helpers.oracle_problem(w, inp).forward(rows)
    o = out.reshape(-1, w.head_dim)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    l = lse.reshape(-1)[torch.from_numpy(rows).cuda()].cpu().numpy()
    helpers.compare(o, l, ref_o, ref_l, w.dtype, name)
    # whole-output properties at full size
    assert bool(torch.isfinite(out.float()).all())
    if w.padding:
        V = w.valid_len
        assert bool((out[:, :, V:] == 0).all())
        assert bool(torch.isneginf(lse[:, :, V:]).all())
        assert bool(torch.isfinite(lse[:, :, :V]).all())


def _small(base, **kw):
    return dataclasses.replace(workloads.SMALL[base], **kw)


EDGE = [
    ("r0", _small("longformer_base", window=(0,) * 4, num_global=0, global_mode="none")),
    ("full_window", _small("longformer_base", window=(5000,) * 4, num_global=0, global_mode="none")),
    ("full_window_causal", _small("swan_swa", window=(5000,) * 8)),
    ("one_valid_row", _small("longformer_base", padding=999, num_global=1)),
    ("many_globals", _small("dilated", num_global=150, seq_len=700)),
    ("globals_only_pad", _small("longformer_base", padding=500)),
    ("side_not_tile_multiple", _small("longt5_tglobal", seq_len=1600, side_block=16)),
    ("side_block_7", _small("longt5_tglobal", seq_len=777, side_block=7, padding=20)),
    ("causal_dilated", _small("swan_swa", dilation=(1, 2, 3, 4, 1, 2, 3, 4), window=(40,) * 8)),
    ("gqa_d64", _small("swan_swa", head_dim=64, q_heads=6, kv_heads=2, window=(130,) * 6,
                       dilation=(1,) * 6)),
    ("noncausal_d128", _small("swan_swa", causal=False, window=(200,) * 8)),
    ("batch3_tiny_n", _small("dilated", batch=3, seq_len=77, window=(9,) * 4, num_global=3)),
    ("n_one", _small("longformer_base", seq_len=1, padding=0, num_global=0, global_mode="none")),
    # GQA head pairs on one KV head (a unit = the same rows of two heads)
    ("pair_dilated_globals", _small("swan_swa", causal=False, window=(60,) * 8,
                                    dilation=(1, 1, 2, 2, 3, 3, 1, 1), num_global=6,
                                    global_mode="random", padding=41)),
    ("pair_side_no_bias", _small("longt5_tglobal", q_heads=4, kv_heads=2, window=(127,) * 4,
                                 dilation=(1,) * 4, side_bias=False)),
    ("pair_d64_ragged", _small("swan_swa", head_dim=64, seq_len=333, window=(90,) * 8)),
    ("fp32_gqa_side", dataclasses.replace(workloads.SMALL["longt5_tglobal"], dtype="fp32",
                                          q_heads=4, kv_heads=2, window=(20,) * 4,
                                          dilation=(1, 2, 1, 2), seq_len=300)),
    ("fp32_globals_pad", dataclasses.replace(workloads.SMALL["longformer_base"], dtype="fp32",
                                             seq_len=400, padding=33, num_global=7)),
    # local relative-position bias on window keys (LongT5 local attention)
    ("local_globals", _small("longformer_base", local_bias=True)),
    ("local_tglobal_side_bias", _small("longt5_tglobal", local_bias=True, padding=30)),
    ("local_dilated_globals", _small("dilated", local_bias=True)),
    ("local_causal_gqa_d128", _small("swan_swa", local_bias=True)),
    ("local_window_covers_seq", _small("longformer_base", seq_len=300, window=(5000,) * 4,
                                       num_global=0, global_mode="none", padding=0,
                                       local_bias=True)),
    ("local_r766_d64", _small("longt5_local", seq_len=2000, window=(766,) * 3, padding=0)),
    ("local_d128_noncausal", _small("swan_swa", causal=False, window=(200, 1, 0, 200, 37, 37, 5, 9),
                                    local_bias=True)),
    ("local_fp32_dilated", dataclasses.replace(workloads.SMALL["longt5_local"], dtype="fp32",
                                               seq_len=500, window=(40,) * 3, dilation=(1, 2, 3))),
]


@pytest.mark.parametrize("name,w", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(name, w):
    _need_gpu()
    _check_workload(w)


# Key rows scaled up so that later key tiles score far above the running max of the
# earlier ones: x30 makes some rows jump by more than 2^64 (log2 units) within a
# unit, x3 by a few powers of two, x0.01 shrinks a block.  The separate-P kernels
# (D = 64) take a tile's exponentials against the running max and find the tile max
# alongside them, redoing a tile that jumps past the guard; D = 128 takes the max
# first.  Both must still match the oracle.
JUMPS = [
    ("d64_window", _small("longt5_local", local_bias=False, window=(300,) * 3, padding=0)),
    ("d64_local_bias", _small("longt5_local", window=(300,) * 3)),
    ("d64_side_keys", _small("longt5_tglobal")),
    ("d64_globals_padding", _small("longformer_base")),
    ("d128_causal_gqa", _small("swan_swa")),
]


@pytest.mark.parametrize("name,w", JUMPS, ids=[e[0] for e in JUMPS])
def test_scores_jumping_between_key_tiles(name, w):
    _need_gpu()
    inp = workloads.make_inputs(w)
    k = inp["k"].float()
    n = k.shape[2]
    for lo, hi, f in ((n * 3 // 8, n * 3 // 8 + 120, 30.0), (n * 5 // 8, n * 5 // 8 + 100, 3.0),
                      (n * 7 // 8, n * 7 // 8 + 60, 0.01)):
        k[:, :, lo:hi] *= f
    inp["k"] = k.to(w.torch_dtype)
    _check_workload(w, inp)


SUPPORT = [
    # (n, D, r, dilation, causal, g, padding)
    (128, 128, 5, 1, False, 0, 0),
    (128, 128, 7, 2, False, 3, 9),
    (120, 128, 4, 3, True, 0, 5),
    (128, 128, 40, 1, True, 0, 0),
    (64, 64, 3, 1, False, 2, 0),
    (64, 64, 2, 2, False, 0, 7),
    (100, 128, 0, 1, False, 4, 0),
]


@pytest.mark.parametrize("n,D,r,d,causal,g,pad", SUPPORT)
def test_support_exact(n, D, r, d, causal, g, pad):
    """V = identity rows: o_i[j] = weight of key j -> zero exactly off K(i), > 0 on it."""
    _need_gpu()
    from sliding_window_global_b200 import Plan
    gen = torch.Generator("cpu").manual_seed(n * 1000 + r * 10 + d)
    B, H = 2, 2
    q = torch.randn((B, H, n, D), generator=gen).to(torch.bfloat16)
    k = torch.randn((B, H, n, D), generator=gen).to(torch.bfloat16)
    v = torch.zeros((B, H, n, D))
    v[:, :, torch.arange(n), torch.arange(n)] = 1.0
    v = v.to(torch.bfloat16)
    V = n - pad
    gl = None
    if g:
        gl = torch.stack([torch.sort(torch.randperm(V, generator=gen)[:g]).values for _ in range(B)])
        gl = gl.to(torch.int32)
    vl = torch.full((B,), V, dtype=torch.int32) if pad else None
    plan = Plan(B, n, H, H, D, torch.bfloat16, max_global=g)
    out, _ = plan.forward(q.cuda(), k.cuda(), v.cuda(), window=r, dilation=d, causal=causal,
                          global_idx=None if gl is None else gl.cuda(),
                          valid_len=None if vl is None else vl.cuda())
    o = out.float().cpu().numpy()
    for b in range(B):
        for h in range(H):
            for i in range(n):
                keys = oracle.key_list(B, H, n, b, h, i, window=r, dilation=d, causal=causal,
                                       global_idx=None if gl is None else gl.numpy(),
                                       valid_len=None if vl is None else vl.numpy())
                inside = np.zeros(n, bool)
                inside[keys] = True
                row = o[b, h, i, :n]
                assert np.all(row[~inside] == 0.0), (b, h, i)
                assert np.all(row[inside] > 0.0), (b, h, i)


RANDOM = [
    # BigBird random key blocks on top of windows, globals, padding, GQA and D = 128
    ("rand_globals_pad", _small("bigbird_itc")),
    ("rand_no_globals", _small("bigbird_itc", num_global=0, global_mode="none", padding=0)),
    ("rand_gqa_pairs_d128", _small("swan_swa", causal=False, window=(150,) * 8, num_rand=2)),
    ("rand_local_bias", _small("bigbird_itc", local_bias=True, num_rand=4)),
    ("rand_window_covers_seq", _small("bigbird_itc", window=(3000,) * 4, num_global=0,
                                      global_mode="none")),
    ("rand_tiny_seq", _small("bigbird_itc", seq_len=100, num_global=3, padding=7)),
    # windows on both sides of r = 64, where a global key that a random block of the
    # tile already counts switches from a per-key test to the one-compare mask
    ("rand_globals_windows_around_64", _small("bigbird_itc", window=(40, 63, 64, 100))),
    ("rand_fp32", dataclasses.replace(workloads.SMALL["bigbird_itc"], dtype="fp32", seq_len=500,
                                      num_global=5)),
]


@pytest.mark.parametrize("name,w", RANDOM, ids=[e[0] for e in RANDOM])
def test_random_blocks(name, w):
    _need_gpu()
    _check_workload(w)


@pytest.mark.parametrize("window", [None, (40, 63, 64, 100)], ids=["r100", "r40_63_64_100"])
def test_random_blocks_with_repeats_and_overlaps(window):
    """Hand-written draws: a block repeated in the list, the query block itself, its
    neighbours (overlapping the window), a block holding global keys and the block
    holding the padded tail -- each key must still count once."""
    _need_gpu()
    w = _small("bigbird_itc", seq_len=1000, num_rand=5, padding=60)
    if window is not None:
        w = dataclasses.replace(w, window=window)
    inp = workloads.make_inputs(w)
    nqb = (w.seq_len + 127) // 128
    rb = torch.empty((1, w.q_heads, nqb, 5), dtype=torch.int32)
    for h in range(w.q_heads):
        for qb in range(nqb):
            rb[0, h, qb] = torch.tensor([qb, (qb + 3) % nqb, max(qb - 1, 0), 0, nqb - 1])
            if h % 2:
                rb[0, h, qb, 1] = rb[0, h, qb, 0]          # a repeated block
    inp["rand_blocks"] = rb
    _check_workload(w, inp)


def test_random_blocks_unsupported_with_dilation_or_causal():
    _need_gpu()
    from sliding_window_global_b200 import SwaError
    for w in (_small("bigbird_itc", dilation=(1, 2, 1, 1)),
              _small("bigbird_itc", causal=True, num_global=0, global_mode="none")):
        dinp = helpers.to_dev(helpers.host_problem(w))
        with pytest.raises(SwaError) as e:
            helpers.run_gpu(w, dinp)
        assert e.value.status == 2


def test_local_bias_window_beyond_staging_limit_is_unsupported():
    """bf16 kernels stage the local-bias row of a unit: min(r, ceil(n/d)) <= 766."""
    _need_gpu()
    from sliding_window_global_b200 import SwaError
    w = _small("longt5_local", seq_len=2000, window=(767,) * 3, padding=0)
    dinp = helpers.to_dev(helpers.host_problem(w))
    with pytest.raises(SwaError) as e:
        helpers.run_gpu(w, dinp)
    assert e.value.status == 2
    # the same window with dilation 3 spans ceil(2000 / 3) = 667 class rows: supported
    w = _small("longt5_local", seq_len=2000, window=(767,) * 3, dilation=(3,) * 3, padding=0)
    _check_workload(w)


def test_local_bias_table_too_small_is_invalid():
    _need_gpu()
    from sliding_window_global_b200 import SwaError
    w = workloads.SMALL["longt5_local"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    dinp["local_bias"] = dinp["local_bias"][:, 1:-1].contiguous()     # radius 126 < 127
    with pytest.raises(SwaError) as e:
        helpers.run_gpu(w, dinp)
    assert e.value.status == 1


def test_side_aggregate_matches_oracle():
    _need_gpu()
    from sliding_window_global_b200 import side_aggregate
    gen = torch.Generator("cpu").manual_seed(5)
    x = torch.randn((2, 3, 1000, 64), generator=gen).to(torch.bfloat16)
    vl = torch.tensor([1000, 937], dtype=torch.int32)
    got = side_aggregate(x.cuda(), 16, vl.cuda()).float().cpu().numpy()
    ref = oracle.side_aggregate(x, 16, vl.numpy())
    # the device rounds an fp32 mean to bf16: within one bf16 ulp of the fp64 mean
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(got - ref) <= ulp)


@pytest.mark.parametrize("padding,seq_len", [(0, 1024), (45, 1000)], ids=["plain", "padded_ragged"])
def test_side_keys_built_from_kv(padding, seq_len):
    """side_from_kv: the band kernel builds the Transient-Global side keys / values in
    its prologue (one launch in all) -- bit-identical to passing swa_side_aggregate's
    block means, and within tolerance of the oracle's block means -> attention.  The
    ragged case has a trailing partial block (n % 16 = 8) and padded tokens."""
    _need_gpu()
    import dataclasses
    from sliding_window_global_b200 import Plan, side_aggregate
    w = dataclasses.replace(workloads.SMALL["longt5_tglobal"], seq_len=seq_len, padding=padding,
                            name=f"tglobal_fused_{seq_len}")
    inp = helpers.host_problem(w)
    dinp = helpers.to_dev(inp)
    plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, torch.bfloat16,
                num_side=w.num_side, side_block=w.side_block)
    kw = dict(window=dinp["window"], dilation=dinp["dilation"], bias=dinp["bias"],
              valid_len=dinp["valid_len"])
    out_f, lse_f = plan.forward(dinp["q"], dinp["k"], dinp["v"], side_from_kv=True, **kw)
    assert plan.last_launches == 1                    # the band kernel builds them in its prologue
    sk = side_aggregate(dinp["k"], w.side_block, dinp["valid_len"])
    sv = side_aggregate(dinp["v"], w.side_block, dinp["valid_len"])
    out_x, lse_x = plan.forward(dinp["q"], dinp["k"], dinp["v"], side_k=sk, side_v=sv, **kw)
    torch.cuda.synchronize()
    assert plan.check() == 0
    assert torch.equal(out_f, out_x) and torch.equal(lse_f, lse_x)
    ref_o, ref_l, _ = helpers.oracle_problem(w, inp).forward()
    helpers.compare(out_f.float().cpu().numpy(), lse_f.cpu().numpy(), ref_o, ref_l, "bf16",
                    "side_from_kv")


def test_side_from_kv_argument_checks():
    _need_gpu()
    from sliding_window_global_b200 import Plan, SwaError
    w = workloads.SMALL["longt5_tglobal"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, torch.bfloat16,
                num_side=w.num_side, side_block=w.side_block)
    with pytest.raises(SwaError) as e:          # side keys passed as well
        plan.forward(dinp["q"], dinp["k"], dinp["v"], window=dinp["window"], side_k=dinp["side_k"],
                     side_v=dinp["side_v"], side_from_kv=True)
    assert e.value.status == 1
    plan2 = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, torch.bfloat16,
                 num_side=w.num_side - 1, side_block=w.side_block)   # S != n / block
    with pytest.raises(SwaError) as e:
        plan2.forward(dinp["q"], dinp["k"], dinp["v"], window=dinp["window"], side_from_kv=True)
    assert e.value.status == 1


def test_debug_mode_flags_bad_global_index():
    """A global index list that is not strictly increasing inside [0, valid_len) is a
    precondition failure.  Debug mode checks it on the device and reads the result
    back before any kernel that indexes with global_idx is enqueued: the status is
    SWA_ERR_DEVICE_CHECK, only the check kernel ran, and out is untouched."""
    _need_gpu()
    from sliding_window_global_b200 import Plan, SwaError
    w = workloads.SMALL["longformer_base"]
    inp = helpers.to_dev(helpers.host_problem(w))
    n, V = w.seq_len, w.valid_len
    plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, torch.bfloat16,
                max_global=4, debug=True)
    out = torch.full((w.batch, w.q_heads, n, w.head_dim), 7.0, dtype=torch.bfloat16, device="cuda")
    for bad in ([3, 2, 5, 9],            # not increasing
                [2, 3, 5, n + 40],       # beyond the sequence
                [2, 3, 5, V],            # a padded position
                [-1, 3, 5, 9]):          # negative
        idx = torch.tensor([bad], dtype=torch.int32, device="cuda")
        with pytest.raises(SwaError) as e:
            plan.forward(inp["q"], inp["k"], inp["v"], window=inp["window"], global_idx=idx,
                         valid_len=inp["valid_len"], out=out)
        assert e.value.status == 6, bad
        assert plan.last_launches == 1, bad          # the check kernel alone
        assert plan.check() == 0                     # the word was read and cleared
        torch.cuda.synchronize()
        assert bool((out == 7.0).all()), bad
    good = torch.tensor([[2, 3, 5, 9]], dtype=torch.int32, device="cuda")
    plan.forward(inp["q"], inp["k"], inp["v"], window=inp["window"], global_idx=good,
                 valid_len=inp["valid_len"])
    assert plan.check() == 0


def test_debug_mode_flags_bad_random_block():
    """Random key blocks outside [0, ceil(n/128)) fail the debug check the same way."""
    _need_gpu()
    from sliding_window_global_b200 import Plan, SwaError
    w = workloads.SMALL["bigbird_itc"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    plan = Plan(w.batch, w.seq_len, w.q_heads, w.kv_heads, w.head_dim, torch.bfloat16,
                max_global=w.num_global, debug=True)
    kw = dict(window=dinp["window"], global_idx=dinp["global_idx"], valid_len=dinp["valid_len"])
    plan.forward(dinp["q"], dinp["k"], dinp["v"], rand_blocks=dinp["rand_blocks"], **kw)
    assert plan.check() == 0
    nqb = (w.seq_len + 127) // 128
    for val in (nqb, -1):
        rb = dinp["rand_blocks"].clone()
        rb[0, 1, 2, 0] = val
        with pytest.raises(SwaError) as e:
            plan.forward(dinp["q"], dinp["k"], dinp["v"], rand_blocks=rb, **kw)
        assert e.value.status == 6 and plan.last_launches == 1


def test_repeat_calls_deterministic_and_launch_count():
    _need_gpu()
    w = workloads.SMALL["dilated"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    o1, l1, plan = helpers.run_gpu(w, dinp)
    o2, l2, _ = helpers.run_gpu(w, dinp, plan=plan)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert plan.last_launches == 4   # gather (q, k, v in one launch), band, global rows, merge


def test_bounded_wait_expires_into_a_status_and_the_context_survives():
    """Failure path: a wait on a barrier nothing signals gives up after its limit,
    the error word reports SWA_ERR_TIMEOUT once, and the next forward is unaffected."""
    _need_gpu()
    import time
    w = workloads.SMALL["longformer_base"]
    dinp = helpers.to_dev(helpers.host_problem(w))
    out0, lse0, plan = helpers.run_gpu(w, dinp)
    assert plan.check() == 0
    t0 = time.perf_counter()
    plan.selftest_wait_timeout(50_000_000)          # 50 ms
    assert plan.check() == 5                        # SWA_ERR_TIMEOUT
    assert time.perf_counter() - t0 >= 0.04
    assert plan.check() == 0                        # the word was cleared
    out1, lse1, _ = helpers.run_gpu(w, dinp, plan=plan)
    assert plan.check() == 0
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
