"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: library
dtype conversions, the OFP8 code table, a hand-worked example, a pure-Python
brute force, closed forms and invariants of the definition. The last test
plants mistakes in the oracle and shows each one trips a pin.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.brute import mla_decode_brute
from mla_paged_decode_04_b200.inputs import make_inputs_custom

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- decoders

def test_e4m3_decoder_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_values("fp8", codes.numpy())
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


@pytest.mark.parametrize("dtype,tdt", [("bf16", torch.bfloat16), ("fp16", torch.float16)])
def test_16bit_decoders_match_torch_all_codes(dtype, tdt):
    codes = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = codes.view(tdt).to(torch.float64).numpy()
    got = oracle.decode_values(dtype, codes.view(torch.uint8).numpy())
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_e4m3_golden_codes():
    path = os.path.join(GOLDEN, "e4m3fn_codes.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    codes = np.array([int(c, 16) for c, _ in rows], dtype=np.uint8)
    want = np.array([float(v) for _, v in rows])
    got = oracle.decode_values("fp8", codes)
    for c, w, g in zip(codes, want, got):
        if math.isnan(w):
            assert math.isnan(g), hex(c)
        else:
            assert g == w and math.copysign(1, g) == math.copysign(1, w), hex(c)


# ---------------------------------------------------------------- helpers

def _values(t, scale=1.0):
    """Element values through torch's conversion (independent of the oracle decoders)."""
    return t.to(torch.float64).numpy() * scale


def _decode(inp, **kw):
    return oracle.mla_decode(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                             inp.softmax_scale, dtype=inp.dtype, q_scale=inp.q_scale,
                             kv_scale=inp.kv_scale, **kw)


def _keys(inp, b):
    """Visible cache rows of entry b gathered by the test itself, [N_b, 576] float64."""
    n = int(inp.seq_lens[b])
    cache = _values(inp.kv_cache, inp.kv_scale)
    idx = [int(inp.block_tables[b, j // 64]) for j in range(n)]
    return np.stack([cache[idx[j], j % 64] for j in range(n)]) if n else np.zeros((0, 576))


# ---------------------------------------------------------------- pins
# Each pin returns the largest deviation it saw so the mutation test can reuse it.

def pin_two_key_example(mutation="none"):
    path = os.path.join(GOLDEN, "two_key_example.txt")
    vals = dict(l.split() for l in open(path) if l.strip() and not l.startswith("#"))
    errs = []
    for dtype, tdt in [("bf16", torch.bfloat16), ("fp16", torch.float16),
                       ("fp8", torch.float8_e4m3fn)]:
        q = torch.zeros(1, 1, 1, 576)
        q[0, 0, 0, 0] = 1
        cache = torch.zeros(1, 64, 576)
        cache[0, 0, 1] = 4
        cache[0, 1, 0] = 1
        cache[0, 1, 2] = 8
        bt = torch.zeros(1, 1, dtype=torch.int32)
        sl = torch.tensor([2], dtype=torch.int32)
        scale = math.log(float(vals["softmax_scale_ln"]))
        out, lse = oracle.mla_decode(q.to(tdt), cache.to(tdt), bt, sl, scale, dtype=dtype,
                                     mutation=mutation)
        want = np.zeros(512)
        want[0], want[1], want[2] = (float(vals[f"out_{i}"]) for i in range(3))
        errs.append(np.abs(out[0] - want).max())
        errs.append(abs(lse[0] - math.log(float(vals["lse_ln"]))))
    return max(errs)


def pin_brute_force(mutation="none"):
    worst = 0.0
    cases = [(2, 3, 2, "bf16", [130, 5]), (1, 4, 3, "fp16", [199]), (2, 2, 4, "fp8", [70, 2]),
             (1, 1, 2, "bf16", [64])]
    for i, (B, T, H, dt, sl) in enumerate(cases):
        inp = make_inputs_custom(B, T, H, dt, sl, seed=10 + i, pool=1.5)
        out, lse = _decode(inp, mutation=mutation)
        bo, bl = mla_decode_brute(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                                  inp.softmax_scale, inp.q_scale, inp.kv_scale)
        bo, bl = np.array(bo), np.array(bl)
        fin = np.isfinite(bl)
        if not np.array_equal(fin, np.isfinite(lse)):
            return math.inf
        worst = max(worst, np.abs(out - bo).max(), np.abs(lse[fin] - bl[fin]).max(initial=0))
    return worst


def pin_zero_query(mutation="none"):
    inp = make_inputs_custom(2, 3, 2, "bf16", [100, 70], seed=3, pool=2.0)
    inp.q.zero_()
    out, lse = _decode(inp, mutation=mutation)
    worst = 0.0
    T, H = 3, 2
    for b in range(2):
        K = _keys(inp, b)
        for t in range(T):
            n = int(inp.seq_lens[b]) - T + t + 1
            for h in range(H):
                r = (b * T + t) * H + h
                worst = max(worst, np.abs(out[r] - K[:n, :512].mean(axis=0)).max(),
                            abs(lse[r] - math.log(n)))
    return worst


def pin_single_and_two_keys(mutation="none"):
    # seq_len 2 with q_len 2: token 0 sees one key, token 1 sees two.
    inp = make_inputs_custom(1, 2, 3, "fp16", [2], seed=4)
    out, lse = _decode(inp, mutation=mutation)
    K = _keys(inp, 0)
    qv = _values(inp.q)[0]
    worst = 0.0
    for h in range(3):
        s0 = inp.softmax_scale * float(np.dot(qv[0, h], K[0]))
        worst = max(worst, np.abs(out[h] - K[0, :512]).max(), abs(lse[h] - s0))
        s = inp.softmax_scale * (K[:2] @ qv[1, h])
        L = np.logaddexp(s[0], s[1])
        want = (1 / (1 + np.exp(s[1] - s[0]))) * K[0, :512] + (1 / (1 + np.exp(s[0] - s[1]))) * K[1, :512]
        worst = max(worst, np.abs(out[3 + h] - want).max(), abs(lse[3 + h] - L))
    return worst


def pin_one_hot(mutation="none"):
    inp = make_inputs_custom(1, 1, 1, "bf16", [150], seed=5, kv_std=0.01)
    # plant key 77 parallel to q with a large score
    j = 77
    page = int(inp.block_tables[0, j // 64])
    q = torch.zeros(576)
    q[3], q[540] = 1.0, 1.0
    inp.q[0, 0, 0] = q.to(torch.bfloat16)
    inp.kv_cache[page, j % 64] = (q * 2000.0).to(torch.bfloat16)
    inp.kv_cache[page, j % 64, 10] = 5.0
    out, lse = _decode(inp, mutation=mutation)
    want = _values(inp.kv_cache)[page, j % 64, :512]
    return np.abs(out[0] - want).max()


def pin_split_merge(mutation="none"):
    inp = make_inputs_custom(2, 4, 2, "fp8", [300, 131], seed=6, pool=2.0)
    full_o, full_l = _decode(inp, mutation=mutation)
    bounds = [0, 64, 65, 200, 256, 10 ** 9]
    parts = [_decode(inp, key_range=(lo, hi), mutation=mutation)
             for lo, hi in zip(bounds[:-1], bounds[1:])]
    worst = 0.0
    for r in range(full_o.shape[0]):
        o, l = oracle.lse_merge(np.stack([p[0][r] for p in parts]), [p[1][r] for p in parts])
        worst = max(worst, np.abs(o - full_o[r]).max(), abs(l - full_l[r]))
    return worst


def pin_causal(mutation="none"):
    T, H = 4, 2
    inp = make_inputs_custom(1, T, H, "bf16", [90], seed=7)
    out, lse = _decode(inp, mutation=mutation)
    worst = 0.0
    for t in range(T):
        n = 90 - T + t + 1
        single = make_inputs_custom(1, 1, H, "bf16", [n], seed=7)
        single.q = inp.q[:, t:t + 1].clone()
        single.kv_cache = inp.kv_cache
        single.block_tables = inp.block_tables
        o1, l1 = _decode(single, mutation=mutation)
        worst = max(worst, np.abs(out[t * H:(t + 1) * H] - o1).max(),
                    np.abs(lse[t * H:(t + 1) * H] - l1).max())
    # keys past token 0's limit changed: token 0's rows unchanged
    pert = make_inputs_custom(1, T, H, "bf16", [90], seed=7)
    page = int(pert.block_tables[0, 88 // 64])
    pert.kv_cache[page, 88 % 64] += 3.0
    o2, l2 = _decode(pert, mutation=mutation)
    worst = max(worst, np.abs(o2[:H] - out[:H]).max(), np.abs(l2[:H] - lse[:H]).max())
    return worst


def pin_heads_independent(mutation="none"):
    inp = make_inputs_custom(1, 2, 3, "fp16", [77], seed=8)
    out, lse = _decode(inp, mutation=mutation)
    worst = 0.0
    for h in range(3):
        one = make_inputs_custom(1, 2, 1, "fp16", [77], seed=8)
        one.q = inp.q[:, :, h:h + 1].clone()
        one.kv_cache, one.block_tables = inp.kv_cache, inp.block_tables
        o1, l1 = _decode(one, mutation=mutation)
        worst = max(worst, np.abs(out[[h, 3 + h]] - o1).max(), np.abs(lse[[h, 3 + h]] - l1).max())
    return worst


def pin_page_permutation(mutation="none"):
    inp = make_inputs_custom(2, 2, 2, "bf16", [140, 60], seed=9, pool=2.0)
    out, lse = _decode(inp, mutation=mutation)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(inp.num_pages, generator=g)
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(inp.num_pages)
    moved = make_inputs_custom(2, 2, 2, "bf16", [140, 60], seed=9, pool=2.0)
    moved.kv_cache = inp.kv_cache[perm].clone()  # new page p holds old page perm[p]
    bt = inp.block_tables.clone()
    bt[bt >= 0] = inv[bt[bt >= 0].long()].to(torch.int32)
    moved.block_tables = bt
    o2, l2 = _decode(moved, mutation=mutation)
    return max(np.abs(o2 - out).max(), np.abs(l2 - lse).max())


def pin_gaussian_closed_form(mutation="none"):
    # k ~ N(0, s^2 I), large n: LSE -> ln n + s^2 scale^2 |q|^2 / 2 and
    # out -> s^2 scale q[0:512] (exponential tilting of a Gaussian).
    sigma, n = 0.5, 20000
    inp = make_inputs_custom(1, 1, 4, "fp16", [n], seed=11, q_std=1.0, kv_std=sigma)
    out, lse = _decode(inp, mutation=mutation)
    qv = _values(inp.q)[0, 0]
    worst = 0.0
    for h in range(4):
        qq = qv[h]
        tau2 = (sigma * inp.softmax_scale) ** 2 * float(qq @ qq)
        lse_want = math.log(n) + tau2 / 2
        out_want = sigma ** 2 * inp.softmax_scale * qq[:512]
        # n_eff = n / exp(tau2); fluctuations are O(1/sqrt(n_eff))
        tol = 6.0 / math.sqrt(n / math.exp(tau2))
        worst = max(worst, abs(lse[h] - lse_want) / tol,
                    np.sqrt(np.mean((out[h] - out_want) ** 2)) / (sigma * tol))
    return worst  # in units of the tolerance: <= 1 passes


PINS = [
    ("two_key_example", pin_two_key_example, 1e-12),
    ("brute_force", pin_brute_force, 1e-12),
    ("zero_query", pin_zero_query, 1e-12),
    ("single_two_keys", pin_single_and_two_keys, 1e-12),
    ("one_hot", pin_one_hot, 1e-12),
    ("split_merge", pin_split_merge, 1e-12),
    ("causal", pin_causal, 1e-12),
    ("heads", pin_heads_independent, 1e-12),
    ("page_perm", pin_page_permutation, 0.0),
    ("gaussian", pin_gaussian_closed_form, 1.0),
]


@pytest.mark.parametrize("name,fn,tol", PINS, ids=[p[0] for p in PINS])
def test_pin(name, fn, tol):
    err = fn()
    assert err <= tol, f"{name}: {err}"


def test_empty_rows_and_entries():
    # seq_len < q_len: early tokens see nothing; seq_len 0: nothing at all.
    inp = make_inputs_custom(2, 4, 2, "bf16", [2, 0], seed=12, max_pages=1)
    out, lse = _decode(inp)
    T, H = 4, 2
    for b in range(2):
        for t in range(T):
            n = int(inp.seq_lens[b]) - T + t + 1
            rows = [(b * T + t) * H + h for h in range(H)]
            if n <= 0:
                assert np.all(out[rows] == 0) and np.all(np.isneginf(lse[rows]))
            else:
                assert np.all(np.isfinite(lse[rows]))


def test_bad_page_is_an_error():
    inp = make_inputs_custom(1, 1, 1, "bf16", [10], seed=13)
    inp.block_tables[0, 0] = inp.num_pages
    with pytest.raises(ValueError):
        _decode(inp)


def test_row_subset_matches_full():
    inp = make_inputs_custom(2, 2, 3, "fp8", [100, 65], seed=14, pool=2.0)
    out, lse = _decode(inp)
    rows = [11, 0, 7, 3]
    o2, l2 = _decode(inp, rows=rows)
    assert np.array_equal(o2, out[rows]) and np.array_equal(l2, lse[rows])


@pytest.mark.parametrize("mutation", [m for m in oracle.MUTATIONS if m != "none"])
def test_planted_mistakes_are_caught(mutation):
    """Every planted oracle mistake makes at least one pin fail."""
    caught = []
    for name, fn, tol in PINS:
        err = fn(mutation)
        if not (err <= tol):
            caught.append(name)
    assert caught, f"mutation {mutation} passed every pin"


# ---------------------------------------------------------------- sliding window
# A window W > 0 limits a row with n visible keys to keys n - W .. n - 1
# (a decode option the TokenSpeed MLA article lists among its tests, section 六).

@pytest.mark.parametrize("window", [1, 3, 64, 70])
def test_window_matches_the_brute_force_decode(window):
    worst = 0.0
    cases = [(2, 3, 2, "bf16", [130, 5]), (1, 4, 3, "fp16", [199]), (2, 2, 4, "fp8", [70, 2])]
    for i, (B, T, H, dt, sl) in enumerate(cases):
        inp = make_inputs_custom(B, T, H, dt, sl, seed=40 + i, pool=1.5)
        out, lse = _decode(inp, window=window)
        bo, bl = mla_decode_brute(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                                  inp.softmax_scale, inp.q_scale, inp.kv_scale, window=window)
        bo, bl = np.array(bo), np.array(bl)
        fin = np.isfinite(bl)
        assert np.array_equal(fin, np.isfinite(lse))
        worst = max(worst, np.abs(out - bo).max(), np.abs(lse[fin] - bl[fin]).max(initial=0))
    assert worst <= 1e-12


def test_window_covering_the_sequence_changes_nothing():
    inp = make_inputs_custom(2, 4, 3, "bf16", [300, 9], seed=44, pool=1.5)
    o0, l0 = _decode(inp)
    o1, l1 = _decode(inp, window=300)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_window_of_one_returns_the_newest_visible_key():
    inp = make_inputs_custom(2, 3, 2, "fp16", [90, 40], seed=45, pool=1.5)
    out, lse = _decode(inp, window=1)
    T, H = 3, 2
    for b in range(2):
        K = _keys(inp, b)
        for t in range(T):
            n = int(inp.seq_lens[b]) - T + t + 1
            for h in range(H):
                r = (b * T + t) * H + h
                qv = _values(inp.q, inp.q_scale)[b, t, h]
                assert np.array_equal(out[r], K[n - 1, :512])  # weight 1 on one key
                assert abs(lse[r] - inp.softmax_scale * float(qv @ K[n - 1])) <= 1e-12


def test_window_ignores_keys_before_its_start():
    inp = make_inputs_custom(1, 2, 2, "bf16", [200], seed=46, pool=1.5)
    o0, l0 = _decode(inp, window=50)
    # overwrite every cache row the rows' windows do not reach (keys 0 .. 148)
    bt = inp.block_tables[0]
    for j in range(149):
        inp.kv_cache[int(bt[j // 64]), j % 64] = 7.0
    o1, l1 = _decode(inp, window=50)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


# ---------------------------------------------------------------- ragged prefill
# tokenspeed-mla package card, "What it is and what it does": prefill of
# variable-length sequences packed without padding. Entry b's token t sees keys
# 0 .. seq_lens[b] - q_len_b + t.

from oracle.brute import mla_prefill_brute  # noqa: E402
from mla_paged_decode_04_b200.inputs import make_prefill_inputs  # noqa: E402


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_prefill_matches_the_brute_force_loop(dtype):
    # an empty entry, one token, a new sequence (no prefix), tokens spanning two pages
    inp = make_prefill_inputs([3, 0, 1, 5], [2, 4, 0, 60], 2, dtype, seed=71, pool=2.0)
    o, l = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                              inp.softmax_scale, dtype=dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale)
    bo, bl = mla_prefill_brute(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                               inp.softmax_scale, inp.q_scale, inp.kv_scale)
    assert sorted(bo) == list(range(inp.total_q * inp.heads))
    for r in range(inp.total_q * inp.heads):
        assert np.allclose(o[r], bo[r], rtol=0, atol=1e-12)
        assert abs(l[r] - bl[r]) <= 1e-12


def test_prefill_token_is_a_single_token_decode_of_its_prefix():
    """Each new token's row equals a q_len = 1 decode over the keys up to its own position."""
    inp = make_prefill_inputs([4, 2, 7], [0, 9, 130], 3, "fp16", seed=72, pool=1.5)
    o, l = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                              inp.softmax_scale, dtype="fp16")
    cu, H = inp.cu_seqlens_q.tolist(), inp.heads
    for b in range(inp.batch):
        qlen = cu[b + 1] - cu[b]
        for i in range(cu[b], cu[b + 1]):
            n_i = int(inp.seq_lens[b]) - qlen + (i - cu[b]) + 1
            d_o, d_l = oracle.mla_decode(inp.q[i].reshape(1, 1, H, 576), inp.kv_cache, inp.block_tables[b:b + 1],
                                         torch.tensor([n_i], dtype=torch.int32), inp.softmax_scale, dtype="fp16")
            assert np.allclose(o[i * H:(i + 1) * H], d_o, rtol=0, atol=1e-12)
            assert np.allclose(l[i * H:(i + 1) * H], d_l, rtol=0, atol=1e-12)


def test_prefill_rows_before_any_key_are_empty_and_rows_subset_matches():
    inp = make_prefill_inputs([5, 3], [0, 40], 2, "bf16", seed=73)
    sl = inp.seq_lens.clone()
    sl[0] = 2  # fewer keys than new tokens: the first three tokens see nothing
    o, l = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, sl, inp.softmax_scale,
                              dtype="bf16")
    H = inp.heads
    assert (o[:3 * H] == 0).all() and np.isneginf(l[:3 * H]).all()
    assert np.isfinite(l[3 * H:]).all()
    rows = [15, 0, 9, 3]
    so, sl_ = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, sl, inp.softmax_scale,
                                 dtype="bf16", rows=rows)
    assert np.array_equal(so, o[rows]) and np.array_equal(sl_, l[rows])


@pytest.mark.parametrize("window", [1, 3, 50])
def test_prefill_with_a_window_matches_the_brute_force_loop(window):
    inp = make_prefill_inputs([4, 6], [20, 0], 2, "bf16", seed=74, pool=1.5)
    o, l = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                              inp.softmax_scale, dtype="bf16", window=window)
    bo, bl = mla_prefill_brute(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                               inp.softmax_scale, window=window)
    for r in range(inp.total_q * inp.heads):
        assert np.allclose(o[r], bo[r], rtol=0, atol=1e-12)
        assert abs(l[r] - bl[r]) <= 1e-12
