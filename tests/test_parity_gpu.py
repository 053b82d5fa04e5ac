"""GPU parity: the CUDA path against the fp64 oracle, through the C ABI.

Small cases are compared on every row; the full-size workloads run in the
launch configuration the bench times (automatic plan) and are compared on
sampled rows the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200.inputs import make_inputs, make_inputs_custom
from helpers import compare, oracle_rows, sample_rows

pytestmark = pytest.mark.gpu

# tcgen05: the default tensor-core kernel (for FP8 the CTA-pair form);
# tcgen05_solo: the FP8 variant without cross-CTA MMAs; simt: the cross-check.
KERNELS = ["tcgen05", "simt", "tcgen05_solo"]


def run(inp, kernel="auto", split_kv=0, fold=0, want_lse=True, window=0):
    if kernel == "tcgen05_solo" and inp.dtype != "fp8":
        pytest.skip("the solo variant is FP8 only")
    dev = torch.device("cuda", 0)
    g = inp.to(dev)
    dec = mla.MlaDecoder(g.batch, g.q_len, g.heads, max(g.max_seq_len, 0), g.dtype, dev,
                         split_kv=split_kv, fold=fold, kernel=kernel, window=window)
    out, lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale,
                   g.q_scale, g.kv_scale, want_lse=want_lse)
    torch.cuda.synchronize()
    status = dec.status()
    return out, lse, status, dec


SMALL = [
    # (B, T, H, dtype, seq_lens, pool, q_std, kv_std)
    (1, 1, 16, "bf16", [256], "exact", 1.0, 1.0),
    (2, 4, 32, "bf16", [1000, 77], 2.0, 1.0, 0.5),
    (3, 4, 16, "fp16", [64, 65, 300], 2.0, 1.0, 1.0),
    (2, 4, 64, "fp16", [513, 130], 2.0, 1.0, 1.0),
    (2, 2, 128, "bf16", [700, 3], 2.0, 1.0, 0.5),
    (2, 4, 32, "fp8", [900, 128], 2.0, 1.0, 1.0),
    (1, 3, 40, "fp8", [200], 1.0, 1.0, 1.0),
    (4, 1, 8, "bf16", [1, 2, 63, 64], 1.0, 1.0, 1.0),
    (3, 4, 32, "fp16", [2, 0, 5], 1.0, 1.0, 1.0),   # seq_len < q_len and empty entries
    (3, 1, 16, "fp8", [64, 130, 1], 2.0, 1.0, 1.0),  # 16 rows; odd page counts; one key
    (4, 4, 32, "fp8", [2, 0, 191, 4097], 1.5, 1.0, 1.0),  # seq_len < q_len, empty entry, ragged tails
    (2, 2, 48, "fp8", [300, 64], 1.0, 1.0, 1.0),    # 96 rows: the second CTA holds 32 live rows
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_cases_all_rows(case, kernel):
    B, T, H, dt, sl, pool, qs, ks = SMALL[case]
    inp = make_inputs_custom(B, T, H, dt, sl, seed=100 + case, pool=pool, q_std=qs, kv_std=ks)
    out, lse, status, _ = run(inp, kernel)
    assert status == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, dt, what=f"case {case}")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("split_kv", [1, 2, 3, 7, 10 ** 6])
def test_forced_splits_agree(split_kv, kernel):
    inp = make_inputs_custom(2, 4, 32, "bf16", [1500, 640], seed=7, pool=2.0, kv_std=0.5)
    out, lse, status, dec = run(inp, kernel, split_kv=split_kv)
    assert status == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, "bf16", what=f"split {dec.plan.split_kv}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_fold_on_and_off_agree(kernel):
    inp = make_inputs_custom(2, 4, 16, "fp16", [333, 1200], seed=8, pool=2.0)
    ref_o, ref_l = oracle_rows(inp)
    for fold in (1, 2, 4):
        out, lse, status, dec = run(inp, kernel, fold=fold)
        assert dec.plan.fold == fold and status == 0
        compare(out, lse, ref_o, ref_l, "fp16", what=f"fold {fold}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_page_shuffle_is_bitwise_invariant(kernel):
    inp = make_inputs_custom(2, 4, 32, "fp8", [777, 2000], seed=9, pool=2.0)
    out1, lse1, _, _ = run(inp, kernel)
    perm = torch.randperm(inp.num_pages, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(inp.num_pages)
    moved = make_inputs_custom(2, 4, 32, "fp8", [777, 2000], seed=9, pool=2.0)
    moved.kv_cache = inp.kv_cache[perm].clone()
    bt = inp.block_tables.clone()
    bt[bt >= 0] = inv[bt[bt >= 0].long()].to(torch.int32)
    moved.block_tables = bt
    out2, lse2, _, _ = run(moved, kernel)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


@pytest.mark.parametrize("kernel", KERNELS)
def test_keys_past_the_causal_limit_do_not_matter(kernel):
    T, H = 4, 32
    inp = make_inputs_custom(1, T, H, "bf16", [300], seed=10)
    out1, lse1, _, _ = run(inp, kernel)
    # key 298 is visible only to tokens 2 and 3 (limits 296, 297, 298, 299)
    pert = make_inputs_custom(1, T, H, "bf16", [300], seed=10)
    page = int(pert.block_tables[0, 298 // 64])
    pert.kv_cache[page, 298 % 64] = 7.0
    out2, lse2, _, _ = run(pert, kernel)
    assert torch.equal(out1[:, :2], out2[:, :2]) and torch.equal(lse1[:, :2], lse2[:, :2])
    assert not torch.equal(out1[:, 2:], out2[:, 2:])


@pytest.mark.parametrize("kernel", KERNELS)
def test_lse_optional(kernel):
    inp = make_inputs_custom(1, 2, 16, "bf16", [500], seed=11)
    out1, _, _, _ = run(inp, kernel, want_lse=False)
    out2, _, _, _ = run(inp, kernel)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("kernel", KERNELS)
def test_cuda_graph_replay_matches_eager(kernel, dtype):
    if kernel == "tcgen05_solo" and dtype != "fp8":
        pytest.skip("the solo variant is FP8 only")
    dev = torch.device("cuda", 0)
    inp = make_inputs_custom(2, 4, 32, dtype, [900, 2100], seed=12, pool=2.0).to(dev)
    dec = mla.MlaDecoder(2, 4, 32, 2100, dtype, dev, kernel=kernel)
    out = torch.empty(2, 4, 32, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(2, 4, 32, dtype=torch.float32, device=dev)
    sc = (inp.q_scale, inp.kv_scale)
    dec(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens, inp.softmax_scale, *sc, out=out, lse=lse)
    torch.cuda.synchronize()
    eager_o, eager_l = out.clone(), lse.clone()
    out.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dec(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens, inp.softmax_scale, *sc, out=out, lse=lse)
    for _ in range(3):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager_o) and torch.equal(lse, eager_l)
    del g


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("kernel", KERNELS)
def test_status_word_flags_bad_pages_and_long_sequences(kernel, dtype):
    if kernel == "tcgen05_solo" and dtype != "fp8":
        pytest.skip("the solo variant is FP8 only")
    inp = make_inputs_custom(2, 1, 16, dtype, [200, 100], seed=13, pool=1.0)
    inp.block_tables[1, 0] = inp.num_pages + 5          # outside the pool
    _, _, status, _ = run(inp, kernel)
    assert status & mla.MLA_DEV_BAD_PAGE
    inp2 = make_inputs_custom(1, 1, 16, dtype, [200], seed=14, pool=1.0)
    dev = torch.device("cuda", 0)
    g = inp2.to(dev)
    dec = mla.MlaDecoder(1, 1, 16, 100, dtype, dev, kernel=kernel)   # planned for 100 keys
    out, lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() & mla.MLA_DEV_SEQ_TOO_LONG
    assert torch.isfinite(out.float()).all()
    # a clean call clears the word again
    g.seq_lens.fill_(90)
    dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    assert dec.status() == 0


def test_batch_zero_is_a_no_op():
    dev = torch.device("cuda", 0)
    dec = mla.MlaDecoder(0, 1, 16, 0, "bf16", dev)
    q = torch.empty(0, 1, 16, 576, dtype=torch.bfloat16, device=dev)
    cache = torch.zeros(1, 64, 576, dtype=torch.bfloat16, device=dev)
    bt = torch.zeros(0, 1, dtype=torch.int32, device=dev)
    sl = torch.zeros(0, dtype=torch.int32, device=dev)
    out, lse = dec(q, cache, bt, sl, 0.04)
    torch.cuda.synchronize()
    assert out.numel() == 0 and dec.status() == 0


FULL = ["tiny_bf16", "mtp_bf16", "fp8_long_b4", "fp8_long_b16", "fold_fp16_h16", "fold_fp16_h64",
        "highconc_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads(name):
    """Automatic plan (what the bench times); every row for the small ones, sampled rows otherwise."""
    dev = torch.device("cuda", 0)
    inp = make_inputs(name, device=dev)
    out, lse, status, dec = run(inp)
    assert status == 0
    B, T, H = inp.batch, inp.q_len, inp.heads
    rows = None if B * T * H * inp.max_seq_len <= 512 * 8192 else sample_rows(B, T, H, n=48)
    ref_o, ref_l = oracle_rows(inp, rows)
    compare(out, lse, ref_o, ref_l, inp.dtype, rows=rows, what=name)
    # properties that hold at any size: finite outputs, LSE bounded by the closed form
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_host_pointers_are_refused_before_launch():
    """A pageable host pointer reaching the C ABI (here the block table) is refused with
    MLA_ERR_INVALID_ARG and nothing is enqueued; the context stays usable."""
    import ctypes
    from mla_paged_decode_04_b200 import _lib
    dev = torch.device("cuda", 0)
    inp = make_inputs_custom(1, 1, 16, "bf16", [256], seed=15, pool="exact")
    g = inp.to(dev)
    dec = mla.MlaDecoder(1, 1, 16, 256, "bf16", dev)
    out = torch.empty(1, 1, 16, 512, dtype=torch.bfloat16, device=dev)
    host_bt = inp.block_tables.contiguous()          # CPU tensor
    assert not host_bt.is_cuda
    vp = ctypes.c_void_p
    rc = _lib.lib().mla_decode(ctypes.byref(dec.plan), vp(g.q.data_ptr()), vp(g.kv_cache.data_ptr()),
                               g.kv_cache.shape[0], 64, vp(host_bt.data_ptr()), host_bt.shape[1],
                               vp(g.seq_lens.data_ptr()), g.softmax_scale, 1.0, 1.0, vp(out.data_ptr()),
                               None, vp(dec.workspace.data_ptr()), dec.workspace.numel(),
                               vp(torch.cuda.current_stream().cuda_stream))
    assert rc == -1
    torch.cuda.synchronize()
    o, l = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0 and torch.isfinite(o.float()).all()


@pytest.mark.parametrize("dtype", ["fp8", "bf16", "fp16"])
@pytest.mark.parametrize("pairs", [1, 2, 3, 7, 74])
def test_balanced_schedule_forced_pairs(pairs, dtype):
    """CTA-pair kernels with the balanced schedule forced onto few pairs: units are cut
    between pairs and pairs cover several units (empty, one-key, ragged, single-term entries)."""
    inp = make_inputs_custom(6, 2, 32, dtype, [0, 1, 130, 700, 4097, 20000], seed=31, pool=1.5)
    out, lse, status, dec = run(inp, "tcgen05", split_kv=pairs)
    assert dec.plan.schedule == 1 and status == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, dtype, what=f"{pairs} pairs")


@pytest.mark.parametrize("dtype", ["fp8", "bf16", "fp16"])
def test_balanced_schedule_many_ragged_units(dtype):
    g = torch.Generator().manual_seed(33)
    sl = torch.randint(0, 3000, (40,), generator=g).tolist()
    sl[3] = 0
    sl[7] = 1
    inp = make_inputs_custom(40, 1, 16, dtype, sl, seed=34, pool=1.3)
    out, lse, status, dec = run(inp, "tcgen05")
    assert dec.plan.schedule == 1 and status == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, dtype, what="40 ragged units")


def test_past_the_balanced_unit_limit_16bit_takes_fixed_splits():
    """More units than the balanced decode schedule takes (16384): 16-bit inputs go to the
    fixed-split exchange kernel, still exact against the oracle (sampled rows)."""
    g = torch.Generator().manual_seed(35)
    sl = torch.randint(1, 200, (16400,), generator=g).tolist()
    inp = make_inputs_custom(16400, 1, 16, "bf16", sl, seed=36, pool=1.2)
    out, lse, status, dec = run(inp, "tcgen05")
    assert dec.plan.schedule == 0 and dec.plan.kernel == 1 and status == 0
    rows = sample_rows(16400, 1, 16, n=400, seed=37)
    ref_o, ref_l = oracle_rows(inp, rows)
    compare(out, lse, ref_o, ref_l, "bf16", rows=rows, what="16400 units, fixed splits")


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_thousands_of_short_units_on_the_balanced_schedule(dtype):
    """4000 one-token entries of 1..300 keys: far more units than pairs, every pair's piece list
    spills past shared memory, and the combine's blocks take several units each."""
    g = torch.Generator().manual_seed(38)
    sl = torch.randint(0, 300, (4000,), generator=g).tolist()
    inp = make_inputs_custom(4000, 1, 16, dtype, sl, seed=39, pool=1.2)
    out, lse, status, dec = run(inp, "tcgen05")
    assert dec.plan.schedule == 1 and status == 0
    rows = sample_rows(4000, 1, 16, n=400, seed=40)
    ref_o, ref_l = oracle_rows(inp, rows)
    compare(out, lse, ref_o, ref_l, dtype, rows=rows, what="4000 short units, balanced")


@pytest.mark.parametrize("kernel", ["tcgen05", "tcgen05_solo"])
def test_fp8_entries_around_the_two_term_threshold(kernel):
    """FP8 rows just below and above 8192 visible keys: two-term P below, one E4M3 term above;
    every row within the tolerances."""
    inp = make_inputs_custom(4, 4, 32, "fp8", [8190, 8196, 12000, 16383], seed=45, pool=1.2)
    out, lse, status, dec = run(inp, kernel)
    assert status == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, "fp8", what=f"threshold {kernel}")


# ---------------------------------------------------------------- sliding window
# A row with n visible keys attends to keys [max(0, n - W), n) (a decode option
# the TokenSpeed MLA article lists among its tests, section 六). The CTA-pair
# kernels skip the tiles below the unit's lowest window start and mask the
# rest per row; the SIMT kernel starts each row's loop at its window start.

WINDOW_LENS = [0, 1, 3, 130, 700, 4097]  # empty, single key, seq_len < q_len, ragged tails


@pytest.mark.parametrize("dtype", ["fp8", "bf16", "fp16"])
@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
@pytest.mark.parametrize("window", [1, 2, 63, 64, 65, 200, 1000])
def test_window_matches_the_oracle(window, kernel, dtype):
    inp = make_inputs_custom(6, 4, 32, dtype, WINDOW_LENS, seed=41, pool=1.5)
    out, lse, status, dec = run(inp, kernel, window=window)
    assert dec.plan.window == window and status == 0
    ref_o, ref_l = oracle_rows(inp, window=window)
    compare(out, lse, ref_o, ref_l, dtype, what=f"{kernel} W={window}")


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
@pytest.mark.parametrize("pairs", [1, 3, 74])
def test_window_with_units_cut_between_pairs(pairs, dtype):
    """Few pairs, long entries: windowed units are still cut into pieces that the combine merges."""
    inp = make_inputs_custom(3, 2, 64, dtype, [20000, 5000, 129], seed=42, pool=1.3)
    out, lse, status, dec = run(inp, "tcgen05", split_kv=pairs, window=3000)
    assert dec.plan.schedule == 1 and status == 0
    ref_o, ref_l = oracle_rows(inp, window=3000)
    compare(out, lse, ref_o, ref_l, dtype, what=f"W=3000, {pairs} pairs")


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_window_past_every_length_is_bitwise_full_attention(dtype):
    inp = make_inputs_custom(6, 4, 32, dtype, WINDOW_LENS, seed=43, pool=1.5)
    o0, l0, s0, _ = run(inp, "tcgen05")
    ow, lw, sw, _ = run(inp, "tcgen05", window=4097)
    assert s0 == 0 and sw == 0
    assert torch.equal(o0, ow) and torch.equal(l0, lw)


@pytest.mark.parametrize("name,window", [("fp8_long_b16", 8192), ("fp8_long_b16", 4096), ("fold_fp16_h16", 8192)])
def test_window_full_size_sampled_rows(name, window):
    """Full-size workloads with a sliding window. An FP8 row then attends to min(n, W) keys, so
    W = 8192 keeps the single-term P encoding (two terms are taken below 8192 keys) and W = 4096
    takes the two-term encoding on every row of the 80K-key entries."""
    inp = make_inputs(name, device=torch.device("cuda", 0))
    out, lse, status, dec = run(inp, "auto", window=window)
    assert dec.plan.window == window and status == 0
    rows = sample_rows(inp.batch, inp.q_len, inp.heads, n=48, seed=45)
    ref_o, ref_l = oracle_rows(inp, rows, window=window)
    compare(out, lse, ref_o, ref_l, inp.dtype, rows=rows, what=f"{name} W={window}")
