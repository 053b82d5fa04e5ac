"""GPU parity of the ragged (prefill) path and of long piece lists, through the C ABI.

Ragged prefill (tokenspeed-mla package card, "What it is and what it does":
variable-length sequences packed without padding): entry b's q_len_b new
tokens are packed in q; token t sees keys 0 .. seq_lens[b] - q_len_b + t.
Compared with the fp64 oracle on every row for small cases and on sampled
rows at full size, within the tolerances in helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200.inputs import make_inputs_custom, make_prefill_inputs, make_prefill_workload
from helpers import compare, oracle_rows

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def run_prefill(inp, kernel="auto", split_kv=0, window=0, want_lse=True, max_q_len=None):
    g = inp.to(DEV)
    pre = mla.MlaPrefill(g.batch, max_q_len or g.max_q_len, g.heads, max(g.max_seq_len, 0), g.dtype, DEV,
                         split_kv=split_kv, kernel=kernel, window=window)
    out, lse = pre(g.q, g.cu_seqlens_q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale,
                   g.kv_scale, want_lse=want_lse)
    torch.cuda.synchronize()
    return out, lse, pre.status(), pre


def prefill_oracle(inp, rows=None, window=0):
    """Oracle rows of `inp` (tensors on any device; the oracle reads host copies of the same bytes)."""
    return oracle.mla_prefill(inp.q.cpu(), inp.cu_seqlens_q.cpu(), inp.kv_cache.cpu(), inp.block_tables.cpu(),
                              inp.seq_lens.cpu(), inp.softmax_scale, dtype=inp.dtype, q_scale=inp.q_scale,
                              kv_scale=inp.kv_scale, rows=rows, window=window)


# (q_lens, prefix_lens, H): an entry without new tokens, one token, tokens that
# are not a multiple of the fold, a new sequence (no prefix), long prefixes
SMALL = [
    ([0, 1, 7, 33, 130, 200], [5, 0, 64, 1000, 0, 2000], 16),   # F = 8
    ([3, 50, 1, 64], [100, 0, 4000, 63], 32),                    # F = 4
    ([5, 17, 2], [0, 300, 129], 48),                             # F = 2, 96 rows per unit
    ([9, 1, 40], [10, 700, 0], 128),                             # F = 1
]


@pytest.mark.parametrize("dtype", ["fp8", "bf16", "fp16"])
@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_prefill_small_cases_all_rows(case, kernel, dtype):
    ql, pre, H = SMALL[case]
    inp = make_prefill_inputs(ql, pre, H, dtype, seed=200 + case, pool=1.5)
    out, lse, status, p = run_prefill(inp, kernel)
    assert status == 0 and p.plan.varlen == 1
    ref_o, ref_l = prefill_oracle(inp)
    compare(out, lse, ref_o, ref_l, dtype, what=f"prefill case {case} {kernel}")


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_prefill_plan_longer_than_every_entry_and_few_pairs(dtype):
    """max_q_len above every entry (empty query groups) and units cut between 3 pairs."""
    inp = make_prefill_inputs([40, 3, 0, 77], [3000, 10, 500, 2000], 32, dtype, seed=211, pool=1.3)
    out, lse, status, p = run_prefill(inp, "tcgen05", split_kv=3, max_q_len=300)
    assert status == 0 and p.plan.q_groups == 75
    ref_o, ref_l = prefill_oracle(inp)
    compare(out, lse, ref_o, ref_l, dtype, what="max_q_len 300, 3 pairs")


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_prefill_with_a_sliding_window(dtype):
    inp = make_prefill_inputs([30, 1, 90], [500, 64, 1000], 32, dtype, seed=212, pool=1.5)
    out, lse, status, p = run_prefill(inp, "tcgen05", window=200)
    assert status == 0 and p.plan.window == 200
    ref_o, ref_l = prefill_oracle(inp, window=200)
    compare(out, lse, ref_o, ref_l, dtype, what="prefill W=200")


def test_prefill_bad_query_range_sets_the_status_and_spares_the_rest():
    inp = make_prefill_inputs([4, 6, 5], [10, 20, 30], 16, "bf16", seed=213)
    bad = inp.to(DEV)
    cu_dev = inp.cu_seqlens_q.clone().to(DEV)
    cu_dev[2] = 3
    pre = mla.MlaPrefill(inp.batch, inp.max_q_len + 4, inp.heads, inp.max_seq_len, "bf16", DEV)
    out = torch.full((inp.total_q, inp.heads, 512), 7.0, dtype=torch.bfloat16, device=DEV)
    out, lse = pre(bad.q, cu_dev, bad.kv_cache, bad.block_tables, bad.seq_lens, inp.softmax_scale, out=out)
    torch.cuda.synchronize()
    assert pre.status() & mla.MLA_DEV_BAD_QLEN
    # cu = [0, 4, 3, 15]: entry 1 runs backwards and entry 2 holds 12 tokens, more than the
    # plan's max_q_len of 10; entry 0 is still computed, and no other row is written
    assert (out[4:].float() == 7.0).all()
    H = inp.heads
    ref_o, ref_l = prefill_oracle(inp, rows=np.arange(4 * H))
    compare(out[:4], lse[:4], ref_o, ref_l, "bf16", what="entry 0 beside a bad range")


@pytest.mark.parametrize("name", ["prefill_fp8", "prefill_bf16"])
def test_prefill_full_size_sampled_rows(name):
    inp = make_prefill_workload(name, device=DEV)
    out, lse, status, p = run_prefill(inp)
    assert status == 0 and p.plan.schedule == 1
    H = inp.heads
    rng = np.random.default_rng(7)
    cu = inp.cu_seqlens_q.tolist()
    toks = {0, inp.total_q - 1} | {c for c in cu[1:-1]} | set(int(x) for x in rng.choice(inp.total_q, 40, False))
    rows = np.array(sorted(t * H + int(rng.integers(H)) for t in toks), dtype=np.int64)
    ref_o, ref_l = prefill_oracle(inp, rows=rows)
    compare(out, lse, ref_o, ref_l, inp.dtype, rows=rows, what=name)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_skewed_decode_batch_spills_long_piece_lists(dtype):
    """Hundreds of one-tile entries ahead of a few long ones: the first pairs' ranges meet more
    units than a pair keeps in shared memory, so their piece lists go to the workspace."""
    g = torch.Generator().manual_seed(214)
    short = torch.randint(1, 100, (250,), generator=g).tolist()
    sl = short + [20000] * 50
    inp = make_inputs_custom(300, 1, 16, dtype, sl, seed=215, pool=1.1)
    dec = mla.MlaDecoder(300, 1, 16, 20000, dtype, DEV)
    gi = inp.to(DEV)
    out, lse = dec(gi.q, gi.kv_cache, gi.block_tables, gi.seq_lens, gi.softmax_scale, gi.q_scale, gi.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0 and dec.plan.schedule == 1
    rng = np.random.default_rng(3)
    rows = np.array(sorted(set(range(0, 250 * 16, 7)) | set(int(x) for x in rng.choice(np.arange(4000, 4800), 40,
                                                                                            False))))
    ref_o, ref_l = oracle_rows(inp, rows)
    compare(out, lse, ref_o, ref_l, dtype, rows=rows, what="skewed decode batch")


def test_long_fresh_prefill_keeps_two_term_p_for_its_early_rows():
    """9000 new tokens with no cached prefix (FP8): the entry has more keys than the two-term
    threshold, but its first tokens see only a few keys; their units must still send P as
    two E4M3 terms (the choice follows the unit's fewest visible keys, not the entry's)."""
    inp = make_prefill_inputs([9000], [0], 16, "fp8", seed=216, pool=1.1)
    out, lse, status, p = run_prefill(inp)
    assert status == 0
    H = inp.heads
    rng = np.random.default_rng(9)
    toks = sorted(set(range(0, 40)) | set(range(8950, 9000)) | set(int(x) for x in rng.choice(9000, 60, False)))
    rows = np.array([t * H + h for t in toks for h in range(H)], dtype=np.int64)
    ref_o, ref_l = prefill_oracle(inp, rows=rows)
    compare(out, lse, ref_o, ref_l, "fp8", rows=rows, what="9000 fresh tokens")
