"""The bounds-checking build, libmla_decode_check.so (compiled with MLA_BOUNDS_CHECK=1).

Its CTA-pair partial kernels, their on-device schedule and the balanced
combine test every global index against its buffer; an index outside sets
MLA_DEV_BOUNDS and the access is skipped. The tests route the package's
calls through that build (the binding's library handle is swapped for the
test) and check:
  - on valid inputs no check fires and the results match the oracle: FP8 and
    BF16 decode, a skewed batch whose piece lists spill to the workspace, and
    a ragged FP8 prefill;
  - in the checking build's store-fault test mode (plan.fault_test = 2, which
    moves every output row and partial slot of the FP8 pair kernel past its
    buffer) every such store is caught: the call returns, the status word
    holds MLA_DEV_BOUNDS and nothing else, and the next clean call on the same
    workspace has status 0 and matches the oracle.
No access outside a buffer is made at any point: the test mode exists only in
this build, and its checks skip each store they catch.
"""
import numpy as np
import pytest
import torch

import oracle
import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200 import _lib
from mla_paged_decode_04_b200.inputs import make_inputs_custom, make_prefill_inputs
from helpers import compare, oracle_rows

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture
def checking(monkeypatch):
    lib = _lib.load_library(_lib.CHECK_LIB_PATH)
    monkeypatch.setattr(_lib, "_lib", lib)
    assert mla.bounds_checked()
    return lib


@pytest.mark.parametrize("dtype,lens", [("fp8", [3000, 1200, 700]), ("bf16", [5000, 64, 2100])])
def test_checking_build_matches_the_oracle(checking, dtype, lens):
    inp = make_inputs_custom(3, 4, 32, dtype, lens, seed=71, pool=2.0, kv_std=0.5)
    g = inp.to(DEV)
    dec = mla.MlaDecoder(3, 4, 32, max(lens), dtype, DEV)
    assert dec.plan.schedule == 1  # the balanced schedule (MLA_SCHEDULE_BALANCED)
    out, lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, dtype, what=f"checking build ({dtype})")


def test_checking_build_with_spilled_piece_lists(checking):
    """Hundreds of one-tile entries ahead of a few long ones: piece lists go to the workspace's spill
    area, whose reads and writes are checked too."""
    gen = torch.Generator().manual_seed(214)
    sl = torch.randint(1, 100, (250,), generator=gen).tolist() + [20000] * 50
    inp = make_inputs_custom(300, 1, 16, "bf16", sl, seed=215, pool=1.1)
    g = inp.to(DEV)
    dec = mla.MlaDecoder(300, 1, 16, 20000, "bf16", DEV)
    out, lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    rows = np.array(sorted(set(range(0, 250 * 16, 11)) | set(range(4000, 4800, 9))))
    ref_o, ref_l = oracle_rows(inp, rows)
    compare(out, lse, ref_o, ref_l, "bf16", rows=rows, what="checking build, spilled piece lists")


def test_checking_build_ragged_prefill(checking):
    inp = make_prefill_inputs([3, 50, 1, 64], [100, 0, 4000, 63], 32, "fp8", seed=201, pool=1.5)
    g = inp.to(DEV)
    pre = mla.MlaPrefill(g.batch, g.max_q_len, g.heads, g.max_seq_len, "fp8", DEV)
    out, lse = pre(g.q, g.cu_seqlens_q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale,
                   g.kv_scale)
    torch.cuda.synchronize()
    assert pre.status() == 0
    ref_o, ref_l = oracle.mla_prefill(inp.q.cpu(), inp.cu_seqlens_q.cpu(), inp.kv_cache.cpu(),
                                      inp.block_tables.cpu(), inp.seq_lens.cpu(), inp.softmax_scale, dtype="fp8",
                                      q_scale=inp.q_scale, kv_scale=inp.kv_scale)
    compare(out, lse, ref_o, ref_l, "fp8", what="checking build, ragged prefill")


def test_store_fault_is_caught_and_the_next_call_is_clean(checking):
    lens = [3000, 1200, 700]
    inp = make_inputs_custom(3, 4, 32, "fp8", lens, seed=73, pool=2.0, kv_std=0.5)
    g = inp.to(DEV)
    dec = mla.MlaDecoder(3, 4, 32, max(lens), "fp8", DEV)
    args = (g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale)
    out = torch.empty(3, 4, 32, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(3, 4, 32, device=DEV)
    faulty = _lib.MlaPlan.from_buffer_copy(dec.plan)
    faulty.fault_test = 2  # every output row and partial slot of the FP8 pair kernel past its buffer
    mla.mla_decode(faulty, *args, out, lse, dec.workspace, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == mla.MLA_DEV_BOUNDS

    out2, lse2 = dec(*args, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out2, lse2, ref_o, ref_l, "fp8", what="after a caught store fault")
