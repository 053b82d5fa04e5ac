"""Failure detection without a GPU fault: bounded waits that run out.

Every wait in the library's kernels has a time limit, after which the kernel
sets MLA_DEV_TIMEOUT in the workspace status word and returns; nothing traps.
Two waits are made to run out, each on a flag or barrier that nothing
completes, and each test checks that the call returns after about the limit,
that the status word then holds MLA_DEV_TIMEOUT, and that the next complete
decode on the same workspace is clean and matches the oracle:
  - the combine of the balanced schedule, launched alone on a zeroed
    workspace, waits (0.5 s limit) for the unit table's ready flag, which only
    the partial kernel sets; no TMA, cluster or tensor-memory state is
    involved;
  - the FP8 CTA-pair partial kernel, given a plan in its failure-detection
    test mode, never loads the first tile of each pair: the S issuer's wait
    for it runs out, the other roles see the abort flag or run out in turn,
    the leader waits (bounded) for the loads it issued, both CTAs meet at the
    final cluster barrier and free their tensor memory, and the combine's
    waits for the missing pieces run out too.
"""
import time

import pytest
import torch

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200.inputs import make_inputs_custom
from helpers import compare, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_combine_wait_runs_out_and_the_next_call_is_clean(dtype):
    dev = torch.device("cuda", 0)
    inp = make_inputs_custom(2, 4, 32, dtype, [3000, 1200], seed=61, pool=2.0, kv_std=0.5)
    g = inp.to(dev)
    dec = mla.MlaDecoder(2, 4, 32, 3000, dtype, dev)
    assert dec.plan.schedule == 1        # the balanced schedule (MLA_SCHEDULE_BALANCED)
    args = (g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale)
    out, lse = dec(*args, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0

    dec.workspace.zero_()          # the unit table's ready flag now reads 0, and no kernel will set it
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mla.mla_decode_combine(dec.plan, *args, out, lse, dec.workspace, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert dec.status() & mla.MLA_DEV_TIMEOUT
    assert 0.3 < waited < 10.0, waited   # each block gives up after its 0.5 s limit

    # the context is usable and the workspace recovers: a full decode is clean and correct
    out2, lse2 = dec(*args, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out2, lse2, ref_o, ref_l, dtype, what=f"after a timeout ({dtype})")


def test_partial_kernel_wait_runs_out_and_the_next_call_is_clean():
    dev = torch.device("cuda", 0)
    inp = make_inputs_custom(2, 4, 32, "fp8", [3000, 1200], seed=62, pool=2.0)
    g = inp.to(dev)
    dec = mla.MlaDecoder(2, 4, 32, 3000, "fp8", dev)
    assert dec.plan.schedule == 1 and dec.plan.kernel == 1   # the FP8 CTA-pair kernel, balanced schedule
    args = (g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale)
    out, lse = dec(*args, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0

    faulty = type(dec.plan).from_buffer_copy(dec.plan)
    faulty.fault_test = 1          # every pair leaves its first tile unloaded
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mla.mla_decode(faulty, *args, out, lse, dec.workspace, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert dec.status() & mla.MLA_DEV_TIMEOUT
    assert 0.3 < waited < 20.0, waited

    out2, lse2 = dec(*args, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out2, lse2, ref_o, ref_l, "fp8", what="after a partial-kernel timeout")
