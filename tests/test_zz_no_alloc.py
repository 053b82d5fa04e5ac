"""mla_decode_no_alloc: the decode entry point for callers that cannot allocate.

Some callers cannot give the decode a workspace, because they have no way to
allocate device memory (an engine that owns all device memory, or a context
where cudaMalloc is not allowed). For them the library offers
mla_decode_no_alloc, which uses a scratch array inside the library instead of
a caller workspace, and mla_decode_no_alloc_status, which reads that array's
device status word. This file checks, through the C ABI, that two calls in a
row match both the fp64 oracle and mla_decode with a workspace; that a bad
block-table entry shows up in the status word; that a plan whose workspace
reaches close to the end of the scratch array is computed correctly; and that
a plan too large for the array is refused. It is named so that pytest
collects it last.
"""
import ctypes

import pytest
import torch

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200 import _lib
from mla_paged_decode_04_b200.inputs import make_inputs_custom
from helpers import ABS_TOL, LSE_TOL, REL_TOL, compare, oracle_rows

pytestmark = pytest.mark.gpu


def _entry():
    fn = ctypes.CDLL(_lib.LIB_PATH).mla_decode_no_alloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(_lib.MlaPlan), vp, vp, ctypes.c_int64, ctypes.c_int, vp, ctypes.c_int,
                   vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _status(clear=True):
    fn = ctypes.CDLL(_lib.LIB_PATH).mla_decode_no_alloc_status
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int32)]
    fn.restype = ctypes.c_int
    v = ctypes.c_int32(-1)
    assert fn(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), int(clear), ctypes.byref(v)) == 0
    return int(v.value)


def _no_alloc(fn, plan, g, out, lse):
    vp = ctypes.c_void_p
    return fn(ctypes.byref(plan), vp(g.q.data_ptr()), vp(g.kv_cache.data_ptr()), g.kv_cache.shape[0], 64,
              vp(g.block_tables.data_ptr()), g.block_tables.shape[1], vp(g.seq_lens.data_ptr()),
              g.softmax_scale, g.q_scale, g.kv_scale, vp(out.data_ptr()), vp(lse.data_ptr()),
              vp(torch.cuda.current_stream().cuda_stream))


def _same_as(out, lse, ref_out, ref_lse):
    o, r = out.float(), ref_out.float()
    assert ((o - r).abs() <= ABS_TOL + REL_TOL * r.abs()).all()
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isneginf(lse), torch.isneginf(ref_lse))
    assert ((lse[fin] - ref_lse[fin]).abs() <= LSE_TOL).all()


def _outputs(B, T, H, dev):
    out = torch.full((B, T, H, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, T, H), float("nan"), dtype=torch.float32, device=dev)
    return out, lse


def test_no_alloc_matches_the_oracle_and_the_workspace_entry_point_on_two_calls():
    dev = torch.device("cuda", 0)
    fn = _entry()
    cases = [(2, 4, 32, "bf16", [1500, 700], 21), (2, 4, 32, "fp8", [2000, 333], 22)]
    for B, T, H, dt, sl, seed in cases:   # two calls in a row, different shapes and dtypes
        inp = make_inputs_custom(B, T, H, dt, sl, seed=seed, pool=2.0)
        g = inp.to(dev)
        plan = mla.mla_decode_plan(B, T, H, max(sl), dt)
        assert plan.split_kv > 1 and plan.workspace_bytes <= _lib.MLA_NO_ALLOC_SCRATCH_BYTES
        out, lse = _outputs(B, T, H, dev)
        assert _no_alloc(fn, plan, g, out, lse) == 0
        torch.cuda.synchronize()
        assert _status() == 0
        ref_o, ref_l = oracle_rows(inp)
        compare(out, lse, ref_o, ref_l, dt, what=f"no-alloc {dt}")
        dec = mla.MlaDecoder(B, T, H, max(sl), dt, dev)
        ws_out, ws_lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
        torch.cuda.synchronize()
        assert dec.status() == 0
        _same_as(out, lse, ws_out, ws_lse)


def test_no_alloc_status_reports_a_bad_page_and_clears():
    dev = torch.device("cuda", 0)
    fn = _entry()
    inp = make_inputs_custom(2, 1, 16, "fp8", [200, 100], seed=24, pool=1.0)
    inp.block_tables[1, 0] = inp.num_pages + 5          # outside the pool: masked, flagged
    g = inp.to(dev)
    plan = mla.mla_decode_plan(2, 1, 16, 200, "fp8")
    out, lse = _outputs(2, 1, 16, dev)
    assert _no_alloc(fn, plan, g, out, lse) == 0
    assert _status(clear=False) & mla.MLA_DEV_BAD_PAGE
    assert _status(clear=True) & mla.MLA_DEV_BAD_PAGE   # still set: the first read did not clear it
    assert _status() == 0
    assert torch.isfinite(out.float()).all()
    # the same call with a valid table: clean status and oracle parity
    clean = make_inputs_custom(2, 1, 16, "fp8", [200, 100], seed=24, pool=1.0)
    g2 = clean.to(dev)
    assert _no_alloc(fn, plan, g2, out, lse) == 0
    assert _status() == 0
    ref_o, ref_l = oracle_rows(clean)
    compare(out, lse, ref_o, ref_l, "fp8", what="no-alloc after a bad page")


def test_no_alloc_with_a_workspace_near_the_end_of_its_scratch():
    """Fixed splits over 1408 rows: the plan's workspace reaches past 90% of the scratch array, so
    the partial LSEs at its end are written and read back by the combine."""
    dev = torch.device("cuda", 0)
    fn = _entry()
    B, T, H, n = 11, 2, 64, 2048
    plan = mla.mla_decode_plan_custom(B, T, H, n, "fp8", split_kv=16, kernel="tcgen05_solo")
    limit = _lib.MLA_NO_ALLOC_SCRATCH_BYTES
    assert plan.schedule == 0 and 0.9 * limit < plan.workspace_bytes <= limit
    inp = make_inputs_custom(B, T, H, "fp8", [n - 37 * b for b in range(B)], seed=25, pool=1.5)
    g = inp.to(dev)
    out, lse = _outputs(B, T, H, dev)
    assert _no_alloc(fn, plan, g, out, lse) == 0
    torch.cuda.synchronize()
    assert _status() == 0
    ref_o, ref_l = oracle_rows(inp)
    compare(out, lse, ref_o, ref_l, "fp8", what="no-alloc near the scratch end")


def test_no_alloc_refuses_plans_larger_than_its_scratch():
    dev = torch.device("cuda", 0)
    fn = _entry()
    g = make_inputs_custom(1, 1, 16, "bf16", [100], seed=23).to(dev)
    # fixed splits over 32768 rows: partials far above the scratch
    plan = mla.mla_decode_plan_custom(128, 2, 128, 81920, "bf16", kernel="simt")
    assert plan.workspace_bytes > _lib.MLA_NO_ALLOC_SCRATCH_BYTES
    out = torch.empty(1, 1, 16, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, 1, 16, device=dev)
    assert _no_alloc(fn, plan, g, out, lse) == -3   # MLA_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
