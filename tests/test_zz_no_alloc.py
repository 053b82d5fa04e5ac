"""mla_decode_no_alloc: the decode entry point for callers that cannot allocate.

Some callers cannot give the decode a workspace, because they have no way to
allocate device memory (an engine that owns all device memory, or a context
where cudaMalloc is not allowed). For them the library offers
mla_decode_no_alloc, which uses a scratch array inside the library instead of
a caller workspace. This file checks, through the C ABI, that it gives the
same results as mla_decode with a workspace on two calls in a row, and that a
plan too large for the scratch array is refused. It is named so that pytest
collects it last.
"""
import ctypes

import pytest
import torch

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200 import _lib
from mla_paged_decode_04_b200.inputs import make_inputs_custom
from helpers import ABS_TOL, LSE_TOL, REL_TOL

pytestmark = pytest.mark.gpu


def _entry():
    fn = ctypes.CDLL(_lib.LIB_PATH).mla_decode_no_alloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(_lib.MlaPlan), vp, vp, ctypes.c_int64, ctypes.c_int, vp, ctypes.c_int,
                   vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _no_alloc(fn, plan, g, out, lse):
    vp = ctypes.c_void_p
    return fn(ctypes.byref(plan), vp(g.q.data_ptr()), vp(g.kv_cache.data_ptr()), g.kv_cache.shape[0], 64,
              vp(g.block_tables.data_ptr()), g.block_tables.shape[1], vp(g.seq_lens.data_ptr()),
              g.softmax_scale, g.q_scale, g.kv_scale, vp(out.data_ptr()), vp(lse.data_ptr()),
              vp(torch.cuda.current_stream().cuda_stream))


def _check(out, lse, ref_out, ref_lse):
    o, r = out.float(), ref_out.float()
    assert ((o - r).abs() <= ABS_TOL + REL_TOL * r.abs()).all()
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isneginf(lse), torch.isneginf(ref_lse))
    assert ((lse[fin] - ref_lse[fin]).abs() <= LSE_TOL).all()


def test_no_alloc_matches_the_workspace_entry_point_on_two_calls():
    dev = torch.device("cuda", 0)
    fn = _entry()
    cases = [(2, 4, 32, "bf16", [1500, 700], 21), (2, 4, 32, "fp8", [2000, 333], 22)]
    for B, T, H, dt, sl, seed in cases:   # two calls in a row, different shapes and dtypes
        g = make_inputs_custom(B, T, H, dt, sl, seed=seed, pool=2.0).to(dev)
        plan = mla.mla_decode_plan(B, T, H, max(sl), dt)
        assert plan.split_kv > 1 and plan.workspace_bytes <= _lib.MLA_NO_ALLOC_SCRATCH_BYTES
        dec = mla.MlaDecoder(B, T, H, max(sl), dt, dev)
        ref_out, ref_lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale,
                               g.q_scale, g.kv_scale)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _no_alloc(fn, plan, g, out, lse) == 0
        torch.cuda.synchronize()
        _check(out, lse, ref_out, ref_lse)


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
