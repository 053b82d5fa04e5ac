"""Shared test helpers: run the oracle on chosen rows and compare with the GPU.

Tolerances (the accuracy bar for the GPU path against the fp64 oracle):
  out (BF16):  |gpu - ref| <= 1e-2 + 2e-2 * |ref| elementwise, and a
               relative L2 error <= 1e-2 (16-bit P) / 3e-2 (E4M3 P), since
               decode outputs are small and the absolute bound alone is weak;
  lse (fp32):  |gpu - ref| <= 1e-3, and -inf exactly where the oracle has -inf.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

ABS_TOL, REL_TOL, LSE_TOL = 1e-2, 2e-2, 1e-3
REL_L2 = {"bf16": 1e-2, "fp16": 1e-2, "fp8": 3e-2}


def oracle_rows(inp, rows=None, window=0):
    """Oracle (out, lse) for flat rows (b*T+t)*H+h of `inp` (tensors on any device),
    with each row restricted to its last `window` visible keys when window > 0.

    Only the pages of the touched batch entries are copied to the host; the
    oracle sees exactly the bytes the GPU path reads.
    """
    B, T, H = inp.batch, inp.q_len, inp.heads
    rows = np.arange(B * T * H) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, 512))
    lse = np.zeros(rows.size)
    sl = inp.seq_lens.cpu()
    bt = inp.block_tables.cpu()
    per_b = {}
    for i, r in enumerate(rows):
        per_b.setdefault(int(r) // (T * H), []).append(i)
    for b, idx in per_b.items():
        n = max(0, int(sl[b]))
        npg = (n + 63) // 64
        pages = bt[b, :npg].long()
        if npg:
            cache_b = inp.kv_cache.index_select(0, pages.to(inp.kv_cache.device)).cpu()
        else:
            cache_b = inp.kv_cache[:1].cpu()
        bt_b = torch.arange(max(npg, 1), dtype=torch.int32)[None]
        local = rows[idx] - b * T * H
        o, l = oracle.mla_decode(inp.q[b:b + 1].cpu(), cache_b, bt_b, sl[b:b + 1],
                                 inp.softmax_scale, dtype=inp.dtype, q_scale=inp.q_scale,
                                 kv_scale=inp.kv_scale, rows=local, window=window)
        out[idx] = o
        lse[idx] = l
    return out, lse


def compare(out_gpu, lse_gpu, ref_out, ref_lse, dtype, rows=None, what=""):
    """Assert the BF16 output and fp32 LSE match the oracle within the tolerances."""
    o = out_gpu.float().reshape(-1, 512).cpu().double().numpy()
    if rows is not None:
        o = o[np.asarray(rows)]
    err = np.abs(o - ref_out)
    bound = ABS_TOL + REL_TOL * np.abs(ref_out)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, max err "
                           f"{err.max():.3e}, worst at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    ref_norm = np.linalg.norm(ref_out)
    rel_l2 = float(np.linalg.norm(o - ref_out) / ref_norm) if ref_norm > 0 else 0.0
    assert rel_l2 <= REL_L2[dtype], f"{what}: rel-L2 {rel_l2:.3e}"
    if lse_gpu is not None:
        l = lse_gpu.reshape(-1).cpu().double().numpy()
        if rows is not None:
            l = l[np.asarray(rows)]
        ninf = np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(l), ninf), f"{what}: -inf pattern differs"
        if (~ninf).any():
            lerr = np.abs(l[~ninf] - ref_lse[~ninf]).max()
            assert lerr <= LSE_TOL, f"{what}: lse err {lerr:.3e}"
    return rel_l2


def sample_rows(B, T, H, n=64, seed=0):
    """Rows spread over entries, tokens and heads, always including first and last."""
    g = np.random.default_rng(seed)
    total = B * T * H
    fixed = {0, total - 1}
    for t in range(T):
        fixed.add(t * H)
        fixed.add(((B - 1) * T + t) * H + H - 1)
    extra = g.choice(total, size=min(total, max(0, n - len(fixed))), replace=False)
    return np.array(sorted(fixed | set(int(x) for x in extra)), dtype=np.int64)


def expected_kv_bytes(inp):
    esize = 1 if inp.dtype == "fp8" else 2
    return int(inp.seq_lens.clamp(min=0).sum()) * 576 * esize


def isclose_lse(a, b):
    return (math.isinf(a) and math.isinf(b)) or abs(a - b) <= LSE_TOL
