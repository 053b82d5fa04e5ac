"""Seeded random sweep of the GPU path against the oracle (sampled rows).

Each case draws an input type, head count (hence fold), decode or ragged prefill
shape, sequence lengths (empty and shorter-than-q_len entries included), a
sliding window, a forced CTA-pair count and the kernel. The fixed seeds make the
sweep reproducible; each case compares up to 300 rows within the tolerances in
helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200.inputs import make_inputs_custom, make_prefill_inputs
from helpers import compare, oracle_rows

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _decode_case(rng, dtype, H, window, pairs, kernel):
    B, T = int(rng.integers(1, 12)), int(rng.choice([1, 2, 3, 4, 6, 8]))
    sl = [int(x) for x in rng.integers(0, 6000, B)]
    if rng.random() < 0.3:
        sl[0] = int(rng.integers(0, T + 1))
    inp = make_inputs_custom(B, T, H, dtype, sl, seed=int(rng.integers(1 << 30)), pool=1.3)
    g = inp.to(DEV)
    dec = mla.MlaDecoder(B, T, H, max(1, max(sl)), dtype, DEV, split_kv=pairs, kernel=kernel, window=window)
    out, lse = dec(g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert dec.status() == 0
    rows = np.sort(rng.choice(B * T * H, min(B * T * H, 300), replace=False))
    ro, rl = oracle_rows(inp, rows, window=window)
    compare(out, lse, ro, rl, dtype, rows=rows, what=f"decode B={B} T={T} H={H} {dtype} sl={sl} W={window}")


def _prefill_case(rng, dtype, H, window, pairs, kernel):
    B = int(rng.integers(1, 6))
    ql = [int(x) for x in rng.integers(0, 300, B)]
    pre = [int(x) for x in rng.integers(0, 3000, B)]
    inp = make_prefill_inputs(ql, pre, H, dtype, seed=int(rng.integers(1 << 30)), pool=1.3,
                              max_q_len=max(ql + [1]) + int(rng.integers(0, 50)))
    g = inp.to(DEV)
    p = mla.MlaPrefill(B, inp.max_q_len, H, max(1, inp.max_seq_len), dtype, DEV, split_kv=pairs, kernel=kernel,
                       window=window)
    out, lse = p(g.q, g.cu_seqlens_q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, g.q_scale, g.kv_scale)
    torch.cuda.synchronize()
    assert p.status() == 0
    if inp.total_q == 0:
        return
    rows = np.sort(rng.choice(inp.total_q * H, min(inp.total_q * H, 300), replace=False))
    ro, rl = oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                                inp.softmax_scale, dtype=dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale,
                                rows=rows, window=window)
    compare(out, lse, ro, rl, dtype, rows=rows, what=f"prefill B={B} H={H} {dtype} ql={ql} pre={pre} W={window}")


@pytest.mark.parametrize("seed", range(40))
def test_random_case_matches_the_oracle(seed):
    rng = np.random.default_rng(1000 + seed)
    dtype = str(rng.choice(["fp8", "bf16", "fp16"]))
    H = int(rng.choice([8, 16, 32, 48, 64, 128]))
    window = int(rng.choice([0, 0, 1, 37, 200, 3000]))
    pairs = int(rng.choice([0, 0, 1, 5, 74]))
    kernel = str(rng.choice(["tcgen05", "tcgen05", "simt"]))
    if rng.random() < 0.5:
        _decode_case(rng, dtype, H, window, pairs, kernel)
    else:
        _prefill_case(rng, dtype, H, window, pairs, kernel)
