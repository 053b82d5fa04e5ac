"""Pure-Python brute-force MLA decode for tiny inputs (test infrastructure only).

An independent restatement of the definition in ``mla_oracle.c`` used to pin
the C oracle: element values come from torch's own dtype conversions (a
library routine, not the oracle's decoders), and every sum is a Python loop
over ``math.exp`` / ``math.log``. Source of the definition: tokenspeed-mla
package card, "What it is and what it does"; TokenSpeed MLA article
(最快MLA内核背后的秘密), sections 一, 四 and 六.
"""
from __future__ import annotations

import math


def _as_floats(t, scale=1.0):
    # torch's dtype conversion to float64 (library routine), then plain lists
    return [[float(x) * scale for x in row] for row in t.double().reshape(-1, t.shape[-1]).tolist()]


def mla_decode_brute(q, kv_cache, block_tables, seq_lens, softmax_scale,
                     q_scale=1.0, kv_scale=1.0, window=0):
    """q [B,T,H,D], kv_cache [P,page,D] torch tensors; returns (out rows, lse list).

    window W > 0: a row with n visible keys attends to its last W keys only.
    """
    B, T, H, D = (int(x) for x in q.shape)
    _, page, _ = (int(x) for x in kv_cache.shape)
    Dv = 512
    qrows = _as_floats(q, q_scale)
    cache_rows = _as_floats(kv_cache, kv_scale)
    bt = [[int(x) for x in row] for row in block_tables.tolist()]
    sl = [int(x) for x in seq_lens.tolist()]
    outs, lses = [], []
    for b in range(B):
        for t in range(T):
            for h in range(H):
                qv = qrows[(b * T + t) * H + h]
                n = sl[b] - T + t + 1
                if n <= 0:
                    outs.append([0.0] * Dv)
                    lses.append(-math.inf)
                    continue
                first = max(0, n - window) if window > 0 else 0
                keys = []
                for j in range(first, n):
                    p = bt[b][j // page]
                    keys.append(cache_rows[p * page + j % page])
                s = [softmax_scale * math.fsum(qv[d] * k[d] for d in range(D)) for k in keys]
                m = max(s)
                lse = m + math.log(math.fsum(math.exp(x - m) for x in s))
                w = [math.exp(x - lse) for x in s]
                outs.append([math.fsum(w[j] * keys[j][d] for j in range(len(keys))) for d in range(Dv)])
                lses.append(lse)
    return outs, lses


def mla_prefill_brute(q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale,
                      q_scale=1.0, kv_scale=1.0, window=0):
    """Ragged prefill written out directly: packed token i of entry b (cu[b] <= i < cu[b+1])
    sees keys 0 .. seq_lens[b] - (cu[b+1] - cu[b]) + (i - cu[b]); with window W > 0 only the
    last W of them. q [total_q, H, D]."""
    total_q, H, D = (int(x) for x in q.shape)
    _, page, _ = (int(x) for x in kv_cache.shape)
    qrows = _as_floats(q, q_scale)
    cache_rows = _as_floats(kv_cache, kv_scale)
    cu = [int(x) for x in cu_seqlens_q.tolist()]
    bt = [[int(x) for x in row] for row in block_tables.tolist()]
    sl = [int(x) for x in seq_lens.tolist()]
    outs, lses = {}, {}
    for b in range(len(cu) - 1):
        qlen = cu[b + 1] - cu[b]
        for i in range(cu[b], cu[b + 1]):
            last = sl[b] - qlen + (i - cu[b])  # highest visible key
            for h in range(H):
                qv = qrows[i * H + h]
                if last < 0:
                    outs[i * H + h], lses[i * H + h] = [0.0] * 512, -math.inf
                    continue
                first = max(0, last + 1 - window) if window > 0 else 0
                keys = [cache_rows[bt[b][j // page] * page + j % page] for j in range(first, last + 1)]
                s = [softmax_scale * math.fsum(qv[d] * k[d] for d in range(D)) for k in keys]
                m = max(s)
                lse = m + math.log(math.fsum(math.exp(x - m) for x in s))
                w = [math.exp(x - lse) for x in s]
                outs[i * H + h] = [math.fsum(w[j] * keys[j][d] for j in range(len(keys))) for d in range(512)]
                lses[i * H + h] = lse
    return outs, lses
