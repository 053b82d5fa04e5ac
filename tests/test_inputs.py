"""Seeded input generator: reproducibility, layout and FP8 encoding (CPU)."""
import torch

from mla_paged_decode_04_b200.inputs import (FP8_MAX, WORKLOADS, draw_seq_lens,
                                             make_inputs, make_inputs_custom)


def test_same_seed_same_bytes():
    a = make_inputs_custom(2, 4, 8, "fp8", [300, 77], seed=5, pool=2.0)
    b = make_inputs_custom(2, 4, 8, "fp8", [300, 77], seed=5, pool=2.0)
    for x, y in [(a.q, b.q), (a.kv_cache, b.kv_cache)]:
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    assert torch.equal(a.block_tables, b.block_tables) and a.kv_scale == b.kv_scale


def test_block_tables_are_a_partial_permutation():
    inp = make_inputs_custom(3, 2, 4, "bf16", [130, 64, 1], seed=6, pool=2.0)
    pages = [3, 1, 1]
    used = []
    for b, npg in enumerate(pages):
        row = inp.block_tables[b]
        assert (row[:npg] >= 0).all() and (row[npg:] == -1).all()
        used += row[:npg].tolist()
    assert len(set(used)) == len(used) and max(used) < inp.num_pages
    assert inp.num_pages == 10  # ceil(2.0 * 5)


def test_fp8_scale_and_range():
    inp = make_inputs_custom(1, 4, 16, "fp8", [500], seed=7, pool=2.0)
    for codes, scale in [(inp.q, inp.q_scale), (inp.kv_cache, inp.kv_scale)]:
        v = codes.to(torch.float32)
        assert v.abs().max().item() <= FP8_MAX
        assert v.abs().max().item() >= 0.9 * FP8_MAX  # amax maps near the top code
        assert scale == float(torch.tensor(scale, dtype=torch.float32))


def test_workload_table_matches_the_configs():
    w = WORKLOADS
    assert (w["tiny_bf16"].batch, w["tiny_bf16"].q_len, w["tiny_bf16"].heads) == (1, 1, 16)
    assert (w["mtp_bf16"].batch, w["mtp_bf16"].q_len, w["mtp_bf16"].heads) == (4, 4, 32)
    assert w["fp8_long_b16"].max_seq_len == 81920 and w["fp8_long_b4"].batch == 4
    assert (w["highconc_bf16"].batch, w["highconc_bf16"].q_len, w["highconc_bf16"].heads) == (128, 2, 128)
    g = torch.Generator().manual_seed(1005)
    sl = draw_seq_lens(w["highconc_bf16"], g)
    assert sl.min() >= 2 and sl.max() <= 81920
    g = torch.Generator().manual_seed(1004)
    sl = draw_seq_lens(w["fold_fp16_h16"], g)
    assert sl.min() >= 1024 and sl.max() <= 65536


def test_tiny_workload_layout():
    inp = make_inputs("tiny_bf16")
    assert inp.num_pages == 4 and inp.block_tables.shape == (1, 4)
    assert sorted(inp.block_tables[0].tolist()) == [0, 1, 2, 3]
    assert inp.q.shape == (1, 1, 16, 576) and inp.kv_cache.shape == (4, 64, 576)


def test_prefill_inputs_are_seeded_and_consistent():
    from mla_paged_decode_04_b200.inputs import make_prefill_inputs, make_prefill_workload, PREFILL_WORKLOADS
    a = make_prefill_inputs([5, 0, 70], [3, 9, 0], 16, "fp8", seed=3)
    b = make_prefill_inputs([5, 0, 70], [3, 9, 0], 16, "fp8", seed=3)
    assert torch.equal(a.q.view(torch.uint8), b.q.view(torch.uint8))
    assert torch.equal(a.kv_cache.view(torch.uint8), b.kv_cache.view(torch.uint8))
    assert a.cu_seqlens_q.tolist() == [0, 5, 5, 75] and a.seq_lens.tolist() == [8, 9, 70]
    assert a.total_q == 75 and a.max_q_len == 70 and a.q.shape == (75, 16, 576)
    # every page an entry needs is a distinct page of the pool; unused table slots are -1
    used = []
    for bi, n in enumerate(a.seq_lens.tolist()):
        npg = (n + 63) // 64
        row = a.block_tables[bi].tolist()
        assert all(0 <= pg < a.kv_cache.shape[0] for pg in row[:npg]) and all(pg == -1 for pg in row[npg:])
        used += row[:npg]
    assert len(used) == len(set(used))
    w = PREFILL_WORKLOADS["prefill_bf16"]
    small = make_prefill_workload("prefill_bf16", batch=2)
    assert small.batch == 2 and small.max_q_len == w.max_q_len and small.dtype == "bf16"
    ql = [small.cu_seqlens_q[i + 1] - small.cu_seqlens_q[i] for i in range(2)]
    assert all(w.q_lens[1] <= int(q) <= w.q_lens[2] for q in ql)
