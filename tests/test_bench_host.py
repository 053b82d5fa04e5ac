"""Host arithmetic of the bench's roofline: algorithmic flops and the peaks it divides by."""
import json
import os

import bench


def _flops_by_rows(seq_lens, q_lens, heads):
    # every (token, head) row costs 2 * (576 + 512) flops per key it sees
    total = 0
    for n, q in zip(seq_lens, q_lens):
        for t in range(q):
            total += max(0, n - q + t + 1) * heads * 2 * (576 + 512)
    return total


def test_decode_flops_count_every_visible_key_of_every_row():
    sl = [81920, 3, 0, 130]
    assert bench.algorithmic_flops(sl, 4, 32) == _flops_by_rows(sl, [4] * 4, 32)
    # q_len = 1: one row per head over all n keys
    assert bench.algorithmic_flops([100], 1, 2) == 100 * 2 * 2 * 1088


def test_prefill_flops_follow_each_entrys_own_query_length():
    q_lens, prefix = [5, 0, 3], [10, 7, 0]
    cu = [0, 5, 5, 8]
    seq = [q + p for q, p in zip(q_lens, prefix)]
    assert bench.prefill_flops(cu, seq, 16) == _flops_by_rows(seq, q_lens, 16)


def test_tensor_peak_is_the_sustained_bf16_figure_doubled_for_fp8():
    bf16, src = bench.measured_tensor_peak("bf16", sustained=True)
    fp8, src8 = bench.measured_tensor_peak("fp8", sustained=True)
    assert fp8 == 2 * bf16 and "x 2" in src8 and "x 2" not in src
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        assert bf16 == float(d["bf16_tflops_sustained"])
        assert bench.measured_tensor_peak("bf16", sustained=False)[0] == float(d["bf16_tflops"])
    else:
        assert src.startswith("fallback")
