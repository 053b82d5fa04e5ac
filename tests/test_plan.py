"""Host plan: fold factor, split_kv and workspace sizing (CPU only)."""
import math

import pytest

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200.inputs import WORKLOADS


def _fold_rule(q_len, heads):
    # Largest F with q_len % F == 0 and H*F <= 128 (TokenSpeed MLA article, section 三).
    return max(f for f in range(1, q_len + 1) if q_len % f == 0 and heads * f <= 128)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_fold_per_workload(name):
    w = WORKLOADS[name]
    p = mla.mla_decode_plan(w.batch, w.q_len, w.heads, w.max_seq_len, w.dtype)
    assert p.fold == _fold_rule(w.q_len, w.heads)
    assert p.q_groups * p.fold == w.q_len and p.rows_per_unit == w.heads * p.fold <= 128


def test_fold_examples_from_the_article():
    # H=64, q_len=4 folds F=2 (H_eff=128, two query groups); section 三's example.
    p = mla.mla_decode_plan(32, 4, 64, 65536, "fp16")
    assert (p.fold, p.q_groups, p.rows_per_unit) == (2, 2, 128)
    assert mla.mla_decode_plan(32, 4, 16, 65536, "fp16").fold == 4
    assert mla.mla_decode_plan(4, 4, 32, 8192, "bf16").fold == 4
    assert mla.mla_decode_plan(128, 2, 128, 81920, "bf16").fold == 1
    assert mla.mla_decode_plan(1, 3, 48, 100, "bf16").fold == 1   # 48*3 > 128
    assert mla.mla_decode_plan(1, 6, 20, 100, "bf16").fold == 6   # 120 <= 128


@pytest.mark.parametrize("batch,q_len,heads,n", [(1, 1, 16, 256), (4, 4, 32, 8192), (4, 4, 32, 81920),
                                                  (16, 4, 32, 81920), (32, 4, 64, 65536),
                                                  (128, 2, 128, 81920), (3, 1, 8, 1), (2, 2, 2, 0)])
def test_split_covers_all_keys(batch, q_len, heads, n):
    # the fixed-split rule (the SIMT kernel and plans past the balanced unit limit use it)
    p = mla.mla_decode_plan_custom(batch, q_len, heads, n, "bf16", kernel="simt")
    tiles = math.ceil(n / 64)
    assert p.keys_per_split % 64 == 0 and p.keys_per_split >= 64
    assert p.split_kv * p.keys_per_split >= n
    assert 1 <= p.split_kv <= max(1, tiles)
    # no empty trailing split
    assert (p.split_kv - 1) * p.keys_per_split < max(n, 1)


def test_workspace_holds_the_partials():
    for (b, t, h, n) in [(4, 4, 32, 81920), (16, 4, 32, 81920), (1, 1, 16, 256)]:
        # fixed splits: [rows, S, 512] partials
        p = mla.mla_decode_plan_custom(b, t, h, n, "fp8", kernel="tcgen05_solo")
        assert p.schedule == 0
        rows = b * t * h
        if p.split_kv > 1:
            assert p.partial_offset >= 256 and p.partial_offset % 256 == 0
            assert p.lse_offset >= p.partial_offset + rows * p.split_kv * 512 * 4
            assert p.workspace_bytes >= p.lse_offset + rows * p.split_kv * 4
        assert p.workspace_bytes >= 256 and p.workspace_bytes % 256 == 0
        # balanced CTA-pair schedule: the status header and the unit
        # completion counters (units + 1 int32, cleared before each launch),
        # 2P slots of M rows, then the unit table
        p = mla.mla_decode_plan(b, t, h, n, "fp8")
        assert p.schedule == 1 and p.kernel == 1 and p.num_ctas == 2 * p.split_kv
        slot_rows = 2 * p.split_kv * p.rows_per_unit
        units = b * p.q_groups
        assert p.partial_offset >= 256 + (units + 1) * 4 and p.partial_offset % 256 == 0
        assert p.lse_offset >= p.partial_offset + slot_rows * 512 * 4 and p.lse_offset % 256 == 0
        assert p.workspace_bytes >= p.lse_offset + slot_rows * 4 + (units + 2) * 4
        assert p.split_kv * p.keys_per_split >= n


def test_balanced_plan_uses_every_sm_and_caps_units():
    p = mla.mla_decode_plan(16, 4, 32, 81920, "fp8")
    assert (p.schedule, p.split_kv, p.num_ctas) == (1, 74, 148)
    assert mla.mla_decode_plan_custom(16, 4, 32, 81920, "fp8", split_kv=5).split_kv == 5
    assert mla.mla_decode_plan_custom(16, 4, 32, 81920, "fp8", split_kv=1000).split_kv == 74
    # more units than the per-pair piece list can hold: fixed splits, solo kernel
    big = mla.mla_decode_plan(20000, 1, 16, 1024, "fp8")
    assert big.schedule == 0 and big.kernel == 3
    # 16-bit inputs take the balanced schedule too (16-bit CTA-pair kernel),
    # and past the unit limit fixed splits on the exchange kernel
    assert mla.mla_decode_plan(16, 4, 32, 81920, "bf16").schedule == 1
    assert mla.mla_decode_plan(128, 2, 128, 81920, "bf16").schedule == 1
    big16 = mla.mla_decode_plan(20000, 1, 16, 1024, "fp16")
    assert big16.schedule == 0 and big16.kernel == 1


LEAD = 24  # weight of a piece transition, charged at the start of every unit with tiles


def _lead(u, t):
    return LEAD if t > 0 else 0


def _balanced_schedule(tiles, P, weights=None, min_weight=4):
    """Host model of the device schedule: a tile weighs 2, or 3 with FP8 two-term P, and every
    unit with tiles starts with a lead-in of LEAD (the cost of moving on to a new unit); pair p
    takes the tiles whose weighted start lies in [W p / np, W (p + 1) / np).
    Returns unit starts, W, np, each pair's pieces (u, t0, t1) and each pair's first unit
    (-1: none)."""
    weights = weights or [2] * len(tiles)
    starts = [0]
    for u, (t, w) in enumerate(zip(tiles, weights)):
        starts.append(starts[-1] + _lead(u, t) + t * w)
    W = starts[-1]
    np_ = max(1, min(P, W // min_weight))
    pieces = []
    for p in range(P):
        lo, hi = (W * p // np_, W * (p + 1) // np_) if p < np_ else (W, W)
        pp = []
        for u, (t, w) in enumerate(zip(tiles, weights)):
            s0 = starts[u] + _lead(u, t)  # weighted start of the unit's first tile
            i0 = min(t, -(-(lo - s0) // w)) if lo > s0 else 0
            i1 = min(t, -(-(hi - s0) // w)) if hi > s0 else 0
            if i1 > i0:
                pp.append((u, i0, i1))
        pieces.append(pp)
    first = [pp[0][0] if pp else -1 for pp in pieces]
    return starts, W, np_, pieces, first


def _pair_of(x, W, np_):
    return ((x + 1) * np_ + W - 1) // W - 1


_rng = __import__("random").Random(5)
_MIXED = [_rng.choice([0, 1, 2, 7, 130, 640]) for _ in range(300)]


@pytest.mark.parametrize("tiles,weights", [
    ([640] * 16, None), ([1, 0, 3, 2], None), ([2] * 2048, None), ([190, 3, 0, 640, 1, 1, 77] * 9, None),
    ([5], None), ([0, 0, 4], None), ([1] * 250 + [157] * 50, None),
    ([640] * 16, [2, 3] * 8), ([1, 0, 3, 2], [3, 3, 2, 3]), (_MIXED, [_rng.choice([2, 3]) for _ in _MIXED]),
    ([3] * 1000 + [400] * 7, [3] * 1000 + [2] * 7),
])
def test_balanced_schedule_covers_each_tile_once(tiles, weights):
    """Every tile of every unit lies in exactly one piece; a pair leaves at most two partial
    pieces (its first and last): a cut piece that begins inside its unit (t0 > 0) in slot 2p,
    one that begins at the unit's start in slot 2p + 1, never both in one slot; the combine's
    rule (the pairs of the unit's first and last tile starts; slot 2p0 + 1 for the first, 2q for
    every later one) finds the same slots, and every pair it waits for holds a piece of the
    unit."""
    P = 74
    w_of = weights or [2] * len(tiles)
    starts, W, np_, pieces, first = _balanced_schedule(tiles, P, weights)
    seen = {}
    slot_of_piece = {}
    for p, pp in enumerate(pieces):
        for k, (u, t0, t1) in enumerate(pp):
            for t in range(t0, t1):
                assert (u, t) not in seen
                seen[(u, t)] = p
            whole = t0 == 0 and t1 == tiles[u]
            if not whole:
                assert k == 0 or k == len(pp) - 1
                assert t0 == 0 or k == 0  # only a pair's first piece begins inside its unit
                assert t0 > 0 or k == len(pp) - 1  # a cut piece from the unit's start is the last
                slot = 2 * p + (0 if t0 > 0 else 1)
                assert slot not in slot_of_piece.values()
                slot_of_piece[(u, p)] = slot
    assert len(seen) == sum(tiles)
    for u, t in enumerate(tiles):
        if t == 0:
            continue
        p0 = _pair_of(starts[u] + _lead(u, t), W, np_)
        p1 = _pair_of(starts[u + 1] - w_of[u], W, np_)
        assert seen[(u, 0)] == p0 and seen[(u, t - 1)] == p1
        if p0 == p1:
            assert (u, p0) not in slot_of_piece  # whole: written directly
            continue
        for q in range(p0, p1 + 1):
            assert any(pu == u for pu, _, _ in pieces[q])  # the combine's wait ends
            slot = 2 * q + 1 if q == p0 else 2 * q
            assert slot_of_piece[(u, q)] == slot


def _tile_work(pp, weights):
    return sum((t1 - t0) * weights[u] for u, t0, t1 in pp)


def _lead_overlap(starts, tiles, W, np_, p):
    """Weight of the units' lead-ins that lies inside pair p's range."""
    lo, hi = W * p // np_, W * (p + 1) // np_
    return sum(max(0, min(hi, starts[u] + _lead(u, t)) - max(lo, starts[u])) for u, t in enumerate(tiles))


def test_weighted_schedule_evens_out_two_term_work():
    # half the units have two-term tiles (weight 3): per-pair weight stays within one tile
    tiles = [100] * 40
    weights = [3] * 20 + [2] * 20
    starts, W, np_, pieces, _ = _balanced_schedule(tiles, 74, weights)
    load = [_tile_work(pp, weights) + _lead_overlap(starts, tiles, W, np_, p) for p, pp in enumerate(pieces)]
    # tile work plus the lead-in weight inside the range stays within a tile of the range size
    assert max(load) - min(load) <= 2 * 3


def test_lead_in_gives_pairs_that_cross_a_unit_boundary_fewer_tiles():
    # 16 entries of 640 pair tiles (the 80K-key FP8 batch): a pair whose range holds a unit start
    # pays a piece transition, so it takes up to LEAD / 2 fewer tiles; tile work plus the lead-in
    # weight a pair holds stays within one tile of every other pair's
    tiles = [640] * 16
    starts, W, np_, pieces, _ = _balanced_schedule(tiles, 74)
    work = [_tile_work(pp, [2] * 16) for pp in pieces]
    load = [w + _lead_overlap(starts, tiles, W, np_, p) for p, w in enumerate(work)]
    assert max(load) - min(load) <= 2 * 2
    # a pair whose range holds a lead-in (a unit start) takes fewer tiles than one that holds none
    held = [_lead_overlap(starts, tiles, W, np_, p) for p in range(len(pieces))]
    with_lead = [w for w, h in zip(work, held) if h > 0]
    without = [w for w, h in zip(work, held) if h == 0]
    assert with_lead and without and max(with_lead) < min(without)
    assert all(h > 0 for p, h in enumerate(held) if len(pieces[p]) == 2)


def test_split_fills_the_gpu_for_the_long_fp8_case():
    p4 = mla.mla_decode_plan_custom(4, 4, 32, 81920, "fp8", kernel="tcgen05_solo")
    assert p4.split_kv * 4 <= 74 and p4.split_kv * 4 >= 60  # one wave of CTA pairs
    p16 = mla.mla_decode_plan_custom(16, 4, 32, 81920, "fp8", kernel="tcgen05_solo")
    waves = math.ceil(p16.split_kv * 16 / 74)
    assert p16.split_kv * 16 / (waves * 74) > 0.85  # little wave quantisation


def test_plan_is_deterministic_and_forced_values_apply():
    a = mla.mla_decode_plan(4, 4, 32, 8192, "bf16").as_dict()
    b = mla.mla_decode_plan(4, 4, 32, 8192, "bf16").as_dict()
    assert a == b
    p = mla.mla_decode_plan_custom(4, 4, 32, 8192, "bf16", split_kv=3, kernel="simt")
    assert p.split_kv == 3 and p.keys_per_split == 64 * math.ceil(128 / 3)
    p = mla.mla_decode_plan_custom(4, 4, 32, 8192, "bf16", split_kv=10 ** 6, kernel="simt")
    assert p.split_kv == 128 and p.keys_per_split == 64
    # the balanced schedule takes a forced split as the number of CTA pairs
    p = mla.mla_decode_plan_custom(4, 4, 32, 8192, "bf16", split_kv=3)
    assert (p.schedule, p.split_kv, p.num_ctas) == (1, 3, 6)
    p = mla.mla_decode_plan_custom(4, 4, 32, 8192, "bf16", fold=2)
    assert (p.fold, p.q_groups, p.rows_per_unit) == (2, 2, 64)
    p = mla.mla_decode_plan_custom(4, 4, 32, 8192, "bf16", kernel="simt")
    assert p.kernel == 2


@pytest.mark.parametrize("args,code", [
    ((-1, 1, 16, 10, "bf16"), -1), ((1, 0, 16, 10, "bf16"), -1), ((1, 1, 0, 10, "bf16"), -1),
    ((1, 1, 16, -5, "bf16"), -1), ((1, 1, 16, 10, 7), -1), ((1, 1, 129, 10, "bf16"), -2),
])
def test_plan_errors(args, code):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan(*args)
    assert e.value.code == code


def test_forced_fold_must_divide():
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan_custom(1, 4, 16, 10, "bf16", fold=3)
    assert e.value.code == -2
    with pytest.raises(mla.MlaError):
        mla.mla_decode_plan_custom(1, 4, 64, 10, "bf16", fold=4)  # 256 rows


def test_window_is_set_only_on_plans_whose_kernels_support_it():
    p = mla.mla_decode_plan(2, 4, 32, 4096, "fp8")
    assert p.window == 0 and p.schedule == 1
    ws = p.workspace_bytes
    assert mla.mla_decode_plan_window(p, 300).window == 300
    assert p.workspace_bytes == ws  # the window changes no buffer
    assert mla.mla_decode_plan_window(p, 0).window == 0
    p16 = mla.mla_decode_plan(2, 4, 32, 4096, "bf16")
    assert mla.mla_decode_plan_window(p16, 64).window == 64
    ps = mla.mla_decode_plan_custom(2, 4, 32, 4096, "fp16", kernel="simt")
    assert mla.mla_decode_plan_window(ps, 1).window == 1
    # fixed-split tensor-core plans (the FP8 solo kernel, the 16-bit exchange
    # kernel past the balanced unit limit) do not take a window
    solo = mla.mla_decode_plan_custom(2, 4, 32, 4096, "fp8", kernel="tcgen05_solo")
    big16 = mla.mla_decode_plan_custom(17000, 1, 16, 256, "bf16")
    assert big16.schedule == 0
    for q in (solo, big16):
        with pytest.raises(mla.MlaError) as e:
            mla.mla_decode_plan_window(q, 128)
        assert e.value.code == -2 and q.window == 0
        assert mla.mla_decode_plan_window(q, 0).window == 0
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan_window(p, -1)
    assert e.value.code == -1
    forged = mla.MlaPlan.from_buffer_copy(p)
    forged.magic = 0
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan_window(forged, 8)
    assert e.value.code == -6


def test_prefill_plan_folds_without_dividing_and_counts_groups():
    # ragged queries: the largest F with H * F <= 128, whether or not it divides max_q_len
    p = mla.mla_prefill_plan(3, 5, 48, 1000, "bf16")
    assert (p.varlen, p.fold, p.q_groups, p.rows_per_unit, p.schedule) == (1, 2, 3, 96, 1)
    p = mla.mla_prefill_plan(2, 4096, 32, 20480, "fp8")
    assert (p.fold, p.q_groups, p.kernel, p.schedule, p.split_kv) == (4, 1024, 1, 1, 74)
    p = mla.mla_prefill_plan(2, 3, 16, 100, "fp16")  # F = 3 <= max_q_len
    assert (p.fold, p.q_groups) == (3, 1)
    # the SIMT cross-check takes fixed splits; the solo FP8 kernel has no ragged form
    p = mla.mla_prefill_plan(2, 100, 16, 5000, "fp8", kernel="simt")
    assert (p.varlen, p.schedule, p.kernel) == (1, 0, 2)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_plan(2, 100, 16, 5000, "fp8", kernel="tcgen05_solo")
    assert e.value.code == -2
    # more than 65536 groups in all
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_plan(17, 4096, 128, 8192, "bf16")
    assert e.value.code == -2
    # a decode plan of the same numbers is not ragged
    assert mla.mla_decode_plan(2, 4, 32, 100, "bf16").varlen == 0


def test_balanced_workspace_holds_the_piece_spill():
    """After the partial slots: two CTAs' spill lists of U + P pieces (12 bytes) and the unit table."""
    p = mla.mla_prefill_plan(8, 4096, 32, 20480, "fp8")
    units = 8 * 1024
    need = (p.lse_offset + 2 * p.split_kv * p.rows_per_unit * 4
            + (2 * (units + p.split_kv) * 12 + 255) // 256 * 256 + ((units + 2) * 4 + 255) // 256 * 256)
    assert p.workspace_bytes >= need


def test_window_applies_to_prefill_plans():
    p = mla.mla_prefill_plan(2, 500, 32, 5000, "fp8")
    ws = p.workspace_bytes
    assert mla.mla_decode_plan_window(p, 256).window == 256 and p.varlen == 1 and p.workspace_bytes == ws
    s = mla.mla_prefill_plan(2, 500, 32, 5000, "bf16", kernel="simt")
    assert mla.mla_decode_plan_window(s, 1).window == 1
    # the fixed-split workspace of a ragged plan holds batch x max_q_len x H rows of partials
    if s.split_kv > 1:
        assert s.lse_offset - s.partial_offset >= 2 * 500 * 32 * s.split_kv * 512 * 4


@pytest.mark.parametrize("seed", range(5))
def test_spilled_piece_lists_of_different_pairs_never_overlap(seed):
    """A pair's spill list starts at entry u_first + p (per CTA rank, U + P entries each) and
    holds one piece per unit its range meets: the lists of all pairs fit and never overlap."""
    import random
    rnd = random.Random(seed)
    U, P = rnd.choice([50, 300, 3000]), 74
    tiles = [rnd.choice([0, 0, 1, 1, 2, 5, 40, 300]) for _ in range(U)]
    weights = [rnd.choice([2, 3]) for _ in range(U)]
    _, _, _, pieces, first = _balanced_schedule(tiles, P, weights)
    used = set()
    for p, pp in enumerate(pieces):
        if not pp:
            continue
        base = first[p] + p
        for k in range(len(pp)):
            idx = base + k
            assert 0 <= idx < U + P and idx not in used
            used.add(idx)


def _sched_unit(B, G, varlen, s):
    """Host mirror of sched_unit: decode plans with G > 1 query groups order the schedule
    group-major (slot s = g * B + b holds unit b * G + g); ragged prefill keeps entry order."""
    return (s % B) * G + s // B if (not varlen and G > 1) else s


def _sched_slot(B, G, varlen, u):
    return (u % G) * B + u // G if (not varlen and G > 1) else u


@pytest.mark.parametrize("B,G,varlen", [(1, 1, 0), (16, 1, 0), (32, 2, 0), (128, 2, 0), (3, 4, 0), (7, 3, 1),
                                        (5, 1024, 1)])
def test_schedule_slot_order_is_a_bijection_and_group_major_for_decode(B, G, varlen):
    U = B * G
    units = [_sched_unit(B, G, varlen, s) for s in range(U)]
    assert sorted(units) == list(range(U))
    assert all(_sched_slot(B, G, varlen, u) == s for s, u in enumerate(units))
    if not varlen and G > 1:
        # the first B slots are group 0 of every entry, in entry order
        assert units[:B] == [b * G for b in range(B)]
    else:
        assert units == list(range(U))


def test_group_major_order_puts_both_groups_of_an_entry_on_pairs_half_the_sequence_apart():
    # 128 entries x 2 groups of equal length (the high-concurrency shape): pair p and pair p + np/2
    # cover the same entries' key tiles, so their reads of a page are close in time
    B, G, t = 128, 2, 50
    tiles = [t] * (B * G)  # in slot order (group-major)
    starts, W, np_, pieces, _ = _balanced_schedule(tiles, 74)
    half = np_ // 2
    for p in range(half):
        a = {(_sched_unit(B, G, 0, s) // G, i) for s, t0, t1 in pieces[p] for i in range(t0, t1)}
        b = {(_sched_unit(B, G, 0, s) // G, i) for s, t0, t1 in pieces[p + half] for i in range(t0, t1)}
        # the same (entry, key tile) sets: both halves of the sequence weigh the same
        assert a == b


def _unit_span(n, qlen, g, F, window):
    """The unit geometry's key span [klo, kend) restated: rows of tokens g*F .. of an entry with
    n keys and qlen new tokens (token t sees keys up to n - qlen + t, its last `window` if set)."""
    t0 = g * F
    tu = min(F, qlen - t0)
    if tu <= 0:
        return 0, 0, 0
    nq = n - qlen + t0
    kend = max(0, nq + tu)
    klo = max(0, nq + 1 - window) if window > 0 else 0
    return tu, klo, kend


@pytest.mark.parametrize("window", [0, 1, 7, 100])
def test_unit_span_is_the_union_of_its_rows_visible_keys(window):
    import random
    rnd = random.Random(window)
    for _ in range(300):
        F = rnd.choice([1, 2, 4, 8])
        qlen = rnd.randint(0, 40)
        n = rnd.randint(0, 200)
        for g in range((max(qlen, 1) + F - 1) // F + 1):
            tu, klo, kend = _unit_span(n, qlen, g, F, window)
            keys = set()
            for t in range(g * F, g * F + max(tu, 0)):
                last = n - qlen + t
                first = max(0, last + 1 - window) if window > 0 else 0
                keys |= set(range(first, last + 1))
            if keys:
                assert (klo, kend) == (min(keys), max(keys) + 1)
            else:
                assert kend <= klo or tu <= 0
