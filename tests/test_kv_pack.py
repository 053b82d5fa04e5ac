"""Fused K/V pack + FP8 quantise: oracle pins (CPU) and bit-exact GPU parity.

The operation (tokenspeed-mla package card, "What it is and what it does";
TokenSpeed MLA article, section 一 kernel table and section 六 row layout):
cache row slot_mapping[i] = [latent_i (512) || rope_i (64)], each element
E4M3FN(x / kv_scale) with the quotient in fp32, or a copy for a 16-bit cache.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200 import _lib


# ---------------------------------------------------------------- oracle pins (CPU)

def _codes_and_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.decode_values("fp8", codes)
    return codes, vals


def test_e4m3_encode_round_trips_every_finite_code():
    codes, vals = _codes_and_values()
    fin = ~np.isnan(vals)
    assert fin.sum() == 254  # S.1111.111 is NaN for both signs
    assert np.array_equal(oracle.encode_e4m3(vals[fin].astype(np.float32)), codes[fin])


def test_e4m3_encode_ties_go_to_the_even_code():
    codes, vals = _codes_and_values()
    for c in range(0, 0x7e):  # positive finite codes and their upper neighbour
        lo, hi = vals[c], vals[c + 1]
        mid = (lo + hi) / 2  # exact in fp32 (both have <= 4 significant bits)
        want = c if c % 2 == 0 else c + 1
        assert oracle.encode_e4m3(np.float32(mid))[0] == want, hex(c)
        # just off the midpoint: the nearer code
        below = np.nextafter(np.float32(mid), np.float32(0))
        above = np.nextafter(np.float32(mid), np.float32(1e9))
        assert oracle.encode_e4m3(below)[0] == c and oracle.encode_e4m3(above)[0] == c + 1, hex(c)
        # the sign is a separate bit
        assert oracle.encode_e4m3(np.float32(-mid))[0] == (want | 0x80)


def test_e4m3_encode_saturates_and_keeps_nan():
    enc = lambda v: int(oracle.encode_e4m3(np.float32(v))[0])
    assert enc(448.0) == 0x7e and enc(-448.0) == 0xfe
    for v in (449.0, 463.9, 464.0, 480.0, 1e30, math.inf):
        assert enc(v) == 0x7e and enc(-v) == 0xfe
    assert enc(math.nan) & 0x7f == 0x7f
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    # subnormal steps are 2^-9: a quarter step rounds to 0, a half step ties to 0 (even),
    # one and a half steps tie up to 2
    assert enc(2.0 ** -11) == 0 and enc(2.0 ** -10) == 0 and enc(3 * 2.0 ** -10) == 2
    # the largest subnormal rounds up into the smallest normal 2^-6 (code 0x08)
    assert enc(7.75 * 2.0 ** -9) == 0x08


def test_e4m3_encode_matches_the_library_cast_in_range():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 3)
    x = x[x.abs() <= 448]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(x.numpy()), ref)


def _rand_tokens(n, dtype, seed, std=1.0, specials=False):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    lat = (torch.randn(n, 512, generator=g) * std).to(tdt)
    rope = (torch.randn(n, 64, generator=g) * std).to(tdt)
    if specials and n >= 4:
        lat[0, :6] = torch.tensor([0.0, -0.0, 1e-8, -3e4, float("nan"), 6e4]).to(tdt)
        rope[1, :3] = torch.tensor([-5e4, 5e3, -1e-7]).to(tdt)
    return lat, rope


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_e4m3_of_a_quotient_is_sign_symmetric(dtype):
    """The FP8 pack's table path encodes only the non-negative 16-bit patterns and sets the sign bit
    for the negative ones. That holds because x / s is -(|x| / s) exactly for s > 0 and the E4M3
    rounding is symmetric: checked here over every non-NaN 16-bit pattern, with the quotient in
    fp32 as the kernels form it, for scales that put values in the subnormal, normal and saturating
    ranges."""
    pos = np.arange(0x8000, dtype=np.uint16)
    x_pos = oracle.decode_values(dtype, pos).astype(np.float32)
    x_neg = oracle.decode_values(dtype, pos | np.uint16(0x8000)).astype(np.float32)
    keep = ~np.isnan(x_pos)
    for s in (0.37, 1.0, 3.0e-3, 2.5e2, 1.0e-6):
        with np.errstate(over="ignore"):  # large values over a small scale overflow to +-inf (saturated)
            q_pos = x_pos / np.float32(s)
            q_neg = x_neg / np.float32(s)
        assert np.array_equal(q_neg[keep], -q_pos[keep])
        c_pos = oracle.encode_e4m3(q_pos[keep])
        c_neg = oracle.encode_e4m3(q_neg[keep])
        assert np.array_equal(c_neg, c_pos | np.uint8(0x80))


def test_oracle_kv_pack_row_layout_and_skipped_slots():
    lat, rope = _rand_tokens(3, "bf16", 3)
    slots = np.array([5, -1, 0], dtype=np.int64)
    scale = 0.03125
    init = np.full(8 * 576, 0xAB, dtype=np.uint8).reshape(1, 8, 576)
    out = oracle.kv_pack(lat, rope, slots, (1, 8, 576), in_dtype="bf16", cache_dtype="fp8",
                         kv_scale=scale, cache=init).reshape(8, 576)
    for i, s in ((0, 5), (2, 0)):
        row = np.concatenate([lat[i].float().numpy(), rope[i].float().numpy()]).astype(np.float32)
        assert np.array_equal(out[s], oracle.encode_e4m3(row / np.float32(scale)))
    untouched = [r for r in range(8) if r not in (0, 5)]
    assert (out[untouched] == 0xAB).all()  # the skipped token wrote nothing
    # a 16-bit cache takes the bits unchanged, latent first
    out16 = oracle.kv_pack(lat, rope, slots, (1, 8, 576), in_dtype="bf16", cache_dtype="bf16")
    rows16 = out16.view(np.uint16).reshape(8, 576)
    assert np.array_equal(rows16[5, :512], lat[0].view(torch.uint16).numpy())
    assert np.array_equal(rows16[5, 512:], rope[0].view(torch.uint16).numpy())
    with pytest.raises(ValueError):
        oracle.kv_pack(lat, rope, np.array([0, 1, 8]), (1, 8, 576), in_dtype="bf16", cache_dtype="fp8")


def test_oracle_kv_amax_ignores_nan():
    lat, rope = _rand_tokens(17, "fp16", 4, std=3.0, specials=True)
    a = np.concatenate([lat.float().numpy().reshape(-1), rope.float().numpy().reshape(-1)])
    assert oracle.kv_amax(lat, rope, in_dtype="fp16") == np.nanmax(np.abs(a))


def test_kv_pack_host_errors_before_any_launch():
    L = _lib.lib()
    vp = None
    # page size, dtypes and scale are checked before anything touches a device
    assert L.mla_kv_pack(vp, vp, 4, vp, vp, 10, 32, 0, 2, 1.0, vp, vp) == _lib.MLA_ERR_UNSUPPORTED_SHAPE
    assert L.mla_kv_pack(vp, vp, 4, vp, vp, 10, 64, 2, 2, 1.0, vp, vp) == _lib.MLA_ERR_INVALID_ARG
    assert L.mla_kv_pack(vp, vp, 4, vp, vp, 10, 64, 0, 1, 1.0, vp, vp) == _lib.MLA_ERR_INVALID_ARG
    assert L.mla_kv_pack(vp, vp, 4, vp, vp, 10, 64, 0, 2, 0.0, vp, vp) == _lib.MLA_ERR_INVALID_ARG
    assert L.mla_kv_pack(vp, vp, -1, vp, vp, 10, 64, 0, 2, 1.0, vp, vp) == _lib.MLA_ERR_INVALID_ARG
    assert L.mla_kv_pack(vp, vp, 0, vp, vp, 10, 64, 0, 2, 1.0, vp, vp) == 0  # no tokens: no-op
    assert L.mla_kv_pack(vp, vp, 4, vp, vp, 10, 64, 0, 2, 1.0, vp, vp) == _lib.MLA_ERR_INVALID_ARG  # null
    assert L.mla_kv_amax(vp, vp, 4, 0, vp, vp) == _lib.MLA_ERR_INVALID_ARG


# ---------------------------------------------------------------- GPU parity (bit-exact)

def _assert_same_codes(got, ref):
    """Byte for byte, except that a NaN may come out as either E4M3 NaN code: the sign of a NaN that a
    division produces is unspecified (IEEE 754, section 6.3), and S.1111.111 is NaN for either S. The
    GPU's division returns its canonical (positive) NaN, the host's keeps the operand's sign."""
    diff = got != ref
    nan_pair = ((got & 0x7F) == 0x7F) & ((ref & 0x7F) == 0x7F)
    assert not (diff & ~nan_pair).any(), f"{int((diff & ~nan_pair).sum())} bytes differ"


def _gpu_case(n, dtype, cache_dtype, num_pages, seed, skip_every=7, specials=True):
    dev = torch.device("cuda", 0)
    lat, rope = _rand_tokens(n, dtype, seed, std=2.0, specials=specials)
    g = torch.Generator().manual_seed(seed + 1)
    slots = torch.randperm(num_pages * 64, generator=g)[:n].to(torch.int64)
    slots[::skip_every] = -1
    cdt = torch.float8_e4m3fn if cache_dtype == "fp8" else lat.dtype
    init = torch.randint(0, 256, (num_pages * 64 * 576 * (1 if cache_dtype == "fp8" else 2),), generator=g,
                         dtype=torch.uint8)
    cache = init.clone().to(dev).view(cdt).view(num_pages, 64, 576)
    return dev, lat, rope, slots, cache, init


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_kv_pack_fp8_matches_the_oracle_bit_for_bit(dtype):
    n, num_pages = 1000, 40
    dev, lat, rope, slots, cache, init = _gpu_case(n, dtype, "fp8", num_pages, seed=11)
    dl, dr, ds = lat.to(dev), rope.to(dev), slots.to(dev)
    amax = mla.kv_amax(dl, dr)
    scale = float(amax.item()) / 448.0
    assert float(amax.item()) == oracle.kv_amax(lat, rope, in_dtype=dtype)
    mla.kv_pack(dl, dr, ds, cache, kv_scale=scale)
    torch.cuda.synchronize()
    ref = oracle.kv_pack(lat, rope, slots.numpy(), (num_pages, 64, 576), in_dtype=dtype, cache_dtype="fp8",
                         kv_scale=scale, cache=init.numpy())
    got = cache.view(torch.uint8).reshape(-1).cpu().numpy()
    _assert_same_codes(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_kv_pack_16bit_cache_copies_the_rows(dtype):
    n, num_pages = 333, 12
    dev, lat, rope, slots, cache, init = _gpu_case(n, dtype, dtype, num_pages, seed=12)
    mla.kv_pack(lat.to(dev), rope.to(dev), slots.to(dev), cache)
    torch.cuda.synchronize()
    ref = oracle.kv_pack(lat, rope, slots.numpy(), (num_pages, 64, 576), in_dtype=dtype, cache_dtype=dtype,
                         cache=init.numpy())
    assert np.array_equal(cache.view(torch.uint8).reshape(-1).cpu().numpy(), ref)


@pytest.mark.gpu
def test_kv_pack_bad_slot_sets_the_status_and_writes_the_rest():
    n, num_pages = 64, 4
    dev, lat, rope, slots, cache, init = _gpu_case(n, "bf16", "fp8", num_pages, seed=13, specials=False)
    slots[5] = num_pages * 64 + 3  # past the cache
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # a small scale: |x| / scale passes 448 for most values, so saturation is exercised
    mla.kv_pack(lat.to(dev), rope.to(dev), slots.to(dev), cache, kv_scale=0.005, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == mla.MLA_DEV_BAD_PAGE
    ok = slots.clone()
    ok[5] = -1
    ref = oracle.kv_pack(lat, rope, ok.numpy(), (num_pages, 64, 576), in_dtype="bf16", cache_dtype="fp8",
                         kv_scale=0.005, cache=init.numpy())
    _assert_same_codes(cache.view(torch.uint8).reshape(-1).cpu().numpy(), ref)


@pytest.mark.gpu
def test_kv_pack_full_size_prefill_matches_the_oracle():
    # one 80K-token entry written at once (the prefill-sized call), permuted pages
    n, num_pages = 81920, 1400
    dev, lat, rope, slots, cache, init = _gpu_case(n, "bf16", "fp8", num_pages, seed=14, skip_every=10 ** 9,
                                                   specials=False)
    dl, dr = lat.to(dev), rope.to(dev)
    scale = float(mla.kv_amax(dl, dr).item()) / 448.0
    mla.kv_pack(dl, dr, slots.to(dev), cache, kv_scale=scale)
    torch.cuda.synchronize()
    ref = oracle.kv_pack(lat, rope, slots.numpy(), (num_pages, 64, 576), in_dtype="bf16", cache_dtype="fp8",
                         kv_scale=scale, cache=init.numpy())
    _assert_same_codes(cache.view(torch.uint8).reshape(-1).cpu().numpy(), ref)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_kv_pack_table_path_encodes_every_bit_pattern(dtype):
    """Calls of more than ~50K tokens encode through a per-CTA table of the non-negative input patterns. The
    latent dims of tokens 1..128 hold every 16-bit pattern once (NaN, infinities, subnormals and -0
    included), one token's slot is past the cache; bit-exact against the oracle (a NaN as either NaN
    code), and the status word reports the bad slot."""
    n, num_pages = 52000, 850
    dev, lat, rope, slots, cache, init = _gpu_case(n, dtype, "fp8", num_pages, seed=15, skip_every=10 ** 9)
    # tokens 1..128 (token 0's slot is the one _gpu_case always skips)
    lat.view(torch.int16)[1:129].reshape(-1)[:] = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
    slots[200] = num_pages * 64 + 5
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 0.37
    mla.kv_pack(lat.to(dev), rope.to(dev), slots.to(dev), cache, kv_scale=scale, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == mla.MLA_DEV_BAD_PAGE
    ok = slots.clone()
    ok[200] = -1
    ref = oracle.kv_pack(lat, rope, ok.numpy(), (num_pages, 64, 576), in_dtype=dtype, cache_dtype="fp8",
                         kv_scale=scale, cache=init.numpy())
    got = cache.view(torch.uint8).reshape(-1).cpu().numpy()
    _assert_same_codes(got, ref)
    # every NaN input did become a NaN code
    nan_in = np.isnan(lat[1:129].float().numpy()).reshape(-1)
    rows = slots[1:129].numpy()
    codes = got.reshape(-1, 576)[rows][:, :512].reshape(-1)
    assert ((codes[nan_in] & 0x7F) == 0x7F).all()
