"""MLA paged-decode oracle (fp64, CPU).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package; the product path
(``mla_paged_decode_04_b200``) never does, and shares no code with it.

``mla_decode`` wraps the C implementation in ``mla_oracle.c`` (plain
definition, fp64, OpenMP over rows). ``brute.py`` holds an independent
pure-Python restatement used to pin the C code on tiny inputs.

Every function states the passage it follows; the definition is the one in
``mla_oracle.c``'s header (tokenspeed-mla package card, "What it is and what
it does"; TokenSpeed MLA article 最快MLA内核背后的秘密, sections 一, 二, 四, 六).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_mla.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"bf16": 0, "fp16": 1, "fp8": 2}

# Planted mistakes for the pin-sensitivity tests (see mla_oracle.c).
MUTATIONS = {
    "none": 0,
    "drop_rope": 1,
    "v_offset": 2,
    "no_causal": 3,
    "no_scale": 4,
    "lse_log2": 5,
    "page_index": 6,
    "wrong_sign": 7,
}


def build(force: bool = False) -> str:
    """Compile mla_oracle.c into liboracle_mla.so (gcc -O3 -fopenmp, no fast-math)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                   "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        vp = ctypes.c_void_p
        lib.oracle_mla_decode_range.argtypes = [
            i32, i32, i32, i32, i32, i32, vp, vp, i64, i32, vp, i32, vp,
            f64, f64, f64, i64, vp, i64, i64, i32, vp, vp]
        lib.oracle_mla_decode_range.restype = i32
        lib.oracle_mla_decode_range_w.argtypes = [
            i32, i32, i32, i32, i32, i32, vp, vp, i64, i32, vp, i32, vp,
            f64, f64, f64, i64, vp, i64, i64, i64, i32, vp, vp]
        lib.oracle_mla_decode_range_w.restype = i32
        lib.oracle_lse_merge.argtypes = [i32, i32, vp, vp, vp, vp]
        lib.oracle_lse_merge.restype = None
        lib.oracle_decode_buffer.argtypes = [i32, vp, ctypes.c_size_t, vp]
        lib.oracle_decode_buffer.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        lib.oracle_set_num_threads.argtypes = [i32]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_encode_e4m3_buffer.argtypes = [vp, ctypes.c_size_t, vp]
        lib.oracle_encode_e4m3_buffer.restype = None
        lib.oracle_kv_pack.argtypes = [i32, i32, vp, vp, i64, vp, ctypes.c_float, vp, i64]
        lib.oracle_kv_pack.restype = i32
        lib.oracle_kv_amax.argtypes = [i32, vp, vp, i64]
        lib.oracle_kv_amax.restype = f64
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops from now on (timing only: a row is always
    computed by one thread, so results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


def _raw_bytes(t) -> np.ndarray:
    """Raw element bytes of a CPU tensor / ndarray as a contiguous uint8 array."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().contiguous().cpu()
            return t.view(torch.uint8).numpy().reshape(-1)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    return a.view(np.uint8).reshape(-1)


def decode_values(dtype: str, raw) -> np.ndarray:
    """Decode raw element bytes (bf16 / fp16 / E4M3FN) to float64 with the oracle's own decoder."""
    b = _raw_bytes(raw)
    esize = 1 if dtype == "fp8" else 2
    n = b.size // esize
    out = np.empty(n, dtype=np.float64)
    _load().oracle_decode_buffer(DTYPE_CODES[dtype], b.ctypes.data, n, out.ctypes.data)
    return out


def mla_decode(q, kv_cache, block_tables, seq_lens, softmax_scale, *, dtype,
               q_scale=1.0, kv_scale=1.0, rows=None, key_range=None, window=0,
               mutation="none"):
    """Oracle MLA decode.

    q: [B, q_len, H, D] and kv_cache: [num_pages, page_size, D] CPU tensors (bf16 /
    fp16 / float8_e4m3fn, or their raw uint8/uint16 views); block_tables [B, P]
    int32, seq_lens [B] int32. rows: optional flat row indices (b*q_len+t)*H+h.
    key_range: optional (lo, hi) restriction of the keys (hi=-1: unbounded).
    window: sliding window W > 0 (a row with n visible keys sees keys >= n - W); 0 = none.
    Returns (out [n_rows, Dv=512] float64, lse [n_rows] float64), natural log.
    """
    lib = _load()
    B, T, H, D = (int(x) for x in q.shape)
    num_pages, page_size, D2 = (int(x) for x in kv_cache.shape)
    assert D2 == D
    Dv = 512
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    assert bt.ndim == 2 and bt.shape[0] == B and sl.shape == (B,)
    qb = _raw_bytes(q)
    cb = _raw_bytes(kv_cache)
    if rows is None:
        n_rows = B * T * H
        rows_ptr = None
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n_rows = rows_arr.size
        rows_ptr = rows_arr.ctypes.data
    out = np.zeros((n_rows, Dv), dtype=np.float64)
    lse = np.zeros((n_rows,), dtype=np.float64)
    lo, hi = (0, -1) if key_range is None else key_range
    rc = lib.oracle_mla_decode_range_w(
        DTYPE_CODES[dtype], B, T, H, D, Dv, qb.ctypes.data, cb.ctypes.data, num_pages,
        page_size, bt.ctypes.data, bt.shape[1], sl.ctypes.data, float(softmax_scale),
        float(q_scale), float(kv_scale), n_rows, rows_ptr, int(lo), int(hi), int(window),
        MUTATIONS[mutation], out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_mla_decode_range failed with code {rc}")
    return out, lse


def mla_prefill(q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, *, dtype,
                q_scale=1.0, kv_scale=1.0, rows=None, window=0):
    """Oracle ragged (prefill) attention over the paged cache.

    tokenspeed-mla package card, "What it is and what it does": prefill of
    variable-length sequences packed without padding. Entry b's new tokens
    are q[cu[b]:cu[b+1]] (q: [total_q, H, D]); token t of the entry sees keys
    0 .. seq_lens[b] - q_len_b + t, which is the decode definition with
    q_len = q_len_b, so each entry is one call of `mla_decode`.
    rows: optional packed row indices token*H + h (each inside some entry).
    Returns (out [n_rows, 512] float64, lse [n_rows] float64).
    """
    cu = [int(x) for x in np.asarray(cu_seqlens_q).reshape(-1)]
    total_q, H, D = (int(x) for x in q.shape)
    B = len(cu) - 1
    bt = np.asarray(block_tables, dtype=np.int32)
    sl = np.asarray(seq_lens, dtype=np.int32)
    all_rows = np.arange(total_q * H) if rows is None else np.asarray(rows, dtype=np.int64).reshape(-1)
    out = np.zeros((all_rows.size, 512))
    lse = np.zeros(all_rows.size)
    tok = all_rows // H
    done = np.zeros(all_rows.size, dtype=bool)
    for b in range(B):
        s, e = cu[b], cu[b + 1]
        sel = np.nonzero((tok >= s) & (tok < e))[0]
        if sel.size == 0:
            continue
        qb = q[s:e].reshape(1, e - s, H, D)
        o, l = mla_decode(qb, kv_cache, bt[b:b + 1], sl[b:b + 1], softmax_scale, dtype=dtype,
                          q_scale=q_scale, kv_scale=kv_scale, rows=all_rows[sel] - s * H, window=window)
        out[sel] = o
        lse[sel] = l
        done[sel] = True
    if not done.all():
        raise ValueError("a requested row lies outside every entry")
    return out, lse


def lse_merge(o_parts, lse_parts):
    """Merge per-split partials of one row: returns (out [Dv], lse)."""
    o = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    n, Dv = o.shape
    out = np.zeros(Dv, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    _load().oracle_lse_merge(n, Dv, o.ctypes.data, l.ctypes.data, out.ctypes.data,
                             lse.ctypes.data)
    return out, float(lse[0])


def encode_e4m3(values) -> np.ndarray:
    """OCP E4M3FN codes of fp32 values: round to nearest even, saturating to +-448, NaN -> S.1111.111
    (0x7f, or 0xff when the NaN's sign bit is set)."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32).reshape(-1))
    out = np.empty(v.size, dtype=np.uint8)
    _load().oracle_encode_e4m3_buffer(v.ctypes.data, v.size, out.ctypes.data)
    return out


def kv_pack(latent, rope, slot_mapping, cache_shape, *, in_dtype, cache_dtype, kv_scale=1.0, cache=None):
    """Oracle fused K/V pack (+ FP8 quantise): cache row slot_mapping[i] = [latent_i || rope_i].

    latent [n, 512] and rope [n, 64] are 16-bit tensors (raw bytes are read);
    the cache (raw element bytes, shape [num_pages, page_size, 576]) starts as
    `cache` (or zeros) and is returned as a uint8 array of those bytes.
    """
    lat = _raw_bytes(latent)
    rp = _raw_bytes(rope)
    n = lat.size // (512 * 2)
    slots = np.ascontiguousarray(np.asarray(slot_mapping, dtype=np.int64).reshape(-1))
    assert slots.size == n and rp.size == n * 64 * 2
    esize = 1 if cache_dtype == "fp8" else 2
    num_slots = int(np.prod(cache_shape[:-1]))
    buf = np.zeros(num_slots * 576 * esize, dtype=np.uint8) if cache is None else _raw_bytes(cache).copy()
    rc = _load().oracle_kv_pack(DTYPE_CODES[in_dtype], DTYPE_CODES[cache_dtype], lat.ctypes.data, rp.ctypes.data,
                                n, slots.ctypes.data, float(kv_scale), buf.ctypes.data, num_slots)
    if rc != 0:
        raise ValueError(f"oracle kv_pack failed ({rc})")
    return buf


def kv_amax(latent, rope, *, in_dtype) -> float:
    """Largest |x| over the non-NaN elements of the latent and rope tensors."""
    lat = _raw_bytes(latent)
    rp = _raw_bytes(rope)
    n = lat.size // (512 * 2)
    return float(_load().oracle_kv_amax(DTYPE_CODES[in_dtype], lat.ctypes.data, rp.ctypes.data, n))
