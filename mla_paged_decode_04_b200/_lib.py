"""ctypes binding of libmla_decode.so (argument marshalling only).

The functions carry the C ABI's names (include/mla_decode.h) and pass raw
device pointers and the current CUDA stream; every step of the decode runs
in the library's kernels. PyTorch is used only to own device memory and
streams. If the shared library is missing this module raises at import: there
is no fallback path. With MLA_DECODE_BOUNDS_CHECK=1 in the environment the
bounds-checking build, libmla_decode_check.so, is loaded instead (slower; its
kernels set MLA_DEV_BOUNDS instead of accessing memory outside a buffer).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
NORMAL_LIB_PATH = os.path.join(_HERE, "libmla_decode.so")
CHECK_LIB_PATH = os.path.join(_HERE, "libmla_decode_check.so")
LIB_PATH = CHECK_LIB_PATH if os.environ.get("MLA_DECODE_BOUNDS_CHECK", "0") == "1" else NORMAL_LIB_PATH

MLA_BF16, MLA_FP16, MLA_FP8_E4M3 = 0, 1, 2
DTYPES = {"bf16": MLA_BF16, "fp16": MLA_FP16, "fp8": MLA_FP8_E4M3}
MLA_KERNEL_AUTO, MLA_KERNEL_TCGEN05, MLA_KERNEL_SIMT, MLA_KERNEL_TCGEN05_SOLO = 0, 1, 2, 3
KERNELS = {"auto": MLA_KERNEL_AUTO, "tcgen05": MLA_KERNEL_TCGEN05, "simt": MLA_KERNEL_SIMT,
           "tcgen05_solo": MLA_KERNEL_TCGEN05_SOLO}

MLA_DEV_BAD_PAGE, MLA_DEV_SEQ_TOO_LONG, MLA_DEV_TIMEOUT, MLA_DEV_BAD_QLEN, MLA_DEV_BOUNDS = 0x1, 0x2, 0x4, 0x8, 0x10
(MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED_SHAPE, MLA_ERR_WORKSPACE_TOO_SMALL, MLA_ERR_ARCH, MLA_ERR_CUDA,
 MLA_ERR_PLAN_MISMATCH) = (-1, -2, -3, -4, -5, -6)

EXPORTED = ["mla_decode_plan", "mla_decode_plan_custom", "mla_decode", "mla_decode_partial",
            "mla_decode_combine", "mla_decode_status", "mla_status_string", "mla_version",
            "mla_decode_no_alloc", "mla_decode_no_alloc_status", "mla_last_cuda_error", "mla_kv_pack", "mla_kv_amax",
            "mla_decode_plan_window", "mla_prefill_plan", "mla_prefill_plan_custom", "mla_prefill",
            "mla_prefill_partial", "mla_prefill_combine", "mla_bounds_checked"]
MLA_NO_ALLOC_SCRATCH_BYTES = 48 << 20


class MlaPlan(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("num_heads", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("fold", ctypes.c_int32), ("q_groups", ctypes.c_int32), ("rows_per_unit", ctypes.c_int32),
        ("split_kv", ctypes.c_int32), ("keys_per_split", ctypes.c_int32),
        ("kernel", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
        ("workspace_bytes", ctypes.c_uint64), ("partial_offset", ctypes.c_uint64),
        ("lse_offset", ctypes.c_uint64), ("magic", ctypes.c_uint32), ("schedule", ctypes.c_uint32),
        ("window", ctypes.c_int32), ("varlen", ctypes.c_int32), ("fault_test", ctypes.c_int32),
    ]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what} failed: {status_string(code)} ({code})"
        self.cuda_error = None
        if code == -5:  # MLA_ERR_CUDA: name the CUDA runtime error behind it
            self.cuda_error = last_cuda_error()
            msg += f" [{self.cuda_error[1]} ({self.cuda_error[0]})]"
        super().__init__(msg)
        self.code = code


def load_library(path):
    """The library at `path` (the normal or the bounds-checking build) with its argument types set."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python mla_paged_decode_04_b200/build.py"
            f"{' --check' if path == CHECK_LIB_PATH else ''}` (there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    i32, i64, u64, f32, vp = (ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float,
                              ctypes.c_void_p)
    P = ctypes.POINTER(MlaPlan)
    lib.mla_decode_plan.argtypes = [i32, i32, i32, i32, i32, P]
    lib.mla_decode_plan.restype = i32
    lib.mla_decode_plan_custom.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P]
    lib.mla_decode_plan_custom.restype = i32
    for name in ("mla_decode", "mla_decode_partial", "mla_decode_combine"):
        fn = getattr(lib, name)
        fn.argtypes = [P, vp, vp, i64, i32, vp, i32, vp, f32, f32, f32, vp, vp, vp, u64, vp]
        fn.restype = i32
    lib.mla_decode_status.argtypes = [vp, vp, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.mla_decode_status.restype = i32
    lib.mla_status_string.argtypes = [i32]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_version.argtypes = []
    lib.mla_version.restype = ctypes.c_char_p
    lib.mla_last_cuda_error.argtypes = [ctypes.POINTER(ctypes.c_char_p)]
    lib.mla_last_cuda_error.restype = i32
    lib.mla_prefill_plan.argtypes = [i32, i32, i32, i32, i32, P]
    lib.mla_prefill_plan.restype = i32
    lib.mla_prefill_plan_custom.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P]
    lib.mla_prefill_plan_custom.restype = i32
    for name in ("mla_prefill", "mla_prefill_partial", "mla_prefill_combine"):
        fn = getattr(lib, name)
        fn.argtypes = [P, vp, i64, vp, vp, i64, i32, vp, i32, vp, f32, f32, f32, vp, vp, vp, u64, vp]
        fn.restype = i32
    lib.mla_decode_plan_window.argtypes = [P, i32]
    lib.mla_decode_plan_window.restype = i32
    lib.mla_kv_pack.argtypes = [vp, vp, i64, vp, vp, i64, i32, i32, i32, f32, vp, vp]
    lib.mla_kv_pack.restype = i32
    lib.mla_kv_amax.argtypes = [vp, vp, i64, i32, vp, vp]
    lib.mla_kv_amax.restype = i32
    lib.mla_bounds_checked.argtypes = []
    lib.mla_bounds_checked.restype = i32
    return lib


_lib = load_library(LIB_PATH)


def bounds_checked() -> bool:
    """True when the loaded library is the bounds-checking build."""
    return bool(_lib.mla_bounds_checked())


def lib():
    return _lib


def status_string(code: int) -> str:
    return _lib.mla_status_string(int(code)).decode()


def last_cuda_error():
    """(code, name) of the CUDA runtime error behind this thread's last MLA_ERR_CUDA."""
    name = ctypes.c_char_p()
    code = _lib.mla_last_cuda_error(ctypes.byref(name))
    return int(code), (name.value.decode() if name.value else "")


def mla_version() -> str:
    return _lib.mla_version().decode()


def _dtype_code(dtype) -> int:
    if isinstance(dtype, str):
        return DTYPES[dtype]
    if dtype == torch.bfloat16:
        return MLA_BF16
    if dtype == torch.float16:
        return MLA_FP16
    if dtype == torch.float8_e4m3fn:
        return MLA_FP8_E4M3
    return int(dtype)


def mla_decode_plan(batch, q_len, num_heads, max_seq_len, dtype) -> MlaPlan:
    p = MlaPlan()
    rc = _lib.mla_decode_plan(batch, q_len, num_heads, max_seq_len, _dtype_code(dtype), ctypes.byref(p))
    if rc != 0:
        raise MlaError(rc, "mla_decode_plan")
    return p


def mla_decode_plan_custom(batch, q_len, num_heads, max_seq_len, dtype, split_kv=0, fold=0,
                           kernel="auto") -> MlaPlan:
    p = MlaPlan()
    k = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    rc = _lib.mla_decode_plan_custom(batch, q_len, num_heads, max_seq_len, _dtype_code(dtype),
                                     split_kv, fold, k, ctypes.byref(p))
    if rc != 0:
        raise MlaError(rc, "mla_decode_plan_custom")
    return p


def mla_decode_plan_window(plan: MlaPlan, window: int) -> MlaPlan:
    """Set the plan's sliding window in place (0 = full attention) and return it."""
    rc = _lib.mla_decode_plan_window(ctypes.byref(plan), int(window))
    if rc != 0:
        raise MlaError(rc, "mla_decode_plan_window")
    return plan


def mla_prefill_plan(batch, max_q_len, num_heads, max_seq_len, dtype, split_kv=0, fold=0,
                     kernel="auto") -> MlaPlan:
    """Plan of a ragged-query (prefill) shape: max_q_len = the most new tokens an entry may have."""
    p = MlaPlan()
    k = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    rc = _lib.mla_prefill_plan_custom(batch, max_q_len, num_heads, max_seq_len, _dtype_code(dtype),
                                      split_kv, fold, k, ctypes.byref(p))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_plan")
    return p


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_tensors(q, **named):
    """Every tensor argument is a contiguous CUDA tensor on q's device."""
    if not (isinstance(q, torch.Tensor) and q.is_cuda):
        raise ValueError("q must be a CUDA tensor")
    for k, t in named.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != q.device:
            raise ValueError(f"{k} must be a CUDA tensor on {q.device} (got "
                             f"{t.device if isinstance(t, torch.Tensor) else type(t).__name__})")
        if not t.is_contiguous():
            raise ValueError(f"{k} must be contiguous")
    for k in ("block_tables", "seq_lens"):
        t = named.get(k)
        if t is not None and t.dtype != torch.int32:
            raise ValueError(f"{k} must be int32")


def _call(name, plan, q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse, workspace,
          q_scale, kv_scale, stream):
    _check_tensors(q, kv_cache=kv_cache, block_tables=block_tables, seq_lens=seq_lens, out=out,
                   lse=lse, workspace=workspace)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream if q.is_cuda else 0
    elif isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    num_pages, page_size = int(kv_cache.shape[0]), int(kv_cache.shape[1])
    rc = getattr(_lib, name)(ctypes.byref(plan), _ptr(q), _ptr(kv_cache), num_pages, page_size,
                         _ptr(block_tables), int(block_tables.shape[1]), _ptr(seq_lens),
                         float(softmax_scale), float(q_scale), float(kv_scale), _ptr(out),
                         _ptr(lse), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                         ctypes.c_void_p(stream))
    if rc != 0:
        raise MlaError(rc, name)


def mla_decode(plan: MlaPlan, q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
               workspace, q_scale=1.0, kv_scale=1.0, stream=None) -> None:
    """Enqueue one decode step on `stream` (default: torch's current stream).

    Tensors are device tensors in the layouts of include/mla_decode.h; `out`
    (bf16 [B, q_len, H, 512]), `lse` (fp32 [B, q_len, H] or None) and
    `workspace` (uint8, >= plan.workspace_bytes, 256-byte aligned) are written.
    """
    _call("mla_decode", plan, q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
          workspace, q_scale, kv_scale, stream)


def mla_decode_partial(plan: MlaPlan, q, kv_cache, block_tables, seq_lens, softmax_scale, out,
                       lse, workspace, q_scale=1.0, kv_scale=1.0, stream=None) -> None:
    """First kernel only (split-KV partials; writes out/lse itself when split_kv == 1)."""
    _call("mla_decode_partial", plan, q, kv_cache, block_tables, seq_lens, softmax_scale, out,
          lse, workspace, q_scale, kv_scale, stream)


def mla_decode_combine(plan: MlaPlan, q, kv_cache, block_tables, seq_lens, softmax_scale, out,
                       lse, workspace, q_scale=1.0, kv_scale=1.0, stream=None) -> None:
    """Second kernel only (LSE merge of the partials; no-op when split_kv == 1)."""
    _call("mla_decode_combine", plan, q, kv_cache, block_tables, seq_lens, softmax_scale, out,
          lse, workspace, q_scale, kv_scale, stream)


def _call_prefill(name, plan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
                  workspace, q_scale, kv_scale, stream):
    _check_tensors(q, cu_seqlens_q=cu_seqlens_q, kv_cache=kv_cache, block_tables=block_tables,
                   seq_lens=seq_lens, out=out, lse=lse, workspace=workspace)
    if cu_seqlens_q is None or cu_seqlens_q.dtype != torch.int32:
        raise ValueError("cu_seqlens_q must be an int32 CUDA tensor")
    num_pages, page_size = int(kv_cache.shape[0]), int(kv_cache.shape[1])
    rc = getattr(_lib, name)(ctypes.byref(plan), _ptr(q), int(q.shape[0]), _ptr(cu_seqlens_q), _ptr(kv_cache),
                             num_pages, page_size, _ptr(block_tables), int(block_tables.shape[1]), _ptr(seq_lens),
                             float(softmax_scale), float(q_scale), float(kv_scale), _ptr(out), _ptr(lse),
                             _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                             ctypes.c_void_p(_stream_of(q, stream)))
    if rc != 0:
        raise MlaError(rc, name)


def mla_prefill(plan: MlaPlan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
                workspace, q_scale=1.0, kv_scale=1.0, stream=None) -> None:
    """Enqueue one ragged prefill step: q [total_q, H, 576] packed, cu_seqlens_q int32 [B + 1],
    out bf16 [total_q, H, 512], lse fp32 [total_q, H] or None (include/mla_decode.h)."""
    _call_prefill("mla_prefill", plan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, out,
                  lse, workspace, q_scale, kv_scale, stream)


def mla_prefill_partial(plan: MlaPlan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, out,
                        lse, workspace, q_scale=1.0, kv_scale=1.0, stream=None) -> None:
    """First kernel of mla_prefill only."""
    _call_prefill("mla_prefill_partial", plan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale,
                  out, lse, workspace, q_scale, kv_scale, stream)


def mla_decode_status(workspace, clear=True, stream=None) -> int:
    """Synchronise and read the device status word (MLA_DEV_* bits)."""
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device).cuda_stream
    v = ctypes.c_int32(0)
    rc = _lib.mla_decode_status(_ptr(workspace), ctypes.c_void_p(stream), int(bool(clear)),
                                ctypes.byref(v))
    if rc != 0:
        raise MlaError(rc, "mla_decode_status")
    return int(v.value)


def _stream_of(t, stream):
    if stream is None:
        return torch.cuda.current_stream(t.device).cuda_stream
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else stream


def kv_pack(latent, rope, slot_mapping, kv_cache, kv_scale=1.0, device_status=None, stream=None) -> None:
    """Write tokens into the paged cache, fused with FP8 quantisation when kv_cache is FP8.

    latent [n, 512] and rope [n, 64] (bf16 or fp16), slot_mapping [n] int64
    (page * 64 + offset; negative = skip), kv_cache [num_pages, 64, 576] of
    the inputs' dtype or float8_e4m3fn; see include/mla_decode.h.
    """
    _check_tensors(latent, rope=rope, slot_mapping=slot_mapping, kv_cache=kv_cache, device_status=device_status)
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    if latent.dtype != rope.dtype:
        raise ValueError("latent and rope must have one dtype")
    in_dtype = _dtype_code(latent.dtype)
    cache_dtype = _dtype_code(kv_cache.dtype)
    rc = _lib.mla_kv_pack(_ptr(latent), _ptr(rope), int(latent.shape[0]), _ptr(slot_mapping), _ptr(kv_cache),
                          int(kv_cache.shape[0]), int(kv_cache.shape[1]), in_dtype, cache_dtype, float(kv_scale),
                          _ptr(device_status), ctypes.c_void_p(_stream_of(latent, stream)))
    if rc != 0:
        raise MlaError(rc, "mla_kv_pack")


def kv_amax(latent, rope, out=None, stream=None) -> torch.Tensor:
    """Device fp32 [1]: the largest |x| over latent and rope (NaN ignored)."""
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=latent.device)
    _check_tensors(latent, rope=rope, out=out)
    rc = _lib.mla_kv_amax(_ptr(latent), _ptr(rope), int(latent.shape[0]), _dtype_code(latent.dtype), _ptr(out),
                          ctypes.c_void_p(_stream_of(latent, stream)))
    if rc != 0:
        raise MlaError(rc, "mla_kv_amax")
    return out


def alloc_workspace(plan: MlaPlan, device) -> torch.Tensor:
    """A zeroed workspace tensor of plan.workspace_bytes (torch allocations are 256-byte aligned)."""
    return torch.zeros(int(plan.workspace_bytes), dtype=torch.uint8, device=device)


class MlaDecoder:
    """Plan + workspace for one decode shape; call it once per decode step."""

    def __init__(self, batch, q_len, num_heads, max_seq_len, dtype, device, split_kv=0, fold=0,
                 kernel="auto", window=0):
        self.plan = mla_decode_plan_custom(batch, q_len, num_heads, max_seq_len, dtype,
                                           split_kv, fold, kernel)
        if window:
            mla_decode_plan_window(self.plan, window)
        self.device = torch.device(device)
        self.workspace = alloc_workspace(self.plan, self.device)
        self.batch, self.q_len, self.num_heads = batch, q_len, num_heads

    def __call__(self, q, kv_cache, block_tables, seq_lens, softmax_scale, q_scale=1.0,
                 kv_scale=1.0, out=None, lse=None, want_lse=True, stream=None):
        B, T, H = self.batch, self.q_len, self.num_heads
        if out is None:
            out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=self.device)
        if lse is None and want_lse:
            lse = torch.empty((B, T, H), dtype=torch.float32, device=self.device)
        mla_decode(self.plan, q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
                   self.workspace, q_scale, kv_scale, stream)
        return out, lse

    def status(self, clear=True) -> int:
        return mla_decode_status(self.workspace, clear)


class MlaPrefill:
    """Plan + workspace for one ragged prefill shape (batch, longest entry, H, longest sequence)."""

    def __init__(self, batch, max_q_len, num_heads, max_seq_len, dtype, device, split_kv=0, fold=0,
                 kernel="auto", window=0):
        self.plan = mla_prefill_plan(batch, max_q_len, num_heads, max_seq_len, dtype, split_kv, fold, kernel)
        if window:
            mla_decode_plan_window(self.plan, window)
        self.device = torch.device(device)
        self.workspace = alloc_workspace(self.plan, self.device)
        self.num_heads = num_heads

    def __call__(self, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, q_scale=1.0,
                 kv_scale=1.0, out=None, lse=None, want_lse=True, stream=None):
        total_q, H = int(q.shape[0]), self.num_heads
        if out is None:
            out = torch.empty((total_q, H, 512), dtype=torch.bfloat16, device=self.device)
        if lse is None and want_lse:
            lse = torch.empty((total_q, H), dtype=torch.float32, device=self.device)
        mla_prefill(self.plan, q, cu_seqlens_q, kv_cache, block_tables, seq_lens, softmax_scale, out, lse,
                    self.workspace, q_scale, kv_scale, stream)
        return out, lse

    def status(self, clear=True) -> int:
        return mla_decode_status(self.workspace, clear)
