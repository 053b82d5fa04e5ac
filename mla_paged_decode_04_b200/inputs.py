"""Seeded synthetic inputs for MLA paged decode.

This module only draws random numbers and lays them out; it holds none of
the decode arithmetic, so both the CUDA path and the oracle consume its
output. Shapes follow the pages' workloads (TokenSpeed MLA article
最快MLA内核背后的秘密, sections 一-三: q_len 4, 16-64 heads, 64K-80K
contexts, FP8 caches; section 六 for the tensor layouts):

* q           [B, q_len, H, 576]    bf16 / fp16 / float8_e4m3fn
* kv_cache    [num_pages, 64, 576]  same dtype as q
* block_tables[B, max_pages]        int32, unused slots -1
* seq_lens    [B]                   int32, counting this step's q_len tokens

Draw order (one ``torch.Generator`` per workload, seed = 1000 + config
number, on the CPU or directly on the GPU for the large pools): seq_lens, q,
cache, page permutation. FP8 tensors are drawn in fp32, scaled per tensor by
amax/448 and cast round-to-nearest-even to E4M3FN.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

D_QK = 576
D_V = 512
PAGE_SIZE = 64
FP8_MAX = 448.0

_TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp8": torch.float8_e4m3fn}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (sizes and value distributions)."""

    name: str
    config: int            # 1-based workload number; the seed is 1000 + config
    batch: int
    q_len: int
    heads: int
    dtype: str             # "bf16" | "fp16" | "fp8"
    seq: tuple             # ("fixed", n) | ("uniform", lo, hi) | ("lognormal", median, sigma, cap)
    pool: object           # "exact" or a float factor over the pages needed
    q_std: float = 1.0
    kv_std: float = 1.0
    description: str = ""

    @property
    def max_seq_len(self) -> int:
        kind = self.seq[0]
        if kind == "fixed":
            return int(self.seq[1])
        if kind == "uniform":
            return int(self.seq[2])
        return int(self.seq[3])


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_bf16", 1, 1, 1, 16, "bf16", ("fixed", 256), "exact", 1.0, 1.0,
                 "B=1 q_len=1 H=16 seq_len=256, 4 pages permuted, q and cache N(0,1)"),
        Workload("mtp_bf16", 2, 4, 4, 32, "bf16", ("fixed", 8192), 2.0, 1.0, 0.5,
                 "B=4 q_len=4 H=32 seq_len=8192, pool 2x, q N(0,1), cache N(0,0.5^2)"),
        Workload("fp8_long_b4", 3, 4, 4, 32, "fp8", ("fixed", 81920), 2.0, 1.0, 1.0,
                 "FP8 E4M3 q and cache, per-tensor scales, q_len=4 H=32 seq_len=81920, B=4"),
        Workload("fp8_long_b16", 3, 16, 4, 32, "fp8", ("fixed", 81920), 2.0, 1.0, 1.0,
                 "FP8 E4M3 q and cache, per-tensor scales, q_len=4 H=32 seq_len=81920, B=16"),
        Workload("fold_fp16_h16", 4, 32, 4, 16, "fp16", ("uniform", 1024, 65536), 2.0, 1.0, 1.0,
                 "FP16 B=32 q_len=4 H=16 (fold 4), seq_lens U[1024,65536]"),
        Workload("fold_fp16_h64", 4, 32, 4, 64, "fp16", ("uniform", 1024, 65536), 2.0, 1.0, 1.0,
                 "FP16 B=32 q_len=4 H=64 (fold 2), seq_lens U[1024,65536]"),
        Workload("highconc_bf16", 5, 128, 2, 128, "bf16", ("lognormal", 16384, 1.0, 81920), 2.0,
                 1.0, 0.5, "BF16 B=128 q_len=2 H=128, seq_lens lognormal median 16K sigma 1 cap 80K"),
    ]
}


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor
    kv_cache: torch.Tensor
    block_tables: torch.Tensor
    seq_lens: torch.Tensor
    dtype: str
    softmax_scale: float
    q_scale: float = 1.0
    kv_scale: float = 1.0
    max_seq_len: int = 0
    name: str = "custom"

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])

    @property
    def q_len(self) -> int:
        return int(self.q.shape[1])

    @property
    def heads(self) -> int:
        return int(self.q.shape[2])

    @property
    def num_pages(self) -> int:
        return int(self.kv_cache.shape[0])

    def to(self, device, non_blocking: bool = False) -> "DecodeInputs":
        return dataclasses.replace(
            self,
            q=self.q.to(device, non_blocking=non_blocking),
            kv_cache=self.kv_cache.to(device, non_blocking=non_blocking),
            block_tables=self.block_tables.to(device, non_blocking=non_blocking),
            seq_lens=self.seq_lens.to(device, non_blocking=non_blocking),
        )

    def kv_tokens(self) -> int:
        return int(self.seq_lens.clamp(min=0).sum().item())


def _draw(shape, g: torch.Generator, std: float, dtype: str, chunk: int = 1 << 26):
    """N(0, std^2) draw cast to the workload dtype, chunk by chunk.

    FP8 gets one per-tensor scale amax/448: a first pass over the chunks finds
    amax, then the generator state is rewound and the same numbers are drawn
    again and cast round-to-nearest-even to E4M3FN. Returns (tensor, scale).
    """
    n = math.prod(shape)
    dev = g.device
    out = torch.empty(n, dtype=_TORCH_DTYPES[dtype], device=dev)
    scale = 1.0
    if dtype == "fp8":
        state = g.get_state()
        amax = 0.0
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            x = torch.randn(e - s, generator=g, dtype=torch.float32, device=dev)
            amax = max(amax, float(x.abs().max().item()) * std)
        scale = amax / FP8_MAX if amax > 0 else 1.0
        scale = float(torch.tensor(scale, dtype=torch.float32).item())  # exactly an fp32 number
        g.set_state(state)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=g, dtype=torch.float32, device=dev)
        if std != 1.0:
            x.mul_(std)
        if dtype == "fp8":
            x.div_(scale).clamp_(-FP8_MAX, FP8_MAX)
        out[s:e] = x.to(out.dtype)
    return out.view(*shape), scale


def draw_seq_lens(w: Workload, g: torch.Generator) -> torch.Tensor:
    kind = w.seq[0]
    if kind == "fixed":
        return torch.full((w.batch,), int(w.seq[1]), dtype=torch.int32)
    if kind == "uniform":
        lo, hi = int(w.seq[1]), int(w.seq[2])
        return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64,
                             device=g.device).to(torch.int32).cpu()
    if kind == "lognormal":
        median, sigma, cap = float(w.seq[1]), float(w.seq[2]), int(w.seq[3])
        z = torch.randn(w.batch, generator=g, dtype=torch.float64, device=g.device).cpu()
        n = torch.exp(math.log(median) + sigma * z).round().clamp(2, cap)
        return n.to(torch.int32)
    raise ValueError(kind)


def make_inputs_custom(batch: int, q_len: int, heads: int, dtype: str,
                       seq_lens: Sequence[int], *, seed: int, pool="exact",
                       q_std: float = 1.0, kv_std: float = 1.0, page_size: int = PAGE_SIZE,
                       max_pages: Optional[int] = None, name: str = "custom",
                       softmax_scale: Optional[float] = None,
                       device="cpu") -> DecodeInputs:
    """Inputs for explicit seq_lens (used by tests for ragged and edge cases)."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    sl = torch.tensor([int(x) for x in seq_lens], dtype=torch.int32)
    return _build(batch, q_len, heads, dtype, sl, g, pool, q_std, kv_std, page_size,
                  max_pages, name, softmax_scale)


def make_inputs(name: str, device="cpu", batch: Optional[int] = None) -> DecodeInputs:
    """Inputs of a named workload (see WORKLOADS), seed 1000 + config number.

    The generator lives on ``device``: the bytes are reproducible per device
    type, and the oracle always consumes the same bytes as the GPU path.
    Small tensors (block tables, seq_lens) are returned on the CPU. `batch`
    draws the same distributions with that many entries (a smaller case of
    the workload, e.g. for profiler captures).
    """
    w = WORKLOADS[name]
    if batch is not None:
        w = dataclasses.replace(w, batch=int(batch))
    g = torch.Generator(device=device).manual_seed(1000 + w.config)
    sl = draw_seq_lens(w, g)
    return _build(w.batch, w.q_len, w.heads, w.dtype, sl, g, w.pool, w.q_std, w.kv_std,
                  PAGE_SIZE, None, name, None, max_seq_len=w.max_seq_len)


def _build(batch, q_len, heads, dtype, sl, g, pool, q_std, kv_std, page_size, max_pages,
           name, softmax_scale, max_seq_len=None) -> DecodeInputs:
    pages_needed = [(int(n) + page_size - 1) // page_size for n in sl.tolist()]
    total_needed = sum(pages_needed)
    if pool == "exact":
        num_pages = max(1, total_needed)
    else:
        num_pages = max(1, int(math.ceil(float(pool) * total_needed)))
    width = max_pages if max_pages is not None else max(1, max(pages_needed) if pages_needed else 1)
    if max_seq_len is None:
        max_seq_len = int(sl.max().item()) if batch > 0 else 0
    q, q_scale = _draw((batch, q_len, heads, D_QK), g, q_std, dtype)
    cache, kv_scale = _draw((num_pages, page_size, D_QK), g, kv_std, dtype)
    perm = torch.randperm(num_pages, generator=g, device=g.device).to(torch.int32).cpu()
    bt = torch.full((batch, width), -1, dtype=torch.int32)
    off = 0
    for b, npg in enumerate(pages_needed):
        bt[b, :npg] = perm[off:off + npg]
        off += npg
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    return DecodeInputs(q=q, kv_cache=cache, block_tables=bt, seq_lens=sl, dtype=dtype,
                        softmax_scale=float(softmax_scale), q_scale=q_scale, kv_scale=kv_scale,
                        max_seq_len=int(max_seq_len), name=name)


def kv_bytes(inp: DecodeInputs) -> int:
    """Bytes of distinct cache rows a decode step must read (each token once)."""
    esize = 1 if inp.dtype == "fp8" else 2
    return inp.kv_tokens() * D_QK * esize


# ---------------------------------------------------------------- ragged prefill
@dataclasses.dataclass
class PrefillInputs:
    """A ragged prefill step: entry b's q_lens[b] new tokens (packed in q) extend a cached
    prefix of prefix_lens[b] tokens; seq_lens = prefix + new, all already in the cache."""
    q: torch.Tensor             # [total_q, H, 576]
    cu_seqlens_q: torch.Tensor  # int32 [B + 1]
    kv_cache: torch.Tensor
    block_tables: torch.Tensor
    seq_lens: torch.Tensor
    dtype: str
    softmax_scale: float
    q_scale: float = 1.0
    kv_scale: float = 1.0
    max_q_len: int = 0
    max_seq_len: int = 0
    name: str = "custom"

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def total_q(self) -> int:
        return int(self.q.shape[0])

    def to(self, device) -> "PrefillInputs":
        return dataclasses.replace(self, q=self.q.to(device), cu_seqlens_q=self.cu_seqlens_q.to(device),
                                   kv_cache=self.kv_cache.to(device), block_tables=self.block_tables.to(device),
                                   seq_lens=self.seq_lens.to(device))


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    seed: int
    batch: int
    heads: int
    dtype: str
    q_lens: tuple      # ("uniform", lo, hi)
    prefix: tuple      # ("uniform", lo, hi)
    max_q_len: int
    max_seq_len: int
    desc: str


PREFILL_WORKLOADS = {
    w.name: w
    for w in [
        PrefillWorkload("prefill_fp8", 2001, 8, 32, "fp8", ("uniform", 512, 4096), ("uniform", 0, 16384),
                        4096, 16384 + 4096,
                        "FP8 ragged prefill: B=8, H=32, new tokens U[512,4096], cached prefix U[0,16384]"),
        PrefillWorkload("prefill_bf16", 2002, 8, 32, "bf16", ("uniform", 512, 4096), ("uniform", 0, 16384),
                        4096, 16384 + 4096,
                        "BF16 ragged prefill: B=8, H=32, new tokens U[512,4096], cached prefix U[0,16384]"),
    ]
}


def make_prefill_inputs(q_lens: Sequence[int], prefix_lens: Sequence[int], heads: int, dtype: str, *,
                        seed: int, pool=1.5, q_std: float = 1.0, kv_std: float = 1.0,
                        max_q_len: Optional[int] = None, max_seq_len: Optional[int] = None,
                        name: str = "custom", device="cpu") -> PrefillInputs:
    """Seeded ragged prefill inputs: packed q [sum q_lens, H, 576], cu_seqlens_q, a permuted page
    pool of `pool` x the pages needed, block tables and seq_lens = prefix + new tokens."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    ql = [int(x) for x in q_lens]
    sl = torch.tensor([int(a) + int(b) for a, b in zip(ql, prefix_lens)], dtype=torch.int32)
    B = len(ql)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    if B:
        cu[1:] = torch.cumsum(torch.tensor(ql, dtype=torch.int64), 0).to(torch.int32)
    pages_needed = [(int(n) + PAGE_SIZE - 1) // PAGE_SIZE for n in sl.tolist()]
    num_pages = max(1, int(math.ceil(float(pool) * sum(pages_needed))))
    width = max(1, max(pages_needed) if pages_needed else 1)
    q, q_scale = _draw((max(int(cu[-1]), 0), heads, D_QK), g, q_std, dtype)
    cache, kv_scale = _draw((num_pages, PAGE_SIZE, D_QK), g, kv_std, dtype)
    perm = torch.randperm(num_pages, generator=g, device=g.device).to(torch.int32).cpu()
    bt = torch.full((B, width), -1, dtype=torch.int32)
    off = 0
    for b, npg in enumerate(pages_needed):
        bt[b, :npg] = perm[off:off + npg]
        off += npg
    return PrefillInputs(q=q, cu_seqlens_q=cu, kv_cache=cache, block_tables=bt, seq_lens=sl, dtype=dtype,
                         softmax_scale=D_QK ** -0.5, q_scale=q_scale, kv_scale=kv_scale,
                         max_q_len=int(max_q_len if max_q_len is not None else max(ql + [1])),
                         max_seq_len=int(max_seq_len if max_seq_len is not None else (int(sl.max()) if B else 0)),
                         name=name)


def make_prefill_workload(name: str, device="cpu", batch: Optional[int] = None) -> PrefillInputs:
    """Inputs of a named ragged prefill workload (lengths from its seed, on the CPU); `batch`
    draws that many entries of the same distributions instead."""
    w = PREFILL_WORKLOADS[name]
    if batch is not None:
        w = dataclasses.replace(w, batch=int(batch))
    gl = torch.Generator().manual_seed(w.seed)
    ql = torch.randint(w.q_lens[1], w.q_lens[2] + 1, (w.batch,), generator=gl).tolist()
    pre = torch.randint(w.prefix[1], w.prefix[2] + 1, (w.batch,), generator=gl).tolist()
    return make_prefill_inputs(ql, pre, w.heads, w.dtype, seed=w.seed + 1, pool=1.5, max_q_len=w.max_q_len,
                               max_seq_len=w.max_seq_len, name=name, device=device)
