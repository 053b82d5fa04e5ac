// Helpers shared by the tensor-core partial kernels: bounded waits, tensor
// maps over [rows, 576] arrays, and the epilogue store of a 32-column chunk.
#pragma once

#include <cuda.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr uint64_t kWaitLimitNs = 500ull * 1000 * 1000;  // per wait: 0.5 s

// Bounded wait on an mbarrier phase. Returns false (after setting the abort
// flag and MLA_DEV_TIMEOUT) when the limit passes, or when another role of
// the CTA has already aborted.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             int32_t* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 127) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(status, MLA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// The same with a CTA-scope acquire (see mbar_try_wait_cta).
__device__ __forceinline__ bool bounded_wait_cta(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                 int32_t* status) {
  if (ptx::mbar_try_wait_cta(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait_cta(bar, parity)) return true;
    if ((it & 127) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(status, MLA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool warp_wait_cta(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              int32_t* status) {
  const bool ok = bounded_wait_cta(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Warp-uniform bounded wait: every lane waits (and so acquires); the warp
// goes on only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
  const bool ok = bounded_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::globaltimer() - t0 < ns) {
  }
}

// Before the producer returns: wait (bounded, even after an abort) for the
// loads it issued into the last `stages` stages, so no copy lands after exit.
__device__ __forceinline__ void drain_loads(uint32_t full_bar0, int stages, int n_tiles) {
  for (int j = n_tiles - stages; j < n_tiles; ++j) {
    if (j < 0) continue;
    const uint32_t bar = full_bar0 + 8u * (uint32_t)(j % stages);
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, (j / stages) & 1) && ptx::globaltimer() - t0 < kWaitLimitNs) {
    }
  }
}

// Wait (bounded, whatever the abort flag says) for the phase of `bar` with
// the given parity to complete.
__device__ __forceinline__ void drain_phase(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity) && ptx::globaltimer() - t0 < kWaitLimitNs) {
  }
}

// The pair's two partial slots hold the previous call's pieces, which its
// combine has read (this kernel runs after it): their L2 lines are dropped
// without a write-back, instead of being written to DRAM while this call
// streams the cache. Each CTA drops the lines of its own 64 rows (with M a
// multiple of 8, a 128-byte line is 8 rows of one 16-byte chunk of a slot),
// long before its epilogue writes them again. Threads t0, t0 + nt, ... of the
// CTA take part. Only when the call streams more cache than the L2 holds
// (estimated from this pair's `tiles`, 72 KB of cache each in both pair
// kernels, times the pairs): otherwise the lines are simply overwritten in L2
// by the next call and dropping them would only cost L2 requests.
__device__ __forceinline__ void discard_pair_slots(const DecodeArgs& a, int pair, uint32_t rank, int tiles, int t0,
                                                   int nt) {
  constexpr int64_t kTileBytes = 128 * MLA_D_QK;  // a pair tile: 128 FP8 or 64 16-bit keys of 576 dims
  constexpr int64_t kL2Bytes = 126ll << 20;
  const int M = a.plan.rows_per_unit;
  if (!a.o_part || M % 8 != 0 || pair >= a.plan.split_kv) return;
  if ((int64_t)tiles * a.plan.split_kv * kTileBytes < kL2Bytes) return;
  const int groups = M / 8;                  // 8-row groups of a chunk
  const int per_slot = (MLA_D_V / 4) * groups;  // lines of a slot
  for (int i = t0; i < 2 * per_slot; i += nt) {
    const int g = i % groups;
    if (g / 8 != (int)rank) continue;  // rows [64 rank, 64 rank + 64)
    const int c4 = (i % per_slot) / groups;
    const int slot = 2 * pair + i / per_slot;
    ptx::discard_l2_line(a.o_part + (((int64_t)slot * (MLA_D_V / 4) + c4) * M + 8 * g) * 4);
  }
}

// Teardown drain of the CTA-pair kernels (layout L, barriers at bar0 + 8 i):
// the last phase of every barrier the leader's MMA commits arrive on, after
// `n_all` tiles and `npc` pieces. Lane k of the calling warp waits for one
// (barrier, parity): the last NK, NV and NQ phases of the K, V and S rings,
// the last two of P_EMPTY and S_FULL, then O_DONE and O_FINAL, so that the
// waits overlap instead of running one after another.
template <class L>
__device__ __forceinline__ void drain_pair_commits(uint32_t bar0, int lane, int n_all, int npc) {
  static_assert(L::NK + L::NV + L::NQ + 6 <= 32, "one barrier per lane");
  // t: the tile (or piece) whose commit completes the phase waited for, on a
  // ring of n barriers from b; negative when there was no such tile
  int k = lane, t = -1, n = 1, b = 0;
  if (k < L::NK) {
    t = n_all - 1 - k, n = L::NK, b = L::B_K_EMPTY;
  } else if ((k -= L::NK) < L::NV) {
    t = n_all - 1 - k, n = L::NV, b = L::B_V_EMPTY;
  } else if ((k -= L::NV) < L::NQ) {
    t = n_all - 1 - k, n = L::NQ, b = L::B_QK_DONE;
  } else if ((k -= L::NQ) < 4) {
    t = n_all - 1 - (k >> 1), n = 2, b = (k & 1) ? L::B_S_FULL : L::B_P_EMPTY;
  } else if ((k -= 4) == 0) {
    t = n_all - 1, n = 1, b = L::B_O_DONE;
  } else if (k == 1) {
    t = npc - 1, n = 1, b = L::B_O_FINAL;
  }
  if (t >= 0) drain_phase(bar0 + 8u * (uint32_t)(b + t % n), (uint32_t)(t / n) & 1);
}

// Write 32 output columns [col, col + 32) of flat row `rg`: BF16 to `out`
// when there is one split, else fp32 to the split's partial. inv = 0 means the
// row saw no key (written as exact zeros).
__device__ __forceinline__ void store_out_chunk(const DecodeArgs& a, int64_t rg, int s, int col,
                                                const uint32_t (&o)[32], float inv) {
  const int S = a.plan.split_kv;
  if (S == 1) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + rg * MLA_D_V + col);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float f0 = inv > 0.f ? __uint_as_float(o[8 * u + 2 * k]) * inv : 0.f;
        const float f1 = inv > 0.f ? __uint_as_float(o[8 * u + 2 * k + 1]) * inv : 0.f;
        __nv_bfloat162 hb = __floats2bfloat162_rn(f0, f1);
        pk[k] = *reinterpret_cast<uint32_t*>(&hb);
      }
      dst[u] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  } else {
    float4* dst = reinterpret_cast<float4*>(a.o_part + (rg * S + s) * MLA_D_V + col);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float4 f;
      f.x = inv > 0.f ? __uint_as_float(o[4 * u + 0]) * inv : 0.f;
      f.y = inv > 0.f ? __uint_as_float(o[4 * u + 1]) * inv : 0.f;
      f.z = inv > 0.f ? __uint_as_float(o[4 * u + 2]) * inv : 0.f;
      f.w = inv > 0.f ? __uint_as_float(o[4 * u + 3]) * inv : 0.f;
      dst[u] = f;
    }
  }
}

// 2-D tensor map over a row-major [rows, 576] array of 1- or 2-byte elements
// (q or the cache viewed as [num_pages * 64, 576]); box = box_x x box_y.
bool encode_rows_576_chunks(CUtensorMap* m, const void* base, int esize, uint64_t rows, uint32_t nchunks,
                            uint64_t chunk_stride, uint32_t box_rows, uint32_t box_chunks);
bool encode_rows_576(CUtensorMap* m, const void* base, int esize, uint64_t rows, uint32_t box_x, uint32_t box_y,
                     CUtensorMapSwizzle sw);

}  // namespace mla
