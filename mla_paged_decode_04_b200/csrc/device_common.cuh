// Device helpers shared by the partial and combine kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "internal.h"

namespace mla {

constexpr float kLn2 = 0.6931471805599453f;

// Element of a q / cache buffer as float (FP8 stays in code units; the
// caller applies the per-tensor scale once).
template <int DT>
__device__ __forceinline__ float load_elem(const void* base, int64_t idx) {
  if constexpr (DT == MLA_BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  } else if constexpr (DT == MLA_FP16) {
    return __half2float(reinterpret_cast<const __half*>(base)[idx]);
  } else {
    const __nv_fp8_storage_t c = reinterpret_cast<const __nv_fp8_storage_t*>(base)[idx];
    return __half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3)));
  }
}

// Keys a batch entry actually has, clamped to what the plan's splits and the
// block table can cover. Out-of-contract lengths set MLA_DEV_SEQ_TOO_LONG
// (when `flag` is set) and are clamped, so no read leaves the table.
__device__ __forceinline__ int effective_seq_len(const DecodeArgs& a, int b, bool flag) {
  int n = a.seq_lens[b];
  const int64_t cap_split = (int64_t)a.plan.split_kv * a.plan.keys_per_split;
  const int64_t cap_table = (int64_t)a.max_pages_per_seq * kTileKeys;
  int64_t cap = cap_split < cap_table ? cap_split : cap_table;
  bool bad = n < 0 || n > a.plan.max_seq_len || (int64_t)n > cap;
  if (bad && flag) atomicOr(a.status, MLA_DEV_SEQ_TOO_LONG);
  if (n < 0) n = 0;
  if ((int64_t)n > cap) n = (int)cap;
  return n;
}

// Sliding window (plan.window = W > 0): query token t of an entry with n
// keys sees keys [n - q_len + t + 1 - W, n - q_len + t]. First key of token t,
// and of the first token of query group g (the lowest key its unit needs).
__device__ __forceinline__ int window_row_lo(const mla_plan& p, int t, int n) {
  if (p.window <= 0) return 0;
  const int lo = n - p.q_len + t + 1 - p.window;
  return lo > 0 ? lo : 0;
}
__device__ __forceinline__ int window_unit_lo(const mla_plan& p, int g, int n) {
  return window_row_lo(p, g * p.fold, n);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace mla
