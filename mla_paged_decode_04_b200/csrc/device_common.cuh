// Device helpers shared by the partial and combine kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "internal.h"

namespace mla {

constexpr float kLn2 = 0.6931471805599453f;

// Device bounds checks of the checking build (compiled with
// MLA_BOUNDS_CHECK=1): in_bounds(a, i, n) is false when i lies outside
// [0, n), after setting MLA_DEV_BOUNDS in the status word, and the caller
// then skips the access. In the normal build it is always true and every
// check compiles away.
__device__ __forceinline__ bool in_bounds(const DecodeArgs& a, int64_t i, int64_t n) {
#if MLA_BOUNDS_CHECK
  if (i >= 0 && i < n) return true;
  atomicOr(a.status, MLA_DEV_BOUNDS);
  return false;
#else
  (void)a, (void)i, (void)n;
  return true;
#endif
}
// Extents the checks compare against: rows of out / lse, the balanced
// schedule's partial slots, its piece spill entries (both CTA ranks) and its
// units.
__device__ __forceinline__ int64_t out_rows(const DecodeArgs& a) { return a.total_q * a.plan.num_heads; }
__device__ __forceinline__ int64_t balanced_slots(const DecodeArgs& a) { return 2 * (int64_t)a.plan.split_kv; }
__device__ __forceinline__ int64_t balanced_units(const DecodeArgs& a) {
  return (int64_t)a.plan.batch * a.plan.q_groups;
}
__device__ __forceinline__ int64_t spill_entries(const DecodeArgs& a) {
  return 2 * (balanced_units(a) + a.plan.split_kv);
}

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
  if (!in_bounds(a, b, a.plan.batch)) return 0;
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

// Query tokens of batch entry b: the first one's index in the packed query
// and how many there are. Decode: q_len tokens each, entry-major. Ragged
// queries (prefill): entry b holds tokens [cu_q[b], cu_q[b + 1]); a range that
// is decreasing, longer than the plan's q_len or past total_q sets
// MLA_DEV_BAD_QLEN (when `flag` is set) and leaves the entry without tokens.
struct EntryQ {
  int64_t q0;
  int qlen;
};
__device__ __forceinline__ EntryQ entry_q(const DecodeArgs& a, int b, bool flag) {
  if (!a.cu_q) return {(int64_t)b * a.plan.q_len, a.plan.q_len};
  if (!in_bounds(a, b, a.plan.batch)) return {0, 0};
  const int s = a.cu_q[b], e = a.cu_q[b + 1];
  if (s < 0 || e < s || e - s > a.plan.q_len || (int64_t)e > a.total_q) {
    if (flag) atomicOr(a.status, MLA_DEV_BAD_QLEN);
    return {0, 0};
  }
  return {(int64_t)s, e - s};
}

// Unit u = (entry b, query group g): tokens g*F .. g*F + F - 1 of entry b
// (fewer in an entry's last group when queries are ragged), H rows each.
// Token t of an entry with n keys and qlen tokens sees keys up to
// n - qlen + t (causal, aligned to the end); with a sliding window W > 0 only
// its last W of them, from n - qlen + t + 1 - W.
struct UnitGeom {
  int b, g;
  int n;         // keys of the entry (clamped seq_len)
  int rows;      // query rows of the unit (0: a group past the entry's tokens)
  int nq;        // last key of the unit's first token; row r sees keys <= nq + r / H
  int klo;       // lowest key a row of the unit sees
  int kend;      // one past the highest key a row of the unit sees
  int64_t row0;  // first output row (token * H + head) of the unit
};
__device__ __forceinline__ UnitGeom unit_geom(const DecodeArgs& a, int u, bool flag) {
  const mla_plan& p = a.plan;
  UnitGeom ug;
  ug.b = u / p.q_groups;
  ug.g = u % p.q_groups;
  const bool first = flag && ug.g == 0;
  ug.n = effective_seq_len(a, ug.b, first);
  const EntryQ e = entry_q(a, ug.b, first);
  const int t0 = ug.g * p.fold;
  const int tu = min(p.fold, e.qlen - t0);
  ug.rows = tu > 0 ? tu * p.num_heads : 0;
  ug.nq = ug.n - e.qlen + t0;
  ug.row0 = (e.q0 + t0) * p.num_heads;
  ug.kend = tu > 0 ? max(0, ug.nq + tu) : 0;
  ug.klo = (tu > 0 && p.window > 0) ? max(0, ug.nq + 1 - p.window) : 0;
  return ug;
}
// First key of the row whose last key is `last` (its sliding window's start).
__device__ __forceinline__ int row_key_lo(const mla_plan& p, int last) {
  return p.window > 0 ? max(0, last + 1 - p.window) : 0;
}
// Tiles of kKeys keys a unit spans, from the tile of its lowest key.
template <int kKeys>
__device__ __forceinline__ int unit_span_tiles(const UnitGeom& ug) {
  return ug.kend > ug.klo ? (ug.kend + kKeys - 1) / kKeys - ug.klo / kKeys : 0;
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
