// Balanced persistent schedule of the CTA-pair kernels (FP8 and 16-bit).
//
// Every unit (entry, query group) is a run of pair tiles counted from the
// device seq_lens (and, for ragged queries, cu_q): from the tile of the
// lowest key a row of the unit sees to the tile of the highest. The units'
// runs, in unit order, form one sequence of W tiles; pair p takes the
// contiguous range [floor(W p / np), floor(W (p + 1) / np)) and walks it as a
// list of pieces (the units its range meets, each cut to the range).
#pragma once

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

// One piece: pair tiles [t0, t1) of unit u.
struct Piece {
  int u, t0, t1;
};
struct SchedInfo {
  int npc;         // pieces of this pair
  int tiles;       // pair tiles of this pair (its range's length)
  int two;         // some piece's entry is shorter than the two-term threshold
  int spill_base;  // piece k >= kMaxSmemPieces is entry spill_base + k of the spill area
};
constexpr int kMaxSmemPieces = 64;  // pieces a pair keeps in shared memory; the rest go to the spill area
constexpr uint32_t kSchedBytes = 1024;
static_assert(kMaxSmemPieces * sizeof(Piece) + sizeof(SchedInfo) <= kSchedBytes, "schedule area");
constexpr int kMinPairTiles = 2;  // fewer tiles than this per pair: use fewer pairs

// Pair tiles (of kKeys keys) of unit u.
template <int kKeys>
__device__ __forceinline__ int unit_tiles(const DecodeArgs& a, int u, bool flag) {
  return unit_span_tiles<kKeys>(unit_geom(a, u, flag));
}

// One warp: the schedule of this pair. Every lane takes a run of consecutive
// units and a warp scan gives each run's first tile; the pieces of the pair's
// range [lo, hi) are written in unit order, the first kMaxSmemPieces to shared
// memory and, when there are more, all of them to this CTA's part of the
// spill area (read back by load_piece). CTA 0 of pair 0 also writes the unit
// start table the combine reads, then its ready flag.
// `two_keys` > 0: report whether a piece's entry lets a row see fewer keys.
template <int kKeys>
__device__ void build_schedule(const DecodeArgs& a, int pair, uint32_t rank, Piece* smem_list, SchedInfo* info,
                               int two_keys) {
  const mla_plan& p = a.plan;
  const int lane = threadIdx.x & 31;
  const int U = p.batch * p.q_groups;
  const int per = (U + 31) / 32;
  const int u_beg = min(U, lane * per), u_end = min(U, u_beg + per);
  const bool writer = pair == 0 && rank == 0;
  int run = 0;
  for (int u = u_beg; u < u_end; ++u) run += unit_tiles<kKeys>(a, u, writer);
  int excl = run;  // inclusive prefix, then exclusive
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, excl, d);
    if (lane >= d) excl += y;
  }
  const int W = __shfl_sync(0xffffffffu, excl, 31);
  excl -= run;
  const int np = max(1, min(p.split_kv, (W + kMinPairTiles - 1) / kMinPairTiles));
  const int64_t lo = pair < np ? balanced_lo(pair, W, np) : W;
  const int64_t hi = pair < np ? balanced_lo(pair + 1, W, np) : W;
  if (writer) {
    int start = excl;
    for (int u = u_beg; u < u_end; ++u) {
      a.sched[u] = start;
      start += unit_tiles<kKeys>(a, u, false);
    }
    if (lane == 31) {
      a.sched[U] = W;
      a.sched[U + 1] = np;
    }
    // the table is complete: the combine (which may already run) reads it
    // once this flag is set
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      ptx::st_release_gpu(a.unit_done + U, 1);
    }
  }
  // pieces: units of this lane's run that meet [lo, hi)
  int cnt = 0, u_first_lane = 0;
  {
    int start = excl;
    for (int u = u_beg; u < u_end; ++u) {
      const int t = unit_tiles<kKeys>(a, u, false);
      if (t > 0 && start < hi && start + t > lo) {
        if (cnt == 0) u_first_lane = u;
        ++cnt;
      }
      start += t;
    }
  }
  int base = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, base, d);
    if (lane >= d) base += y;
  }
  const int npc = __shfl_sync(0xffffffffu, base, 31);
  base -= cnt;
  const unsigned has = __ballot_sync(0xffffffffu, cnt > 0);
  const int u_first = has ? __shfl_sync(0xffffffffu, u_first_lane, __ffs(has) - 1) : 0;
  const int spill_base = (int)rank * (U + p.split_kv) + u_first + pair;
  Piece* spill = npc > kMaxSmemPieces ? reinterpret_cast<Piece*>(a.pieces) + spill_base : nullptr;
  int two = 0;
  {
    int start = excl, k = base;
    for (int u = u_beg; u < u_end; ++u) {
      const UnitGeom ug = unit_geom(a, u, false);
      const int t = unit_span_tiles<kKeys>(ug);
      if (t > 0 && start < hi && start + t > lo) {
        Piece pc;
        pc.u = u;
        pc.t0 = lo > start ? (int)(lo - start) : 0;
        pc.t1 = hi - start < t ? (int)(hi - start) : t;
        if (k < kMaxSmemPieces) smem_list[k] = pc;
        if (spill) spill[k] = pc;
        const int seen = (p.window > 0 && p.window < ug.n) ? p.window : ug.n;
        if (two_keys > 0 && seen < two_keys) two = 1;
        ++k;
      }
      start += t;
    }
  }
  two = __any_sync(0xffffffffu, two);
  if (lane == 0) {
    info->spill_base = spill_base;
    info->npc = npc;
    info->tiles = (int)(hi - lo);
    info->two = two;
  }
}

// Piece k of this CTA's pair (smem: the schedule area at the start of shared
// memory). The spill area is addressed from the kernel parameter, so no role
// keeps a list pointer live across its loops.
__device__ __forceinline__ Piece load_piece(const DecodeArgs& a, const uint8_t* smem, int k) {
  if (k < kMaxSmemPieces) return reinterpret_cast<const Piece*>(smem)[k];
  const SchedInfo* info = reinterpret_cast<const SchedInfo*>(smem + kMaxSmemPieces * sizeof(Piece));
  return reinterpret_cast<const Piece*>(a.pieces)[info->spill_base + k];
}

}  // namespace mla
