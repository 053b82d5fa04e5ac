// Balanced persistent schedule of the CTA-pair kernels (FP8 and 16-bit).
//
// Every unit (entry, query group) is a run of pair tiles counted from the
// device seq_lens (and, for ragged queries, cu_q): from the tile of the
// lowest key a row of the unit sees to the tile of the highest. A tile
// weighs 2, or 3 when its P.V runs twice (FP8 two-term P), so that pairs get
// equal work rather than equal tiles, and every unit with tiles starts with a
// lead-in of kPieceLeadWeight, the cost of a piece transition.
// The units' runs form one sequence of total weight W; pair p takes the tiles
// whose start lies in [floor(W p / np), floor(W (p + 1) / np)) and walks them
// as a list of pieces (the units its range meets, each cut to the range).
//
// Order of the sequence. A decode entry with G > 1 query groups (more query
// tokens than fit one 128-row tile) has G units over the same pages. In entry
// order they sit next to each other and the same pair reads the entry's pages
// once per group, far apart in time, so each page comes from DRAM G times.
// Decode plans with G > 1 therefore take the units group-major (group 0 of
// every entry, then group 1, ...): with equal ranges, pair p and the pair
// W / G weight further on walk the same pages at about the same time, and the
// later read is served by L2. Ragged prefill keeps entry order (its groups
// see different key spans and its pool is mostly L2-resident). Positions in
// the sequence are schedule slots; sched_unit / sched_slot map between them
// and units.
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
  int tiles;       // pair tiles of this pair
  int two;         // some piece has two-term P
  int spill_base;  // piece k >= kMaxSmemPieces is entry spill_base + k of the spill area
};
constexpr int kMaxSmemPieces = 64;  // pieces a pair keeps in shared memory; the rest go to the spill area
constexpr uint32_t kSchedBytes = 1024;
static_assert(kMaxSmemPieces * sizeof(Piece) + sizeof(SchedInfo) <= kSchedBytes, "schedule area");
constexpr int kMinPairWeight = 4;  // pairs get at least this much weight (>= the heaviest tile)

// Unit at schedule slot s, and the slot of unit u (u = entry * G + group).
__host__ __device__ __forceinline__ bool sched_group_major(const mla_plan& p) {
  return !p.varlen && p.q_groups > 1;
}
__host__ __device__ __forceinline__ int sched_unit(const mla_plan& p, int s) {
  return sched_group_major(p) ? (s % p.batch) * p.q_groups + s / p.batch : s;
}
__host__ __device__ __forceinline__ int sched_slot(const mla_plan& p, int u) {
  return sched_group_major(p) ? (u % p.q_groups) * p.batch + u / p.q_groups : u;
}

// Keys the unit's first row sees: the fewest of any of its rows (ragged
// prefill units early in an entry see only a few keys even when the entry
// has many).
__device__ __forceinline__ int unit_min_keys(const mla_plan& p, const UnitGeom& ug) {
  const int n = ug.nq + 1;
  return (p.window > 0 && p.window < n) ? p.window : n;
}

// Weight of one tile of a unit: 3 when its rows' P goes as two E4M3 terms
// (FP8 units whose first row sees fewer than kTwoTermKeys keys), else 2.
__device__ __forceinline__ int tile_weight(const mla_plan& p, const UnitGeom& ug) {
  if (p.dtype != MLA_FP8_E4M3) return 2;
  return unit_min_keys(p, ug) < kTwoTermKeys ? 3 : 2;
}

// Tiles [i0, i1) of a unit with `t` tiles of weight `w` starting at weighted
// position `start` whose own start positions lie in [lo, hi). Positions are
// below W < 2^31 (the plan checks the total weight), so the differences fit
// an int.
__device__ __forceinline__ void tiles_in_range(int64_t start, int t, int w, int64_t lo, int64_t hi, int& i0,
                                               int& i1) {
  const int a0 = lo > start ? ((int)(lo - start) + w - 1) / w : 0;
  const int a1 = hi > start ? ((int)(hi - start) + w - 1) / w : 0;
  i0 = a0 < t ? a0 : t;
  i1 = a1 < t ? a1 : t;
}

// Scratch of the block-wide scans, after the piece list and SchedInfo: one int
// per warp for the first scan, four per warp for the second.
constexpr int kMaxSchedWarps = 12;  // the CTA-pair kernels run 384 threads
constexpr uint32_t kSchedScratchOff = 784;
static_assert(kSchedScratchOff >= kMaxSmemPieces * sizeof(Piece) + sizeof(SchedInfo) &&
                  kSchedScratchOff + 4 * 5 * kMaxSchedWarps <= kSchedBytes,
              "schedule scratch");

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += y;
  }
  return v;
}

// The whole block: the schedule of this pair. Every thread takes a run of
// consecutive schedule slots; block scans (two barriers in all) give each
// run's weighted start and each thread's first piece index. The pieces of the
// pair's range are written in slot order, the first kMaxSmemPieces to shared
// memory and, when there are more, all of them to this CTA's part of the
// spill area (read back by load_piece). CTA 0 of pair 0 also writes the slot
// start table the combine reads, then its ready flag.
template <int kKeys>
__device__ void build_schedule(const DecodeArgs& a, int pair, uint32_t rank, uint8_t* sched_area) {
  const mla_plan& p = a.plan;
  Piece* smem_list = reinterpret_cast<Piece*>(sched_area);
  SchedInfo* info = reinterpret_cast<SchedInfo*>(sched_area + kMaxSmemPieces * sizeof(Piece));
  int* scan1 = reinterpret_cast<int*>(sched_area + kSchedScratchOff);  // [warp]
  int4* scan2 = reinterpret_cast<int4*>(scan1 + kMaxSchedWarps);       // [warp]: pieces, tiles, two, first slot
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = (int)(blockDim.x >> 5);
  const int U = p.batch * p.q_groups;
  const int per = (U + (int)blockDim.x - 1) / (int)blockDim.x;
  const int s_beg = min(U, tid * per), s_end = min(U, s_beg + per);  // this thread's schedule slots
  const bool writer = pair == 0 && rank == 0;
  // Tiles and tile weight of slot sl. The first slot of the thread's run keeps
  // them from the first scan (a plan of at most one slot per thread reads
  // seq_lens once); the others read them again.
  int t_beg = 0, w_beg = 2;
  auto geometry = [&](int sl, int& t, int& w) {
    if (sl == s_beg) {
      t = t_beg, w = w_beg;
      return;
    }
    const UnitGeom ug = unit_geom(a, sched_unit(p, sl), false);
    t = unit_span_tiles<kKeys>(ug), w = tile_weight(p, ug);
  };
  // scan 1: the weighted start of this thread's run
  int run = 0;
  for (int sl = s_beg; sl < s_end; ++sl) {
    const UnitGeom ug = unit_geom(a, sched_unit(p, sl), writer);
    const int t = unit_span_tiles<kKeys>(ug), w = tile_weight(p, ug);
    if (sl == s_beg) t_beg = t, w_beg = w;
    run += unit_lead_weight(t) + t * w;
  }
  int incl = warp_incl_scan(run);
  if (lane == 31) scan1[warp] = incl;
  __syncthreads();
  int W = 0, excl = incl - run;
  for (int w = 0; w < nw; ++w) {
    const int x = scan1[w];
    if (w < warp) excl += x;
    W += x;
  }
  const int np = max(1, min(p.split_kv, W / kMinPairWeight));
  const int64_t lo = pair < np ? balanced_lo(pair, W, np) : W;
  const int64_t hi = pair < np ? balanced_lo(pair + 1, W, np) : W;
  if (writer) {
    int start = excl;
    for (int sl = s_beg; sl < s_end; ++sl) {
      if (in_bounds(a, sl, U)) a.sched[sl] = start;
      int t, w;
      geometry(sl, t, w);
      start += unit_lead_weight(t) + t * w;
    }
    if (tid == 0) {
      a.sched[U] = W;
      a.sched[U + 1] = np;
    }
  }
  // scan 2: this thread's pieces (units of its run with tiles in the range)
  int cnt = 0, tiles = 0, two = 0, s_first_t = 0;
  {
    int start = excl;
    for (int sl = s_beg; sl < s_end; ++sl) {
      int t, w;
      geometry(sl, t, w);
      const int lead = unit_lead_weight(t);
      int i0, i1;
      tiles_in_range(start + lead, t, w, lo, hi, i0, i1);
      if (i1 > i0) {
        if (cnt == 0) s_first_t = sl;
        ++cnt;
        tiles += i1 - i0;
        if (w == 3) two = 1;
      }
      start += lead + t * w;
    }
  }
  const int cnt_incl = warp_incl_scan(cnt);
  const int tiles_w = warp_incl_scan(tiles);
  const unsigned has = __ballot_sync(0xffffffffu, cnt > 0);
  const int two_w = __any_sync(0xffffffffu, two);
  const int first_w = has ? __shfl_sync(0xffffffffu, s_first_t, __ffs(has) - 1) : -1;
  if (lane == 31) scan2[warp] = make_int4(cnt_incl, tiles_w, two_w, first_w);
  __syncthreads();
  int base = cnt_incl - cnt, npc = 0, all_tiles = 0, any_two = 0, s_first = -1;
  for (int w = 0; w < nw; ++w) {
    const int4 x = scan2[w];
    if (w < warp) base += x.x;
    npc += x.x;
    all_tiles += x.y;
    any_two |= x.z;
    if (s_first < 0 && x.x > 0) s_first = x.w;
  }
  // the table is complete (every thread wrote its units before the barrier):
  // the combine, which may already run, reads it once the flag is set
  if (writer && tid == 0) {
    __threadfence();
    ptx::st_release_gpu(a.unit_done + U, 1);
  }
  if (s_first < 0) s_first = 0;
  const int spill_base = (int)rank * (U + p.split_kv) + s_first + pair;
  Piece* spill = npc > kMaxSmemPieces ? reinterpret_cast<Piece*>(a.pieces) + spill_base : nullptr;
  if (cnt > 0) {
    int start = excl, k = base;
    for (int sl = s_beg; sl < s_end; ++sl) {
      const int u = sched_unit(p, sl);
      int t, w;
      geometry(sl, t, w);
      const int lead = unit_lead_weight(t);
      int i0, i1;
      tiles_in_range(start + lead, t, w, lo, hi, i0, i1);
      if (i1 > i0) {
        Piece pc;
        pc.u = u;
        pc.t0 = i0;
        pc.t1 = i1;
        if (k < kMaxSmemPieces) smem_list[k] = pc;
        if (spill && in_bounds(a, spill_base + k, spill_entries(a))) spill[k] = pc;
        ++k;
      }
      start += lead + t * w;
    }
  }
  if (tid == 0) {
    info->spill_base = spill_base;
    info->npc = npc;
    info->tiles = all_tiles;
    info->two = any_two;
  }
}

// Piece k of this CTA's pair (smem: the schedule area at the start of shared
// memory). The spill area is addressed from the kernel parameter, so no role
// keeps a list pointer live across its loops.
__device__ __forceinline__ Piece load_piece(const DecodeArgs& a, const uint8_t* smem, int k) {
  if (k < kMaxSmemPieces) return reinterpret_cast<const Piece*>(smem)[k];
  const SchedInfo* info = reinterpret_cast<const SchedInfo*>(smem + kMaxSmemPieces * sizeof(Piece));
  if (!in_bounds(a, info->spill_base + k, spill_entries(a))) return Piece{0, 0, 0};
  return reinterpret_cast<const Piece*>(a.pieces)[info->spill_base + k];
}

}  // namespace mla
