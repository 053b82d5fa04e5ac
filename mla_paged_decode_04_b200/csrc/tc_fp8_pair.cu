// Split-KV partial kernel for FP8 E4M3 inputs with CTA-pair tensor-core MMAs
// and a balanced, persistent schedule.
//
// The first of the two decode kernels (TokenSpeed MLA article
// 最快MLA内核背后的秘密, section 二) with query-token folding (section 三), using
// the 2-CTA MMA of section 四: the two CTAs of a cluster pair execute every
// tcgen05.mma together (cta_group::2, M = 128), each holding half of the
// operands and half of the result.
//
// Schedule (pair_schedule.cuh). The pairs stay resident (one per two SMs). A
// unit (batch entry, query group) spans the pair tiles of two cache pages
// that hold the keys its rows see; the units' tiles, counted from the device
// seq_lens and weighted by their P.V work, form one sequence that is dealt
// out as equal contiguous ranges, one per pair. A pair walks its range as
// pieces (the part of one unit inside the range): a piece that is a whole
// unit writes out / lse directly; a unit cut between pairs leaves partial O
// and LSE in one of the pair's two slots (2p for a piece that begins inside
// its unit, 2p + 1 for one that begins at the unit's start), merged by the
// combine kernel. Every pair therefore does the same amount of
// work whatever the length mix, and the pipeline runs on across pieces. This
// is the article's split_kv auto-sizing (section 二) made exact on the device.
// The same kernel serves ragged prefill (entries with their own query
// lengths) and sliding windows through the unit geometry of device_common.cuh.
//
// Inside a pair tile, page 2j of the piece goes to CTA 0 and page 2j+1 to CTA 1.
//  * S = Q.K^T (N = 128 keys): CTA c supplies query rows [64c, 64c+64) as
//    the A operand (tensor memory) and its own page as B (shared memory);
//    it receives S for its 64 rows and all 128 keys. No score, page or
//    softmax work is duplicated in the pair.
//  * Softmax: CTA c finishes its own 64 rows. S row r of a CTA lies in TMEM
//    lane r (keys 0..63, the leader's page) and lane 64+r (keys 64..127), so
//    two threads of different warps share a row and swap their maxima
//    through shared memory.
//  * O += P.V (N = 256 output columns per MMA, two MMAs per K step): CTA c
//    supplies its P rows as A and V columns [256h + 128c, 256h + 128c + 128)
//    of all 128 keys as B; its O rows stay in its own TMEM (both column
//    halves h, 256 TMEM columns).
// Because B of the P.V is laid out by output column and B of Q.K^T by key,
// each CTA loads, besides its own page (K ring, freed once S is computed),
// its 256 V columns of both pages into a V ring. Those loads are issued once
// the scores of the tile exist, so they are served by L2 (the pages were
// just read for S) while the softmax runs, and a V slot is held only for
// about the softmax: the split of K and V loads of section 四.
//
// P = 2^(x - m + SIGMA) with x the log2-scaled score and m a lazily updated
// row maximum (moved only when exceeded by more than TAU), as E4M3; for
// entries shorter than kTwoTermKeys it is sent as two E4M3 terms (hi, lo)
// so that short rows keep about 8 significant bits. O is normalised by the
// exact fp32 sum of P, which also gives the LSE.
//
// Roles (384 threads per CTA): warp 0 lane 0 loads Q and the K ring; warp 1
// owns TMEM (both CTAs) and, in the leader (cluster rank 0), issues the
// S MMAs; warp 2 issues the P.V MMAs (leader); warp 3 lane 0 loads the V
// ring; warps 4-11 are two softmax groups of four warps taking alternate
// pair tiles (one thread per (row, key half), 64 keys each), which also do
// the O rescales and the epilogue of every piece. Ring slots and their
// barrier phases follow a tile counter that runs across the pieces; the
// per-piece barriers (Q, O_FINAL, FIN, EPI, O_FREE) advance once per piece.
// Barriers the MMA issuer waits on live in the leader; the follower's loads
// and arrivals reach them through cluster addresses. MMA completions are
// multicast to both CTAs.
//
// Every wait is bounded; on expiry the CTA sets MLA_DEV_TIMEOUT, leaves the
// pipeline, waits for its peer at the final cluster barrier, frees TMEM and
// returns. No TMA load uses multicast.
#include <cuda.h>

#include "device_common.cuh"
#include "pair_schedule.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr float kTau = 4.f;          // lazy-rescale threshold (log2 units)
constexpr float kSigma = 4.f;        // P <= 2^(kTau + kSigma) = 256 <= 448
// The schedule area (pair_schedule.cuh) is at the start of shared memory, the
// same place in both layouts.

// The barriers and the TMEM slot sit at the same place in both layouts, right
// after the schedule area, so that they are set up before the schedule (and
// with it the layout) is known.
constexpr uint32_t kPairBarOff = kSchedBytes;        // 64 mbarriers
constexpr uint32_t kPairMiscOff = kPairBarOff + 512;  // TMEM address, abort flag

template <bool kTwo>
struct PairLayout {
  static constexpr int NK = 3;                                  // K-ring slots: own page
  static constexpr int NV = 2;                                  // V-ring slots: 256 V columns of both pages
  static constexpr uint32_t kBarOff = kPairBarOff;
  static constexpr uint32_t kMiscOff = kPairMiscOff;
  static constexpr uint32_t kQRope = kMiscOff + 512;            // 64 rows x 64 B (SW64)
  static constexpr uint32_t kPPlane = 64 * 128;                 // 64 rows x 128 keys E4M3 (SW128)
  static constexpr uint32_t kPBuf = (kTwo ? 2 : 1) * kPPlane;   // hi (and lo) plane
  static constexpr uint32_t kPOff = kQRope + 4096;              // P[2 buffers] (1024-aligned)
  static constexpr uint32_t kKSlot = 4 * 8192 + 64 * 64;        // 4 latent chunks (SW128) + rope (SW64)
  static constexpr uint32_t kKOff = kPOff + 2 * kPBuf;
  static constexpr uint32_t kVSlot = 4 * 8192;                  // [column half h][page] chunks (SW128)
  static constexpr uint32_t kVOff = kKOff + NK * kKSlot;
  // Q latent dims (64 rows x 512 B) are staged in the last V slot: the K
  // loader fills it once the previous piece's MMAs are all done, and the V
  // loader refills it only after the piece's first S MMAs (so after Q
  // reached TMEM).
  static constexpr uint32_t kQStage = kVOff + (NV - 1) * kVSlot;
  static constexpr uint32_t kMOff = kVOff + NV * kVSlot;        // row reference maxima [tile parity][64]
  static constexpr uint32_t kXOff = kMOff + 512;                // half-row maxima [group][phase][half][64]
  static constexpr uint32_t kFinOff = kXOff + 2048;             // final (l, m) [l|m][group][half][64]
  // barriers ("leader": only the leader's copy is used)
  static constexpr int B_Q_MAIN = 0;                 // local, per piece: staged Q latent landed
  static constexpr int B_Q_ROPE = 1;                 // leader, per piece: both CTAs' Q rope landed
  static constexpr int B_Q_TMEM = 2;                 // leader, per piece: both CTAs copied Q into TMEM
  static constexpr int B_K_FULL = 3;                 // leader, + K slot: both pages landed
  static constexpr int B_K_EMPTY = B_K_FULL + NK;    // both, + K slot
  static constexpr int B_V_FULL = B_K_EMPTY + NK;    // leader, + V slot
  static constexpr int B_V_EMPTY = B_V_FULL + NV;    // both, + V slot
  static constexpr int B_S_FULL = B_V_EMPTY + NV;    // both, + buffer
  static constexpr int B_S_EMPTY = B_S_FULL + 2;     // leader, + buffer
  static constexpr int B_P_FULL = B_S_EMPTY + 2;     // leader, + buffer
  static constexpr int B_P_EMPTY = B_P_FULL + 2;     // both, + buffer
  static constexpr int B_O_DONE = B_P_EMPTY + 2;     // both
  static constexpr int B_O_FINAL = B_O_DONE + 1;     // both, per piece: after the piece's last P.V
  static constexpr int B_M_READY = B_O_FINAL + 1;    // local, + tile parity
  static constexpr int B_X = B_M_READY + 2;          // local, + group: half-row maxima exchanged
  static constexpr int B_FIN = B_X + 2;              // local, per piece: both groups published (l, m)
  // both, + tile % NQ: the scores of the tile exist (the V loads may go).
  // NQ = 6 rules out phase aliasing: S = Q.K^T of tile j+6 needs the scores
  // of tile j+4 read, which needs P of tile j+2 written, which needs the
  // P.V of tile j done, which needs the V loads of tile j issued.
  static constexpr int NQ = 6;
  static constexpr int B_QK_DONE = B_FIN + 1;
  static constexpr int B_EPI = B_QK_DONE + NQ;       // local, per piece: the output tile is staged
  static constexpr int B_O_FREE = B_EPI + 1;         // leader, per piece: both CTAs read O
  static constexpr int kNBars = B_O_FREE + 1;
  static_assert(8 * kNBars <= 512, "barrier area");
  static constexpr uint32_t kSmemBytes = kFinOff + 2048 + 1024;  // + alignment slack of the base
  static_assert(kPOff % 1024 == 0 && kKOff % 1024 == 0 && kKSlot % 1024 == 0 && kVOff % 1024 == 0, "alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // the last piece's epilogue stages the 64 x 512 fp32 output tile in the
  // (then idle) K and V rings
  static_assert(NK * kKSlot + NV * kVSlot >= 64 * MLA_D_V * 4, "staging area");
};
constexpr uint32_t kPairSmemBytes =
    PairLayout<true>::kSmemBytes > PairLayout<false>::kSmemBytes ? PairLayout<true>::kSmemBytes
                                                                 : PairLayout<false>::kSmemBytes;

constexpr int kSoftmaxWarp0 = 4;
constexpr int kSoftmaxWarps = 8;
static_assert(2 * kSoftmaxWarps == kPieceArrivals, "unit counter arrivals per piece");
constexpr int kThreads = 32 * (kSoftmaxWarp0 + kSoftmaxWarps);
static_assert(kThreads <= 32 * kMaxSchedWarps, "the schedule build's scratch");

// tensor memory columns (per CTA)
constexpr uint32_t kOCol = 0;    // O: column half h at [128h, 128h + 128)
constexpr uint32_t kQCol = 256;  // Q latent dims, 4 E4M3 per column, rows duplicated over lane halves
constexpr uint32_t kSCol = 384;  // two S buffers of 64 columns

struct PairParams {
  CUtensorMap tm_q_main, tm_q_rope, tm_kv_main, tm_kv_rope;
  DecodeArgs a;
};

// Per-piece constants every role derives the same way.
struct PieceCtx {
  int b, g, n, nq, rows, key0, key1, n_pt, n_tiles, tile0;
  int64_t row0;
  const int32_t* table;
  bool whole;  // the piece is the whole unit: final output, not a partial
  bool cont;   // the piece begins inside its unit (the pair's first piece)
  bool two;    // two-term P
};

// The unit geometry as a call, not inlined into every role: the roles' code
// stays smaller, which measured ~3% faster on the 80K-key FP8 batch (the
// kernel is sensitive to instruction-cache layout; the 16-bit kernel measured
// faster with it inlined).
__device__ __noinline__ UnitGeom unit_geom_call(const DecodeArgs& a, int u) { return unit_geom(a, u, false); }

__device__ __forceinline__ PieceCtx piece_ctx(const DecodeArgs& a, const Piece& pc, bool kTwo) {
  const mla_plan& p = a.plan;
  PieceCtx c;
  const UnitGeom ug = unit_geom_call(a, pc.u);
  c.b = ug.b;
  c.g = ug.g;
  c.n = ug.n;
  c.nq = ug.nq;
  c.rows = ug.rows;
  const int tlo = ug.klo / kPairTileKeys;  // the unit's first pair tile
  c.key0 = (tlo + pc.t0) * kPairTileKeys;
  c.key1 = min(ug.kend, (tlo + pc.t1) * kPairTileKeys);
  c.n_pt = pc.t1 - pc.t0;
  c.n_tiles = (c.key1 - c.key0 + kTileKeys - 1) / kTileKeys;
  c.tile0 = c.key0 / kTileKeys;
  // (test mode 2 of the checking build: every output row past out's end)
  c.row0 = ug.row0 + (MLA_BOUNDS_CHECK && p.fault_test == 2 ? out_rows(a) : 0);
  c.table = a.block_tables + (int64_t)c.b * a.max_pages_per_seq;
  c.whole = pc.t0 == 0 && c.key1 >= ug.kend;
  c.cont = pc.t0 > 0;
  c.two = kTwo && tile_weight(p, ug) == 3;  // the same rule as the schedule's weights
#if MLA_BOUNDS_CHECK
  // the piece's block-table entries [tile0, tile0 + n_tiles) of row b; if any
  // lies outside, none is read and every key of the piece is masked
  if (c.n_tiles > 0 && !(in_bounds(a, c.b, p.batch) && in_bounds(a, c.tile0, a.max_pages_per_seq) &&
                         in_bounds(a, (int64_t)c.tile0 + c.n_tiles - 1, a.max_pages_per_seq)))
    c.n_tiles = 0;
#endif
  return c;
}

// Block-table entry of 64-key tile t of the piece (0 past its end), read one
// tile ahead of its use: the load is issued before the next barrier wait and
// checked after it, so its latency stays off the ring's critical path.
__device__ __forceinline__ int piece_entry(const PieceCtx& c, int t) {
  return t < c.n_tiles ? ld_nc_ordered(c.table + c.tile0 + t) : 0;
}
// an entry outside the cache reads page 0 (its keys are masked by the softmax)
__device__ __forceinline__ int valid_page(const DecodeArgs& a, int pg) {
  return (pg < 0 || (int64_t)pg >= a.num_pages) ? 0 : pg;
}

template <bool kTwo>
__device__ __forceinline__ void pair_cta(const PairParams& prm, uint8_t* smem, int npc,
                                         int n_all) {
  using L = PairLayout<kTwo>;
  constexpr int NK = L::NK, NV = L::NV, NQ = L::NQ;
  const DecodeArgs& a = prm.a;
  const mla_plan& p = a.plan;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kBarOff + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int H = p.num_heads, M = p.rows_per_unit;
  const int box_q = M < 64 ? M : 64;  // query rows per TMA box (the tensor maps' box height)

  // the leader's copy of barrier i, as a cluster address
  auto lead = [&](int i) -> uint32_t { return mapa(bar(i), 0); };
  // Arrive on the leader's barrier i: a plain local arrive in the leader; in
  // the follower a cluster arrive, after a release fence over this CTA's
  // shared memory when it publishes data the leader's MMA will read (tensor
  // memory writes are ordered by tcgen05.fence::before_thread_sync), relaxed
  // otherwise. A full cluster-scope release would also wait for this
  // thread's outstanding global loads (the block-table prefetch).
  auto arrive_lead = [&](int i) {
    if (rank == 0) mbar_arrive(bar(i)); else mbar_arrive_remote_publish_smem(lead(i));
  };
  auto arrive_lead_relaxed = [&](int i) {
    if (rank == 0) mbar_arrive(bar(i)); else mbar_arrive_remote_relaxed(lead(i));
  };

  // (barriers, TMEM and the cluster sync were set up by pair_setup)
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ Q and K-ring loads
    if (lane == 0) {
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();  // read again right away for V
      int jt = 0;     // tile counter across pieces
      bool ok = true;
      for (int k = 0; ok && k < npc; ++k) {
        const PieceCtx c = piece_ctx(a, load_piece(a, smem, k), kTwo);
        if (k > 0) {
          // Q rope, Q in TMEM and the staging slot are free once every MMA of
          // the previous piece is done: its O_FINAL phase. (The V ring's own
          // barriers could be two phases behind here, since S runs ahead of
          // P.V; O_FINAL cannot, as its next phase needs this very load.)
          if (!(ok = bounded_wait_cta(bar(L::B_O_FINAL), (k - 1) & 1, abort_flag, a.status))) break;
        }
        const int qrow = (int)c.row0 + 64 * (int)rank;  // rows past the unit are read but never stored
        mbar_arrive_expect_tx(bar(L::B_Q_MAIN), 4u * 128u * (uint32_t)box_q);
#pragma unroll
        for (int ci = 0; ci < 4; ++ci)
          tma_load_2d(sb + L::kQStage + ci * 8192, &prm.tm_q_main, 128 * ci, qrow, bar(L::B_Q_MAIN), pol_q);
        if (rank == 0) mbar_arrive_expect_tx(bar(L::B_Q_ROPE), 2u * 64u * (uint32_t)box_q);
        tma_load_2d_pair(sb + L::kQRope, &prm.tm_q_rope, 512, qrow, lead(L::B_Q_ROPE), pol_q);
        int entry_nx = piece_entry(c, (int)rank);
        for (int j = 0; j < c.n_pt; ++j, ++jt) {
          const int sk = jt % NK;
          const int page = valid_page(a, entry_nx);
          if (j + 1 < c.n_pt) entry_nx = piece_entry(c, 2 * (j + 1) + (int)rank);
          if (!(ok = bounded_wait_cta(bar(L::B_K_EMPTY + sk), ((jt / NK) & 1) ^ 1, abort_flag, a.status))) break;
          // failure-detection test mode: the pair's first tile is never loaded,
          // so the S issuer's wait for it runs out (every wait is bounded)
          if (p.fault_test == 1 && jt == 0) continue;
          const uint32_t ks = sb + L::kKOff + sk * L::kKSlot;
          const uint32_t full = lead(L::B_K_FULL + sk);
          if (rank == 0) mbar_arrive_expect_tx(bar(L::B_K_FULL + sk), 2u * L::kKSlot);
#pragma unroll
          for (int ci = 0; ci < 4; ++ci)
            tma_load_2d_pair(ks + ci * 8192, &prm.tm_kv_main, 128 * ci, page * kTileKeys, full, pol_kv);
          tma_load_2d_pair(ks + 4 * 8192, &prm.tm_kv_rope, 512, page * kTileKeys, full, pol_kv);
        }
      }
      // The leader's K_FULL phases count both CTAs' bytes: the leader waits for
      // the last ones before the pair may leave (the follower waits at the
      // final cluster barrier).
      if (rank == 0) drain_loads(bar(L::B_K_FULL), NK, n_all);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ V-ring loads
    if (lane == 0) {
      const uint64_t pol_v = policy_evict_first();  // last use of these bytes
      int jt = 0;
      bool ok = true;
      for (int k = 0; ok && k < npc; ++k) {
        const PieceCtx c = piece_ctx(a, load_piece(a, smem, k), kTwo);
        int e0_nx = piece_entry(c, 0), e1_nx = piece_entry(c, 1);
        for (int j = 0; j < c.n_pt; ++j, ++jt) {
          const int sv = jt % NV;
          const int pg0 = valid_page(a, e0_nx), pg1 = valid_page(a, e1_nx);
          if (j + 1 < c.n_pt) {
            e0_nx = piece_entry(c, 2 * (j + 1));
            e1_nx = piece_entry(c, 2 * (j + 1) + 1);
          }
          // the scores of the tile exist: its pages are in L2 now
          if (!(ok = bounded_wait_cta(bar(L::B_QK_DONE + jt % NQ), (jt / NQ) & 1, abort_flag, a.status))) break;
          if (!(ok = bounded_wait_cta(bar(L::B_V_EMPTY + sv), ((jt / NV) & 1) ^ 1, abort_flag, a.status))) break;
          const uint32_t vs = sb + L::kVOff + sv * L::kVSlot;
          const uint32_t full = lead(L::B_V_FULL + sv);
          if (rank == 0) mbar_arrive_expect_tx(bar(L::B_V_FULL + sv), 2u * L::kVSlot);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int x = 128 * (2 * h + (int)rank);  // this CTA's 128 of the 256 columns of half h
            tma_load_2d_pair(vs + h * 16384, &prm.tm_kv_main, x, pg0 * kTileKeys, full, pol_v);
            tma_load_2d_pair(vs + h * 16384 + 8192, &prm.tm_kv_main, x, pg1 * kTileKeys, full, pol_v);
          }
        }
      }
      if (rank == 0) drain_loads(bar(L::B_V_FULL), NV, n_all);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S = Q.K^T issuer (leader)
    if (rank == 0) {
      constexpr uint32_t idq = instr_desc(0, 0, 0, 128, kPairTileKeys);  // E4M3 x E4M3, K-major B
      const uint64_t dq_rope = smem_desc(sb + L::kQRope, 16, 512, kSw64);
      int jt = 0;
      bool ok = true;
      for (int k = 0; ok && k < npc; ++k) {
        const Piece pk = load_piece(a, smem, k);
        const int n_pt = pk.t1 - pk.t0;
        if (!(ok = warp_wait(bar(L::B_Q_ROPE), k & 1, abort_flag, a.status) &&
                   warp_wait(bar(L::B_Q_TMEM), k & 1, abort_flag, a.status)))
          break;
        for (int j = 0; j < n_pt; ++j, ++jt) {
          const int sk = jt % NK, buf = jt & 1;
          if (!(ok = warp_wait(bar(L::B_K_FULL + sk), (jt / NK) & 1, abort_flag, a.status))) break;
          if (!(ok = warp_wait(bar(L::B_S_EMPTY + buf), ((jt >> 1) & 1) ^ 1, abort_flag, a.status))) break;
          tc_fence_after();
          const uint32_t d = tmem + kSCol + 64u * buf;
          const uint32_t ks = sb + L::kKOff + sk * L::kKSlot;
#pragma unroll
          for (int ci = 0; ci < 4; ++ci) {
            const uint64_t dk = smem_desc(ks + ci * 8192, 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ts_pair_e(d, tmem + kQCol + (uint32_t)(8 * (4 * ci + kk)), dk + (uint64_t)((kk * 32) >> 4),
                               idq, (ci | kk) ? 1u : 0u);
          }
          const uint64_t dr = smem_desc(ks + 4 * 8192, 16, 512, kSw64);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_f8_ss_pair_e(d, dq_rope + (uint64_t)(kk * 2), dr + (uint64_t)(kk * 2), idq, 1u);
          mma_commit_pair_mc_e(bar(L::B_S_FULL + buf), 3);
          mma_commit_pair_mc_e(bar(L::B_K_EMPTY + sk), 3);
          mma_commit_pair_mc_e(bar(L::B_QK_DONE + jt % NQ), 3);
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ O += P.V issuer (leader)
    if (rank == 0) {
      constexpr uint32_t idp = instr_desc(0, 0, 1, 128, 256);  // V is MN-major
      int jt = 0;
      bool ok = true;
      for (int k = 0; ok && k < npc; ++k) {
        const PieceCtx c = piece_ctx(a, load_piece(a, smem, k), kTwo);
        // the piece's first P.V overwrites O: the previous piece's epilogue
        // must have read it
        if (k > 0 && !(ok = warp_wait(bar(L::B_O_FREE), (k - 1) & 1, abort_flag, a.status))) break;
        for (int j = 0; j < c.n_pt; ++j, ++jt) {
          const int buf = jt & 1, sv = jt % NV;
          if (!(ok = warp_wait(bar(L::B_V_FULL + sv), (jt / NV) & 1, abort_flag, a.status))) break;
          if (!(ok = warp_wait(bar(L::B_P_FULL + buf), (jt >> 1) & 1, abort_flag, a.status))) break;
          tc_fence_after();
          const uint32_t vs = sb + L::kVOff + sv * L::kVSlot;
          const uint64_t dp = smem_desc(sb + L::kPOff + buf * L::kPBuf, 16, 1024, kSw128);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {  // 32 keys per MMA: page k4/2, rows (k4%2)*32
              const uint64_t dv =
                  smem_desc(vs + h * 16384 + (k4 >> 1) * 8192 + (k4 & 1) * 4096, 8192, 1024, kSw128);
              mma_f8_ss_pair_e(tmem + kOCol + 128u * h, dp + (uint64_t)((k4 * 32) >> 4), dv, idp,
                               (j > 0 || k4 > 0) ? 1u : 0u);
              if (c.two)
                mma_f8_ss_pair_e(tmem + kOCol + 128u * h, dp + (uint64_t)((L::kPPlane + k4 * 32) >> 4), dv, idp,
                                 1u);
            }
          }
          // O_DONE first: a softmax group that has seen P_EMPTY of tile j-2 may
          // rely on O_DONE having completed that tile's phase too.
          mma_commit_pair_mc_e(bar(L::B_O_DONE), 3);
          mma_commit_pair_mc_e(bar(L::B_P_EMPTY + buf), 3);
          mma_commit_pair_mc_e(bar(L::B_V_EMPTY + sv), 3);
          if (j == c.n_pt - 1) mma_commit_pair_mc_e(bar(L::B_O_FINAL), 3);
        }
      }
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax warps
    // Group grp takes the tiles whose running index has parity grp; warp w
    // serves TMEM lane quarter q = w%4: local rows 32(q%2) .. +31, key half
    // hf = q/2.
    const int q = warp & 3;
    const int grp = (warp - kSoftmaxWarp0) >> 2;
    const int hf = q >> 1;
    const int rl = 32 * (q & 1) + lane;  // local row (0..63)
    const int r = 64 * (int)rank + rl;   // row within the unit
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    float* mref = reinterpret_cast<float*>(smem + L::kMOff);  // [tile parity][64]
    float* xm = reinterpret_cast<float*>(smem + L::kXOff);    // [group][phase][half][64]
    float* fin = reinterpret_cast<float*>(smem + L::kFinOff); // [l|m][group][half][64]
    const float sl2 = a.score_scale_log2;
    bool ok = true;
    int jt = 0;  // running index of the piece's first tile

    for (int k = 0; ok && k < npc; ++k) {
      const PieceCtx c = piece_ctx(a, load_piece(a, smem, k), kTwo);
      const bool last_piece = k == npc - 1;
      // causal limit and sliding-window start of this row (rows past the
      // unit compute on whatever Q holds and are never stored)
      const int limit = (r < c.rows) ? min(c.nq + r / H, c.key1 - 1) : c.key1 - 1;
      const int lower = (r < c.rows) ? row_key_lo(p, c.nq + r / H) : 0;

      // Q latent dims of local row rl into TMEM (A operand of S = Q.K^T): lane
      // quarters q and q^2 both hold rows 32(q%2)..; group g copies chunks
      // 2g, 2g+1. The previous piece's S MMAs read Q until its last tile.
      if (k > 0) {
        const int jl = jt - 1;
        if (!(ok = warp_wait_cta(bar(L::B_S_FULL + (jl & 1)), (jl >> 1) & 1, abort_flag, a.status))) break;
      }
      if (!(ok = warp_wait_cta(bar(L::B_Q_MAIN), k & 1, abort_flag, a.status))) break;
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int cc = 2 * grp + c2;
        const uint8_t* chunk = smem + L::kQStage + cc * 8192 + rl * 128;
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(chunk + ((u ^ (rl & 7)) * 16));
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        if (r >= c.rows) {
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = 0;
        }
        tmem_st32(tmem + tl + kQCol + 32u * cc, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_lead(L::B_Q_TMEM);

      float m_grp = -INFINITY, l_grp = 0.f;  // this group's reference and partial sum (this half row)
      float m_last = -INFINITY;              // the reference of this group's previous tile of the piece
      // block-table entry of this half's page for the group's next tile, read
      // one tile ahead so that the dependent load is off the critical path
      auto table_entry = [&](int jj) -> int {
        const int t = 2 * jj + hf;
        return piece_entry(c, t);
      };
      const int j_first = (jt & 1) == grp ? 0 : 1;
      int pg_next = j_first < c.n_pt ? table_entry(j_first) : 0;
      for (int j = j_first; ok && j < c.n_pt; j += 2) {
        const int jg = jt + j;   // running tile index
        const int buf = jg & 1;  // == grp
        const int ph = (jg >> 1) & 1;
        const int pg_cur = pg_next;
        if (j + 2 < c.n_pt) pg_next = table_entry(j + 2);
        if (!(ok = warp_wait_cta(bar(L::B_S_FULL + buf), ph, abort_flag, a.status))) break;
        tc_fence_after();
        uint32_t sv[64];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
          tmem_ld32(tmem + tl + kSCol + 64u * buf, s0);
          tmem_ld32(tmem + tl + kSCol + 64u * buf + 32u, s1);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead_relaxed(L::B_S_EMPTY + buf);  // the slice was read (wait::ld above)

        const int t = 2 * j + hf;  // 64-key tile of this half
        bool page_ok = t < c.n_tiles;
        if (page_ok && (pg_cur < 0 || (int64_t)pg_cur >= a.num_pages)) {
          page_ok = false;
          if (lane == 0 && (q & 1) == 0) atomicOr(a.status, MLA_DEV_BAD_PAGE);
        }
        const int kb = c.key0 + kPairTileKeys * j + 64 * hf;
        // raw scores; masked keys become -inf (sl2 > 0, so max commutes with the scale)
        if (!(page_ok && kb >= lower && kb + 63 <= limit)) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (!(page_ok && kb + i >= lower && kb + i <= limit)) sv[i] = __float_as_uint(-INFINITY);
        }
        float mt;
        {
          // four independent chains of three-input maxima over 16 keys each
          float m4[4];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t* x = sv + 16 * c4;
            float v = max3f(__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]));
#pragma unroll
            for (int e = 3; e < 15; e += 2) v = max3f(v, __uint_as_float(x[e]), __uint_as_float(x[e + 1]));
            m4[c4] = fmaxf(v, __uint_as_float(x[15]));
          }
          mt = fmaxf(max3f(m4[0], m4[1], m4[2]), m4[3]) * sl2;
        }
        // The other half of the row lives in the warp of quarter q^2: this
        // half's maximum is published now and the partner's read when needed.
        float* xm_own = xm + ((grp * 2 + ph) * 2 + hf) * 64;
        const float* xm_other = xm + ((grp * 2 + ph) * 2 + (hf ^ 1)) * 64;
        xm_own[rl] = mt;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_X + grp));
        // The reference maximum of the tile. Exact order (a piece's first two
        // tiles, or a half whose scores exceed the group's last reference by
        // more than kTau): the row maximum over both halves and the reference
        // after the previous tile (from the other group; a new piece starts
        // afresh but still takes the hand-off, which keeps the reference
        // array's reuse ordered) come first, then P. Speculative order (the
        // steady state, where the reference rarely moves): P is computed
        // against the reference this group used two tiles back, and the
        // exchange and the hand-off are read afterwards, when they have long
        // completed; if the previous tile or this one moved the reference, P
        // is computed again against the exact one before P_FULL. Either way
        // every tile waits for and arrives on B_X and M_READY once.
        bool spec = j >= 2 && m_last != -INFINITY && mt <= m_last + kTau;
        spec = __all_sync(0xffffffffu, spec);
        float m_prev = -INFINITY, m_j = m_last;
        if (!spec) {
          if (!(ok = warp_wait_cta(bar(L::B_X + grp), ph, abort_flag, a.status))) break;
          mt = fmaxf(mt, xm_other[rl]);
          if (jg > 0) {
            if (!(ok = warp_wait_cta(bar(L::B_M_READY + (buf ^ 1)), ((jg - 1) >> 1) & 1, abort_flag, a.status))) break;
            if (j > 0) m_prev = mref[(buf ^ 1) * 64 + rl];
          }
          m_j = (mt > m_prev + kTau) ? mt : m_prev;
          mref[buf * 64 + rl] = m_j;  // both halves write the same value
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::B_M_READY + buf));
        }

        // P buffer is free once the P.V two tiles back has finished
        if (jg >= 2 && !(ok = warp_wait_cta(bar(L::B_P_EMPTY + buf), ph ^ 1, abort_flag, a.status))) break;

        // P = 2^(s * sl2 - m_use), 16 keys (one 16-byte chunk) at a time; this
        // half's 64 keys are bytes [64hf, 64hf + 64) of the 128-byte P row.
        // packed pairs: one FMA and one add for two keys
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        uint64_t se2[2];  // two (even key, odd key) partial sums
        uint8_t* prow = smem + L::kPOff + buf * L::kPBuf + rl * 128;
#pragma unroll 1
        for (;;) {
          const float m_use = (m_j == -INFINITY) ? 0.f : m_j - kSigma;
          const uint64_t nmx2 = f2_pack(-m_use, -m_use);
          se2[0] = se2[1] = 0ull;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int e = 16 * u + 2 * i;
              float a0, a1;
              f2_unpack(fma_f32x2(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sl2x2, nmx2), a0, a1);
              const float p0 = ex2_approx(a0);
              const float p1 = ex2_approx(a1);
              se2[i & 1] = add_f32x2(se2[i & 1], f2_pack(p0, p1));
              const uint32_t qh = cvt_e4m3x2(p0, p1);
              if (i & 1) hi[i >> 1] |= qh << 16; else hi[i >> 1] = qh;
              if (kTwo) {
                const uint32_t rl16 = hsub2(cvt_f16x2(p0, p1), cvt_e4m3x2_to_f16x2(qh));
                const uint32_t ql = cvt_f16x2_to_e4m3x2(rl16);
                if (i & 1) lo[i >> 1] |= ql << 16; else lo[i >> 1] = ql;
              }
            }
            const int phys = (4 * hf + u) ^ (rl & 7);
            *reinterpret_cast<uint4*>(prow + phys * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            if (kTwo && c.two)
              *reinterpret_cast<uint4*>(prow + L::kPPlane + phys * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
          if (!spec) break;
          // confirm the speculation: the row maximum over both halves and the
          // previous tile's reference (j >= 2 here, so jg > 0 and j > 0)
          if (!(ok = warp_wait_cta(bar(L::B_X + grp), ph, abort_flag, a.status))) break;
          mt = fmaxf(mt, xm_other[rl]);
          if (!(ok = warp_wait_cta(bar(L::B_M_READY + (buf ^ 1)), ((jg - 1) >> 1) & 1, abort_flag, a.status))) break;
          m_prev = mref[(buf ^ 1) * 64 + rl];
          const float m_x = (mt > m_prev + kTau) ? mt : m_prev;
          mref[buf * 64 + rl] = m_x;
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::B_M_READY + buf));
          spec = false;
          const bool redo = __any_sync(0xffffffffu, m_x != m_j);
          m_j = m_x;
          if (!redo) break;
        }
        if (!ok) break;
        const float alpha = (m_j == m_prev) ? 1.f : ex2_approx(m_prev - m_j);  // O rescale for tile j

        // rescale this thread's 256 O columns if the reference maximum moved
        // (not on a piece's first tile: O is reset by its first P.V)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!(ok = warp_wait_cta(bar(L::B_O_DONE), (jg - 1) & 1, abort_flag, a.status))) break;
          tc_fence_after();
          // two 32-column chunks per tensor-memory round trip (the score
          // registers are free by now)
#pragma unroll 1
          for (int cc = 0; cc < 8; cc += 2) {
            uint32_t o0[32], o1[32];
            tmem_ld32(tmem + tl + kOCol + 32u * cc, o0);
            tmem_ld32(tmem + tl + kOCol + 32u * (cc + 1), o1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              o0[i] = __float_as_uint(__uint_as_float(o0[i]) * alpha);
              o1[i] = __float_as_uint(__uint_as_float(o1[i]) * alpha);
            }
            tmem_st32(tmem + tl + kOCol + 32u * cc, o0);
            tmem_st32(tmem + tl + kOCol + 32u * (cc + 1), o1);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead(L::B_P_FULL + buf);

        // row-sum bookkeeping, after the hand-off (the P.V does not need it)
        float s0, s1, s2, s3;
        f2_unpack(se2[0], s0, s1);
        f2_unpack(se2[1], s2, s3);
        const float sum = (s0 + s1) + (s2 + s3);
        l_grp = (m_grp == m_j) ? l_grp + sum : fmaf(l_grp, ex2_approx(m_grp - m_j), sum);
        m_grp = m_j;
        m_last = m_j;
      }

      // ---------------------------------------------------------- epilogue of the piece
      // Row sum over both groups and both key halves, relative to the final
      // reference maximum.
      ok = __all_sync(0xffffffffu, ok);
      fin[((0 * 2 + grp) * 2 + hf) * 64 + rl] = l_grp;
      fin[((1 * 2 + grp) * 2 + hf) * 64 + rl] = m_grp;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_FIN));
      if (ok) ok = warp_wait_cta(bar(L::B_FIN), k & 1, abort_flag, a.status);
      float le = 0.f, m_fin = -INFINITY;
      if (ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) m_fin = fmaxf(m_fin, fin[(4 + i) * 64 + rl]);
        if (m_fin != -INFINITY) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float mi = fin[(4 + i) * 64 + rl];
            if (mi != -INFINITY) le += fin[i * 64 + rl] * ex2_approx(mi - m_fin);
          }
        }
      }
      if (ok) ok = warp_wait_cta(bar(L::B_O_FINAL), k & 1, abort_flag, a.status);
      if (!ok) break;
      tc_fence_after();
      const float inv = (le > 0.f) ? a.v_scale / le : 0.f;
      // partial slot of a cut piece: 2p when it begins inside its unit (only
      // a pair's first piece can), 2p + 1 when it begins at the unit's start
      // (then it is cut at the end: the pair's last piece)
      // (test mode 2 of the checking build: every slot past the partials' end)
      const int64_t slot =
          2 * (int64_t)pair + (c.cont ? 0 : 1) + (MLA_BOUNDS_CHECK && p.fault_test == 2 ? balanced_slots(a) : 0);
      if (r < c.rows && grp == 0 && hf == 0) {
        const float lse_val = (le > 0.f) ? (m_fin - kSigma + log2f(le)) * kLn2 : -INFINITY;
        if (c.whole) {
          if (a.lse && in_bounds(a, c.row0 + r, out_rows(a))) a.lse[c.row0 + r] = lse_val;
        } else if (in_bounds(a, slot * M + r, balanced_slots(a) * M)) {
          a.lse_part[slot * M + r] = lse_val;
        }
      }
      if (!(c.whole && last_piece)) {
        // Straight from registers. Partial slots use the layout
        // [slot][16-byte column chunk][row]: the 32 consecutive rows of a warp
        // then store 512 contiguous bytes per instruction. A whole unit that
        // is not the pair's last piece is stored as BF16 rows.
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + kOCol + 128u * grp + 32u * cc, o);
          tmem_wait_ld();
          if (r >= c.rows) continue;
          const int col = 256 * grp + 128 * hf + 32 * cc;
          if (c.whole ? !in_bounds(a, c.row0 + r, out_rows(a)) : !in_bounds(a, slot * M + r, balanced_slots(a) * M))
            continue;
          if (c.whole) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + (c.row0 + r) * MLA_D_V + col);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float f0 = inv > 0.f ? __uint_as_float(o[8 * u + 2 * e]) * inv : 0.f;
                const float f1 = inv > 0.f ? __uint_as_float(o[8 * u + 2 * e + 1]) * inv : 0.f;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(f0, f1);
                pk[e] = *reinterpret_cast<uint32_t*>(&h2);
              }
              dst[u] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int64_t c4 = col / 4 + u;  // 16-byte column chunk
              float4 f;
              f.x = inv > 0.f ? __uint_as_float(o[4 * u + 0]) * inv : 0.f;
              f.y = inv > 0.f ? __uint_as_float(o[4 * u + 1]) * inv : 0.f;
              f.z = inv > 0.f ? __uint_as_float(o[4 * u + 2]) * inv : 0.f;
              f.w = inv > 0.f ? __uint_as_float(o[4 * u + 3]) * inv : 0.f;
              *reinterpret_cast<float4*>(a.o_part + ((slot * (MLA_D_V / 4) + c4) * M + r) * 4) = f;
            }
          }
        }
        if (!c.whole) {
          // this warp's share of the unit's partial O and LSE is stored: one
          // of the kPieceArrivals arrivals the combine waits for per piece
          __syncwarp();
          if (lane == 0) {
            __threadfence();
            const int u = load_piece(a, smem, k).u;
            if (in_bounds(a, u, balanced_units(a))) atomicAdd(a.unit_done + u, 1);
          }
        }
        if (!last_piece) {
          // O may be reset by the next piece's first P.V
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_lead(L::B_O_FREE);
        }
      } else {
        // A whole unit as the pair's last piece: the K and V rings are idle,
        // so the output tile is staged there and written back by whole rows:
        // a warp then stores 512 contiguous bytes per instruction instead of
        // 32 rows' scattered pieces. Staging row r keeps its 16-byte chunk c at
        // position c ^ (r & 7), so that neither the per-row writes nor the
        // per-row reads conflict on shared-memory banks.
        float* stage = reinterpret_cast<float*>(smem + L::kKOff);  // [64 rows][512] fp32
        float* rowinv = mref;                                        // free once the loop is done
        if (grp == 0 && hf == 0) rowinv[rl] = inv;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + kOCol + 128u * grp + 32u * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int ch = 64 * grp + 32 * hf + 8 * cc + i;  // 16-byte chunk of the 2 KB row
            *reinterpret_cast<uint4*>(stage + rl * MLA_D_V + ((ch ^ (rl & 7)) * 4)) =
                make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_EPI));
        if (!(ok = warp_wait_cta(bar(L::B_EPI), 0, abort_flag, a.status))) break;
        // softmax warp w writes local rows 8w .. 8w+7
        const int w8 = warp - kSoftmaxWarp0;
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
          const int rr = 8 * w8 + i;
          if (64 * (int)rank + rr >= c.rows) break;  // rows past the unit belong to no output
          const float inv2 = rowinv[rr];
          const int rr_u = 64 * (int)rank + rr;  // row within the unit
          if (!in_bounds(a, c.row0 + rr_u, out_rows(a))) continue;
          const float* srow = stage + rr * MLA_D_V;
          {
            // BF16: a lane writes 8 consecutive values (16 bytes) per step
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int c0 = 2 * lane + 64 * kk;
              const float4 x0 = *reinterpret_cast<const float4*>(srow + ((c0 ^ (rr & 7)) * 4));
              const float4 x1 = *reinterpret_cast<const float4*>(srow + (((c0 + 1) ^ (rr & 7)) * 4));
              const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 h2 = __floats2bfloat162_rn(inv2 > 0.f ? v[2 * e] * inv2 : 0.f,
                                                          inv2 > 0.f ? v[2 * e + 1] * inv2 : 0.f);
                pk[e] = *reinterpret_cast<uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + (c.row0 + rr_u) * MLA_D_V + 4 * c0) =
                  make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      }
      jt += c.n_pt;
    }
    tc_fence_before();
  }

  // ---------------------------------------------------------------- teardown
  // MMA completions are multicast to both CTAs, and only some of them are
  // consumed: before the pair may leave, each CTA waits for the last phase of
  // every barrier the leader's commits arrive on, so that no arrival lands in
  // shared memory after the CTA has exited. It runs once every role is done
  // (the epilogue saw the last O_FINAL, so every commit has been triggered
  // and each barrier is at most its last arrival short of its final phase).
  // Each wait is bounded; all are skipped after an abort, when the phases may
  // never complete.
  __syncthreads();
  if (warp == 2 && !*abort_flag && n_all > 0) drain_pair_commits<L>(bar(0), lane, n_all, npc);
  __syncthreads();
  tc_fence_before();
  cluster_sync();  // the peer no longer touches this CTA's shared or tensor memory
  if (warp == 1) {
    tc_fence_after();
    if (*abort_flag) spin_ns(1000000ull);  // let any MMA still in flight finish
    tmem_dealloc_pair(tmem, 512);
  }
}

// Set-up that touches no global memory, so that it runs before the kernel
// waits for the grid it depends on: every barrier (both layouts keep them at
// the same place), the abort flag, the zero rows of a short Q rope box, the
// pair's tensor memory and the tensor-map prefetch; then the cluster sync
// after which both CTAs' barriers and TMEM exist.
__device__ __forceinline__ void pair_setup(const PairParams& prm, uint8_t* smem) {
  using L = PairLayout<false>;
  static_assert(PairLayout<true>::kBarOff == L::kBarOff && PairLayout<true>::kMiscOff == L::kMiscOff &&
                    PairLayout<true>::kQRope == L::kQRope && PairLayout<true>::kNBars == L::kNBars,
                "barriers, TMEM slot and Q rope sit at the same place in both layouts");
  constexpr int NK = L::NK, NV = L::NV, NQ = L::NQ;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kBarOff + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = prm.a.plan.rows_per_unit;
  const int box_q = M < 64 ? M : 64;  // query rows per TMA box (the tensor maps' box height)
  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_Q_MAIN), 1);
    mbar_init(bar(L::B_Q_ROPE), 1);
    mbar_init(bar(L::B_Q_TMEM), 2 * kSoftmaxWarps);
    for (int i = 0; i < NK; ++i) {
      mbar_init(bar(L::B_K_FULL + i), 1);
      mbar_init(bar(L::B_K_EMPTY + i), 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(bar(L::B_V_FULL + i), 1);
      mbar_init(bar(L::B_V_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::B_S_FULL + i), 1);
      mbar_init(bar(L::B_S_EMPTY + i), 2 * 4);  // the tile's softmax group in each CTA
      mbar_init(bar(L::B_P_FULL + i), 2 * 4);
      mbar_init(bar(L::B_P_EMPTY + i), 1);
      mbar_init(bar(L::B_M_READY + i), 4);
      mbar_init(bar(L::B_X + i), 4);
    }
    mbar_init(bar(L::B_O_DONE), 1);
    mbar_init(bar(L::B_O_FINAL), 1);
    mbar_init(bar(L::B_FIN), kSoftmaxWarps);
    for (int i = 0; i < NQ; ++i) mbar_init(bar(L::B_QK_DONE + i), 1);
    mbar_init(bar(L::B_EPI), kSoftmaxWarps);
    mbar_init(bar(L::B_O_FREE), 2 * kSoftmaxWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (box_q < 64) {
    // Q rope rows the TMA box does not cover are zero (rows are independent).
    uint4* rb = reinterpret_cast<uint4*>(smem + L::kQRope + box_q * 64);
    for (int i = threadIdx.x; i < (64 - box_q) * 4; i += blockDim.x) rb[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&prm.tm_q_main);
    prefetch_tmap(&prm.tm_q_rope);
    prefetch_tmap(&prm.tm_kv_main);
    prefetch_tmap(&prm.tm_kv_rope);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA use
  tc_fence_after();
}

// A pair with no work (the same in both CTAs) frees its tensor memory.
__device__ __forceinline__ void pair_idle_teardown(uint8_t* smem) {
  __syncthreads();
  tc_fence_before();
  cluster_sync();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc_pair(*reinterpret_cast<volatile uint32_t*>(smem + kPairMiscOff), 512);
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_fp8_pair_kernel(const __grid_constant__ PairParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SchedInfo* info = reinterpret_cast<SchedInfo*>(smem + kMaxSmemPieces * sizeof(Piece));
  // Launched as a programmatic dependent of the workspace clear: the set-up
  // overlaps the previous step's tail, and no global memory is touched before
  // the clear (and, through it, everything before it in the stream) is done.
  pair_setup(prm, smem);
  grid_dep_wait();
  // The combine grid may now start (the unit counters and the table's ready
  // flag it waits on are cleared) and take the SMs of pairs that finish early.
  launch_dependents();
  build_schedule<kPairTileKeys>(prm.a, blockIdx.x >> 1, cluster_ctarank(), smem);  // every thread
  __syncthreads();
  const int npc = info->npc;
  if (npc == 0) {  // no work for this pair (the same in both CTAs)
    pair_idle_teardown(smem);
    return;
  }
  // The softmax warps wait for the first scores anyway: they drop the L2
  // lines of the pair's partial slots meanwhile.
  if (threadIdx.x >= 32 * kSoftmaxWarp0)
    discard_pair_slots(prm.a, blockIdx.x >> 1, cluster_ctarank(), info->tiles, threadIdx.x - 32 * kSoftmaxWarp0,
                       kThreads - 32 * kSoftmaxWarp0);
  // Short entries send P as two E4M3 terms; a pair with any such piece takes
  // the layout with room for both planes (the choice is the same in both CTAs).
  if (info->two)
    pair_cta<true>(prm, smem, npc, info->tiles);
  else
    pair_cta<false>(prm, smem, npc, info->tiles);
}

}  // namespace

cudaError_t launch_tc_fp8_pair_partial(const DecodeArgs& a, cudaStream_t stream) {
  const mla_plan& p = a.plan;
  if (p.batch == 0 || p.split_kv < 1) return cudaSuccess;
  PairParams prm;
  prm.a = a;
  const uint64_t q_rows = (uint64_t)a.total_q * p.num_heads;  // the packed query rows
  const uint64_t kv_rows = (uint64_t)a.num_pages * kTileKeys;
  const uint32_t box_q = p.rows_per_unit < 64 ? (uint32_t)p.rows_per_unit : 64u;
  if (!encode_rows_576(&prm.tm_q_main, a.q, 1, q_rows, 128, box_q, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_q_rope, a.q, 1, q_rows, 64, box_q, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_rows_576(&prm.tm_kv_main, a.kv_cache, 1, kv_rows, 128, kTileKeys, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_kv_rope, a.kv_cache, 1, kv_rows, 64, kTileKeys, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_max_dynamic_smem((const void*)tc_fp8_pair_kernel, (int)kPairSmemBytes, smem_set);
      e != cudaSuccess)
    return e;
  // a programmatic dependent of the previous kernel in the stream (the
  // workspace clear): it waits for it before touching global memory
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * p.split_kv));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_fp8_pair_kernel, prm);
}

}  // namespace mla
