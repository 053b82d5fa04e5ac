// Split-KV partial kernel for FP8 E4M3 inputs on the sm_100a tensor cores.
//
// The first of the two decode kernels (TokenSpeed MLA article
// 最快MLA内核背后的秘密, section 二) with query-token folding (section 三): the
// M = H*F <= 128 query rows of a (batch entry, query group) share each 64-key
// cache page, which is one dense tile for the 128-row tensor core.
//
// Work split without any cross-CTA traffic. The fp32 output of 128 rows x 512
// columns would fill all of an SM's tensor memory, so two CTAs share a
// (entry, group, split): CTA h keeps output columns [256h, 256h+256). Each of
// the two computes the full scores S = Q.K^T and the full softmax itself, so
// they never exchange data; their inputs and instruction streams are the
// same, so the softmax statistics (and P) are bitwise identical in both. The
// two CTAs are adjacent in the grid and read the same pages at about the same
// time, so the second read of a page is served by L2. (Distributed shared
// memory between the CTAs of a cluster moves only ~23 GB/s per SM on B200,
// far too little to exchange per-tile scores at HBM speed.)
//
// Tensor memory (512 columns): O half [0,256); Q latent dims 0..511 as the A
// operand of S = Q.K^T [256,384) (four E4M3 codes per 32-bit column, row r in
// lane r); two S buffers [384,448) and [448,512). The 64 rope dims of Q stay
// in shared memory (A from shared memory for those two MMAs).
//
// P = 2^(x - m + SIGMA) with x the log2-scaled score and m a lazily updated
// row maximum (moved only when exceeded by more than TAU). P is an E4M3
// operand; for entries shorter than kTwoTermKeys it is sent as two E4M3 terms
// (hi = e4m3(P), lo = e4m3(P - hi) via f16; two P.V MMAs) so that short rows
// keep about 8 significant bits; long rows average the 3-bit rounding away.
// O is normalised by the exact fp32 sum of P, which also gives the LSE.
//
// Roles (352 threads): warp 0 lane 0 issues TMA (Q once, then one full
// 576-byte-per-key page per stage through the block table); warp 1 owns TMEM
// and issues S = Q.K^T up to two tiles ahead; warp 10 issues O += P.V; warps
// 2-9 form two softmax groups of four warps that take alternate tiles (one
// thread per row, all 64 keys of the tile), do the O rescales, and share the
// epilogue (group g stores output columns [128g, 128g+128) of the CTA's half).
// Q's latent dims reach TMEM through shared memory (TMA, then tcgen05.st).
// Every wait is bounded; on expiry the CTA sets MLA_DEV_TIMEOUT, leaves the
// pipeline, frees TMEM and returns.
#include <cuda.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr float kTau = 2.f;                // lazy-rescale threshold (log2 units)
constexpr float kSigma = 6.f;              // P <= 2^(kTau + kSigma) = 256 <= 448

// Each cache page is split over two rings of shared-memory slots: the V ring
// holds this CTA's half of the 512 latent dims (the V operand of its P.V, and
// half of K), kept until that P.V completes; the K ring holds the other half
// plus the 64 rope dims, freed as soon as S = Q.K^T has been computed. A K
// slot is held for about the load latency, a V slot for that plus the
// softmax, so splitting the page roughly doubles the pages in flight.
template <bool kTwo>
struct Fp8Layout {
  static constexpr int NK = 4;                                  // K-ring slots
  static constexpr int NV = kTwo ? 6 : 7;                       // V-ring slots
  static constexpr uint32_t kQRope = 0;                         // 128 rows x 64 B (SW64)
  static constexpr uint32_t kPPlane = 128 * 64;                 // one E4M3 plane of P (SW64)
  static constexpr uint32_t kPBuf = (kTwo ? 2 : 1) * kPPlane;   // hi (and lo) plane
  static constexpr uint32_t kPOff = 8192;                       // P[2 buffers]
  static constexpr uint32_t kKSlot = 2 * 8192 + 64 * 64;        // 2 x 8 KB main (SW128) + 4 KB rope (SW64)
  static constexpr uint32_t kKOff = kPOff + 2 * kPBuf;
  static constexpr uint32_t kVSlot = 2 * 8192;                  // 2 x 8 KB main (SW128)
  static constexpr uint32_t kVOff = kKOff + NK * kKSlot;
  static constexpr uint32_t kMOff = kVOff + NV * kVSlot;        // row reference maxima [2 tile parities][128]
  static constexpr uint32_t kFinOff = kMOff + 1024;             // final (l, m) per group [2][2][128]
  static constexpr uint32_t kBarOff = kFinOff + 2048;
  // Q latent dims are staged (TMA, SW128, 4 chunks of 128 rows x 128 B) in
  // V slots NV-4 .. NV-1 before those are first filled with a page.
  static constexpr uint32_t kQStage = kVOff + (NV - 4) * kVSlot;
  // barriers
  static constexpr int B_Q_ROPE = 0;
  static constexpr int B_Q_TMEM = 1;
  static constexpr int B_Q_MAIN = 2;
  static constexpr int B_FULL = 3;                 // + V slot: all 36 KB of the page landed
  static constexpr int B_V_EMPTY = B_FULL + NV;    // + V slot
  static constexpr int B_K_EMPTY = B_V_EMPTY + NV; // + K slot
  static constexpr int B_S_FULL = B_K_EMPTY + NK;  // + buffer
  static constexpr int B_S_EMPTY = B_S_FULL + 2;   // + buffer
  static constexpr int B_P_FULL = B_S_EMPTY + 2;   // + buffer
  static constexpr int B_P_EMPTY = B_P_FULL + 2;   // + buffer
  static constexpr int B_O_DONE = B_P_EMPTY + 2;
  static constexpr int B_O_FINAL = B_O_DONE + 1;   // completes once, after the last P.V
  static constexpr int B_M_READY = B_O_FINAL + 1;  // + tile parity: a group published its row maxima
  static constexpr int B_FIN = B_M_READY + 2;      // both groups published their final (l, m)
  static constexpr int kNBars = B_FIN + 1;
  static_assert(8 * kNBars <= 512, "barrier area");
  static constexpr uint32_t kMiscOff = kBarOff + 512;
  static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;
  static_assert(kKOff % 1024 == 0 && kKSlot % 1024 == 0 && kVOff % 1024 == 0, "alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

constexpr int kSoftmaxWarps = 8;
constexpr int kPvWarp = 10;                          // issues P.V (warp 1 issues S = Q.K^T)
constexpr int kThreads = 32 * (3 + kSoftmaxWarps);

// tensor memory columns
constexpr uint32_t kOCol = 0;
constexpr uint32_t kQCol = 256;
constexpr uint32_t kSCol = 384;

struct Fp8Params {
  CUtensorMap tm_q_main, tm_q_rope, tm_kv_main, tm_kv_rope;
  DecodeArgs a;
};

__device__ __forceinline__ float max32(const float (&x)[32]) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fmaxf(x[4 * i], x[4 * i + 1]), fmaxf(x[4 * i + 2], x[4 * i + 3]));
#pragma unroll
  for (int w = 4; w > 0; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

// One CTA's work; kTwo selects two-term P and the matching shared-memory layout.
template <bool kTwo>
__device__ __forceinline__ void fp8_cta(const Fp8Params& prm, uint8_t* smem_raw) {
  using L = Fp8Layout<kTwo>;
  constexpr int NK = L::NK, NV = L::NV;
  constexpr int B_Q_ROPE = L::B_Q_ROPE, B_Q_TMEM = L::B_Q_TMEM, B_Q_MAIN = L::B_Q_MAIN, B_FULL = L::B_FULL,
                B_V_EMPTY = L::B_V_EMPTY, B_K_EMPTY = L::B_K_EMPTY, B_S_FULL = L::B_S_FULL,
                B_S_EMPTY = L::B_S_EMPTY, B_P_FULL = L::B_P_FULL, B_P_EMPTY = L::B_P_EMPTY,
                B_O_DONE = L::B_O_DONE, B_O_FINAL = L::B_O_FINAL, B_M_READY = L::B_M_READY, B_FIN = L::B_FIN;
  const DecodeArgs& a = prm.a;
  const mla_plan& p = a.plan;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kBarOff + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hv = blockIdx.x & 1;  // output-column half of this CTA
  const int pair = blockIdx.x >> 1;
  const int G = p.q_groups, S = p.split_kv, T = p.q_len, H = p.num_heads, M = p.rows_per_unit;
  const int g = pair % G;
  const int s = (pair / G) % S;
  const int b = pair / (G * S);
  const int n = effective_seq_len(a, b, hv == 0 && s == 0 && g == 0 && threadIdx.x == 0);
  const int key0 = s * p.keys_per_split;
  const int64_t row0 = (int64_t)b * T * H + (int64_t)g * M;

  if (key0 >= n) {
    if (S == 1) {
      for (int r = threadIdx.x; r < M; r += blockDim.x) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + (row0 + r) * MLA_D_V + 256 * hv);
        for (int i = 0; i < 32; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        if (hv == 0 && a.lse) a.lse[row0 + r] = -INFINITY;
      }
    }
    return;
  }
  const int key1 = min(n, key0 + p.keys_per_split);
  const int n_tiles = (key1 - key0 + kTileKeys - 1) / kTileKeys;
  const int tile0 = key0 / kTileKeys;
  const int32_t* table = a.block_tables + (int64_t)b * a.max_pages_per_seq;
  constexpr bool two_term = kTwo;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q_ROPE), 1);
    mbar_init(bar(B_Q_TMEM), kSoftmaxWarps);
    mbar_init(bar(B_Q_MAIN), 1);
    for (int i = 0; i < NV; ++i) {
      mbar_init(bar(B_FULL + i), 1);
      mbar_init(bar(B_V_EMPTY + i), 1);   // released by the P.V issuer
    }
    for (int i = 0; i < NK; ++i) mbar_init(bar(B_K_EMPTY + i), 1);  // released by the QK issuer
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_S_FULL + i), 1);
      mbar_init(bar(B_S_EMPTY + i), 4);   // one softmax group (4 warps) per tile parity
      mbar_init(bar(B_P_FULL + i), 4);
      mbar_init(bar(B_M_READY + i), 4);
      mbar_init(bar(B_P_EMPTY + i), 1);
    }
    mbar_init(bar(B_O_DONE), 1);
    mbar_init(bar(B_O_FINAL), 1);
    mbar_init(bar(B_FIN), kSoftmaxWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (M < 128) {
    // Q rope rows the TMA box does not cover are zero (rows are independent).
    uint4* rb = reinterpret_cast<uint4*>(smem + L::kQRope + M * 64);
    for (int i = threadIdx.x; i < (128 - M) * 4; i += blockDim.x) rb[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&prm.tm_q_main);
      prefetch_tmap(&prm.tm_q_rope);
      prefetch_tmap(&prm.tm_kv_main);
      prefetch_tmap(&prm.tm_kv_rope);
      const uint64_t pol_q = policy_evict_last();
      // The pair's other CTA reads the same pages right after: keep them in L2.
      const uint64_t pol_kv = policy_evict_last();
      mbar_arrive_expect_tx(bar(B_Q_MAIN), 4u * 128u * (uint32_t)M);
#pragma unroll
      for (int ci = 0; ci < 4; ++ci)
        tma_load_2d(sb + L::kQStage + ci * 16384, &prm.tm_q_main, 128 * ci,
                    (int)row0, bar(B_Q_MAIN), pol_q);
      mbar_arrive_expect_tx(bar(B_Q_ROPE), 64u * (uint32_t)M);
      tma_load_2d(sb + L::kQRope, &prm.tm_q_rope, 512, (int)row0, bar(B_Q_ROPE), pol_q);
      for (int j = 0; j < n_tiles; ++j) {
        const int sk = j % NK, sv = j % NV;
        // V slots NV-4 .. NV-1 hold staged Q until it has been copied into TMEM
        if (j == NV - 4 && !bounded_wait(bar(B_Q_TMEM), 0, abort_flag, a.status)) break;
        if (!bounded_wait(bar(B_K_EMPTY + sk), ((j / NK) & 1) ^ 1, abort_flag, a.status)) break;
        if (!bounded_wait(bar(B_V_EMPTY + sv), ((j / NV) & 1) ^ 1, abort_flag, a.status)) break;
        int page = table[tile0 + j];
        if (page < 0 || (int64_t)page >= a.num_pages) page = 0;  // masked by the softmax warps
        const uint32_t vs = sb + L::kVOff + sv * L::kVSlot;
        const uint32_t ks = sb + L::kKOff + sk * L::kKSlot;
        const uint32_t full = bar(B_FULL + sv);
        mbar_arrive_expect_tx(full, L::kVSlot + L::kKSlot);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(vs + c * 8192, &prm.tm_kv_main, 128 * (2 * hv + c), page * kTileKeys, full, pol_kv);
          tma_load_2d(ks + c * 8192, &prm.tm_kv_main, 128 * (2 - 2 * hv + c), page * kTileKeys, full, pol_kv);
        }
        tma_load_2d(ks + 16384, &prm.tm_kv_rope, 512, page * kTileKeys, full, pol_kv);
      }
      drain_loads(bar(B_FULL), NV, n_tiles);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK issuer
    // The whole warp runs this loop with warp-uniform operands; one elected
    // lane issues each MMA and commit. S for tile j needs only a free S buffer
    // and the page, so the scores run up to two tiles ahead of the softmax.
    {
      constexpr uint32_t idq = instr_desc(0, 0, 0, 128, 64);   // E4M3 x E4M3, K-major B
      bool ok = warp_wait(bar(B_Q_ROPE), 0, abort_flag, a.status) &&
                warp_wait(bar(B_Q_TMEM), 0, abort_flag, a.status);
      const uint64_t dq_rope = smem_desc(sb + L::kQRope, 16, 512, kSw64);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int sk = j % NK, sv = j % NV, buf = j & 1;
        if (!(ok = warp_wait(bar(B_FULL + sv), (j / NV) & 1, abort_flag, a.status))) break;
        if (!(ok = warp_wait(bar(B_S_EMPTY + buf), ((j >> 1) & 1) ^ 1, abort_flag, a.status))) break;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + 64u * buf;
        const uint32_t vs = sb + L::kVOff + sv * L::kVSlot;
        const uint32_t ks = sb + L::kKOff + sk * L::kKSlot;
        const uint64_t dr = smem_desc(ks + 16384, 16, 512, kSw64);
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) {
          // latent chunk ci (dims 128ci ..) sits in the V slot for this CTA's half
          const uint64_t dk = smem_desc(((ci >> 1) == hv ? vs : ks) + (ci & 1) * 8192, 16, 1024, kSw128);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts_e(d, tmem + kQCol + (uint32_t)(8 * (4 * ci + kk)), dk + (uint64_t)((kk * 32) >> 4), idq,
                        (ci | kk) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) mma_f8_ss_e(d, dq_rope + (uint64_t)(kk * 2), dr + (uint64_t)(kk * 2), idq, 1u);
        mma_commit_e(bar(B_S_FULL + buf));
        mma_commit_e(bar(B_K_EMPTY + sk));
      }
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ P.V issuer
    constexpr uint32_t idp = instr_desc(0, 0, 1, 128, 256);  // V is MN-major
    bool ok = true;
    for (int j = 0; ok && j < n_tiles; ++j) {
      const int buf = j & 1, sv = j % NV;
      if (!(ok = warp_wait(bar(B_P_FULL + buf), (j >> 1) & 1, abort_flag, a.status))) break;
      tc_fence_after();
      const uint64_t dv = smem_desc(sb + L::kVOff + sv * L::kVSlot, 8192, 1024, kSw128);
      const uint64_t dp = smem_desc(sb + L::kPOff + buf * L::kPBuf, 16, 512, kSw64);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        mma_f8_ss_e(tmem + kOCol, dp + (uint64_t)(kk * 2), dv + (uint64_t)(kk * 256), idp, (j > 0 || kk > 0) ? 1u : 0u);
      if (two_term) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_f8_ss_e(tmem + kOCol, dp + (uint64_t)((L::kPPlane + kk * 32) >> 4), dv + (uint64_t)(kk * 256), idp, 1u);
      }
      // O_DONE first: a softmax group that has seen P_EMPTY of tile j-2 may
      // rely on O_DONE having completed that tile's phase too.
      mma_commit_e(bar(B_O_DONE));
      mma_commit_e(bar(B_P_EMPTY + buf));
      mma_commit_e(bar(B_V_EMPTY + sv));
      if (j == n_tiles - 1) mma_commit_e(bar(B_O_FINAL));
    }
  } else if (warp >= 2 && warp < 2 + kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax warps
    // Two groups of four warps take alternate tiles (group g: tiles g, g+2,
    // ...), so two tiles are in flight. Warp w serves TMEM lane quarter w%4,
    // one thread per row with all 64 keys of the tile. The only per-tile
    // coupling is the row reference maximum, handed from the group of tile j-1
    // to the group of tile j through shared memory.
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int r = 32 * q + lane;  // this thread's row (= TMEM lane)
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int limit = (r < M) ? n - T + g * p.fold + r / H : n - 1;
    float* mref = reinterpret_cast<float*>(smem + L::kMOff);   // [tile parity][row]
    float* fin = reinterpret_cast<float*>(smem + L::kFinOff);  // [l | m][group][row]
    bool ok = true;

    // Q latent dims 0..511 of row r: staged by TMA (SW128 chunks of 128 bytes =
    // 32 TMEM columns), copied into TMEM as the A operand; group g copies
    // chunks 2g and 2g+1.
    ok = warp_wait(bar(B_Q_MAIN), 0, abort_flag, a.status);
    if (ok) {
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int cc = 2 * grp + c2;
        const uint8_t* chunk = smem + L::kQStage + cc * 16384 + r * 128;
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(chunk + ((u ^ (r & 7)) * 16));
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        if (r >= M) {
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = 0;
        }
        tmem_st32(tmem + tl + kQCol + 32u * cc, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_Q_TMEM));
    }

    const float sl2 = a.score_scale_log2;
    float m_grp = -INFINITY, l_grp = 0.f;   // this group's reference and sum (relative to m_grp)
    int pg_next = (grp < n_tiles) ? table[tile0 + grp] : 0;
    for (int j = grp; ok && j < n_tiles; j += 2) {
      const int buf = j & 1;  // == grp
      const int pg = pg_next;
      if (j + 2 < n_tiles) pg_next = table[tile0 + j + 2];  // prefetch: off the critical path
      if (!(ok = warp_wait(bar(B_S_FULL + buf), (j >> 1) & 1, abort_flag, a.status))) break;
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
      if (lane == 0) mbar_arrive(bar(B_S_EMPTY + buf));

      const bool page_ok = pg >= 0 && (int64_t)pg < a.num_pages;
      if (!page_ok && lane == 0 && q == 2) atomicOr(a.status, MLA_DEV_BAD_PAGE);
      const int kb = key0 + kTileKeys * j;
      // raw scores; masked keys become -inf (sl2 > 0, so max commutes with the scale)
      if (!(page_ok && kb + 63 <= limit)) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (!(page_ok && kb + i <= limit)) sv[i] = __float_as_uint(-INFINITY);
      }
      float mt;
      {
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float t = __uint_as_float(sv[8 * i]);
#pragma unroll
          for (int k = 1; k < 8; ++k) t = fmaxf(t, __uint_as_float(sv[8 * i + k]));
          m8[i] = t;
        }
        mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * sl2;
      }
      // reference maximum after tile j-1 (from the other group), lazily updated
      float m_prev = -INFINITY;
      if (j > 0) {
        if (!(ok = warp_wait(bar(B_M_READY + (buf ^ 1)), ((j - 1) >> 1) & 1, abort_flag, a.status))) break;
        m_prev = mref[(buf ^ 1) * 128 + r];
      }
      const float m_j = (mt > m_prev + kTau) ? mt : m_prev;
      mref[buf * 128 + r] = m_j;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_M_READY + buf));
      const float alpha = (m_j == m_prev) ? 1.f : ex2_approx(m_prev - m_j);  // O rescale for tile j
      const float m_use = (m_j == -INFINITY) ? 0.f : m_j - kSigma;

      // P buffer is free once the P.V two tiles back has finished
      if (j >= 2 && !(ok = warp_wait(bar(B_P_EMPTY + buf), ((j >> 1) & 1) ^ 1, abort_flag, a.status))) break;

      // P = 2^(s * sl2 - m_use), 16 keys (one 16-byte chunk) at a time. The
      // exact fp32 sum normalises O and gives the LSE (E4M3 rounding is
      // unbiased and averages out; short rows use the two-term split).
      float se[4] = {0.f, 0.f, 0.f, 0.f};
      uint8_t* prow = smem + L::kPOff + buf * L::kPBuf + r * 64;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = 16 * u + 2 * i;
          const float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -m_use));
          se[i & 3] += p0 + p1;
          const uint32_t qh = cvt_e4m3x2(p0, p1);
          if (i & 1) hi[i >> 1] |= qh << 16; else hi[i >> 1] = qh;
          if (two_term) {
            const uint32_t ph = cvt_f16x2(p0, p1);
            const uint32_t rl = hsub2(ph, cvt_e4m3x2_to_f16x2(qh));
            const uint32_t ql = cvt_f16x2_to_e4m3x2(rl);
            if (i & 1) lo[i >> 1] |= ql << 16; else lo[i >> 1] = ql;
          }
        }
        const int phys = u ^ ((r >> 1) & 3);
        *reinterpret_cast<uint4*>(prow + phys * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (two_term) *reinterpret_cast<uint4*>(prow + L::kPPlane + phys * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      const float sum = (se[0] + se[1]) + (se[2] + se[3]);
      l_grp = (m_grp == m_j) ? l_grp + sum : fmaf(l_grp, ex2_approx(m_grp - m_j), sum);
      m_grp = m_j;

      // rescale O (all 256 columns of this row) if the reference maximum moved
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!(ok = warp_wait(bar(B_O_DONE), (j - 1) & 1, abort_flag, a.status))) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + kOCol + 32u * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + tl + kOCol + 32u * cc, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + buf));
    }

    // ------------------------------------------------------------ epilogue
    // Combine the two groups' sums, relative to the final reference maximum.
    ok = __all_sync(0xffffffffu, ok);
    fin[(0 * 2 + grp) * 128 + r] = l_grp;
    fin[(1 * 2 + grp) * 128 + r] = m_grp;
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_FIN));
    if (ok) ok = warp_wait(bar(B_FIN), 0, abort_flag, a.status);
    float le = 0.f, m_fin = -INFINITY;
    if (ok) {
      const float l0 = fin[0 * 128 + r], l1 = fin[1 * 128 + r];
      const float m0 = fin[2 * 128 + r], m1 = fin[3 * 128 + r];
      m_fin = fmaxf(m0, m1);
      if (m_fin != -INFINITY)
        le = (m0 == -INFINITY ? 0.f : l0 * ex2_approx(m0 - m_fin)) + (m1 == -INFINITY ? 0.f : l1 * ex2_approx(m1 - m_fin));
    }
    // (B_O_DONE's parity cannot tell late phases apart here.)
    if (ok) ok = warp_wait(bar(B_O_FINAL), 0, abort_flag, a.status);
    if (ok) {
      tc_fence_after();
      const float inv = (le > 0.f) ? a.v_scale / le : 0.f;
      const bool live = r < M;
      const int64_t rg = row0 + r;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        const uint32_t col = 128u * grp + 32u * cc;   // group g writes columns [128g, 128g+128)
        tmem_ld32(tmem + tl + kOCol + col, o);
        tmem_wait_ld();
        if (!live) continue;
        store_out_chunk(a, rg, s, 256 * hv + (int)col, o, inv);
      }
      if (live && hv == 0 && grp == 0) {
        const float lse_val = (le > 0.f) ? (m_fin - kSigma + log2f(le)) * kLn2 : -INFINITY;
        if (S == 1) {
          if (a.lse) a.lse[rg] = lse_val;
        } else {
          a.lse_part[rg * S + s] = lse_val;
        }
      }
    }
    tc_fence_before();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (*abort_flag) spin_ns(1000000ull);  // let any MMA still in flight finish
    tmem_dealloc(tmem, 512);
  }
}

static_assert(Fp8Layout<true>::kSmemBytes == Fp8Layout<false>::kSmemBytes, "both variants share one launch");

__global__ void __launch_bounds__(kThreads, 1) tc_fp8_partial_kernel(const __grid_constant__ Fp8Params prm) {
  extern __shared__ uint8_t smem_raw[];
  const mla_plan& p = prm.a.plan;
  const int b = (blockIdx.x >> 1) / (p.q_groups * p.split_kv);
  // Entries shorter than kTwoTermKeys send P as two E4M3 terms (the choice
  // is per entry, so it is uniform over the CTA).
  if (effective_seq_len(prm.a, b, false) < kTwoTermKeys)
    fp8_cta<true>(prm, smem_raw);
  else
    fp8_cta<false>(prm, smem_raw);
}

}  // namespace

cudaError_t launch_tc_fp8_partial(const DecodeArgs& a, cudaStream_t stream) {
  const mla_plan& p = a.plan;
  const uint64_t pairs = (uint64_t)p.batch * p.q_groups * p.split_kv;
  if (pairs == 0) return cudaSuccess;
  Fp8Params prm;
  prm.a = a;
  const uint64_t q_rows = (uint64_t)p.batch * p.q_len * p.num_heads;
  const uint64_t kv_rows = (uint64_t)a.num_pages * kTileKeys;
  if (!encode_rows_576(&prm.tm_q_main, a.q, 1, q_rows, 128, p.rows_per_unit, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_q_rope, a.q, 1, q_rows, 64, p.rows_per_unit, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_rows_576(&prm.tm_kv_main, a.kv_cache, 1, kv_rows, 128, kTileKeys, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_kv_rope, a.kv_cache, 1, kv_rows, 64, kTileKeys, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_max_dynamic_smem((const void*)tc_fp8_partial_kernel, (int)Fp8Layout<false>::kSmemBytes,
                                           smem_set);
      e != cudaSuccess)
    return e;
  tc_fp8_partial_kernel<<<(unsigned)(2 * pairs), kThreads, Fp8Layout<false>::kSmemBytes, stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace mla
