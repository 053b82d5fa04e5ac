// Split-KV partial kernel on the sm_100a tensor cores (TMA + tcgen05 + TMEM).
//
// The first of the two decode kernels (TokenSpeed MLA article
// 最快MLA内核背后的秘密, section 二), with query-token folding (section 三):
// the M = H*F <= 128 query rows of one (batch entry, query group) share every
// 64-key page of the cache, so each page is one dense contraction with M in
// the tensor core's 128-row dimension.
//
// Work split. One CTA pair (a 2-CTA cluster) per (entry, group, split). The
// fp32 output O of 128 rows x 512 columns alone would fill all 512 TMEM
// columns of an SM, so CTA c keeps the output columns [256c, 256c+256) and
// owns the matching half of the reduction dims of S = Q.K^T: latent dims
// [256c, 256c+256) plus rope dims [512+32c, 512+32c+32). Each CTA therefore
// loads only its 288-dim slice of every cache row (no byte is read twice),
// computes a partial S over its slice, and the partials are summed across
// the pair through distributed shared memory. Row r is "owned" by CTA
// (r / 16) % 2: the owner finishes the softmax of its 64 rows (two threads
// per row, one per 32-key half), writes P for them into its own shared
// memory and copies those rows to the peer, so both CTAs hold the full P for
// their O += P.V with V = their 256-column slice of the same cache tile.
// Lazy rescaling: the reference maximum of a row only moves when the tile
// maximum exceeds it by more than TAU (log2 units); the factor travels with
// P to the peer, which rescales its half of the row.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads (Q slice once, then a
// stage per page through the block table); warp 1 owns TMEM and lane 0
// issues the MMAs; warps 2-5 (TMEM lane quarters 2,3,0,1) run the exchange,
// softmax, rescale and epilogue. Every wait is bounded: on expiry the CTA
// sets MLA_DEV_TIMEOUT, abandons the pipeline, frees TMEM and returns.
#include <cuda.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace mla {
namespace {

using namespace ptx;

template <int DT>
struct Cfg {
  static constexpr int E = (DT == MLA_FP8_E4M3) ? 1 : 2;  // bytes per element
  static constexpr int CHUNK_ELEMS = 128 / E;              // elements per 128-byte swizzle row
  static constexpr int MAIN_CHUNKS = 256 / CHUNK_ELEMS;    // 4 (16-bit) or 2 (FP8)
  static constexpr int ROPE_BYTES = 32 * E;                // bytes of the 32 rope dims per row
  static constexpr uint32_t ROPE_SW = (E == 2) ? kSw64 : kSw32;
  static constexpr int NS = (E == 2) ? 3 : 6;              // pipeline stages (cache tiles)
  static constexpr int MMA_K = 32 / E;                     // K elements per MMA (32 bytes)
  static constexpr int P_ROW = 64 * E;                     // bytes of one P row (64 keys)
  static constexpr int P_PLANES = (E == 2) ? 1 : 2;        // FP8: hi and lo E4M3 terms
  static constexpr uint32_t P_SW = (E == 2) ? kSw128 : kSw64;
  static constexpr uint32_t FMT = (DT == MLA_BF16) ? 1u : 0u;  // bf16=1, fp16=0, e4m3=0

  // shared memory layout (bytes from a 1024-aligned base)
  static constexpr uint32_t Q_MAIN = 0;                                 // MAIN_CHUNKS x 16 KB
  static constexpr uint32_t Q_ROPE = MAIN_CHUNKS * 16384;               // 128 rows x ROPE_BYTES
  static constexpr uint32_t STAGE0 = Q_ROPE + 128 * ROPE_BYTES;         // multiple of 1024
  static constexpr uint32_t STAGE_MAIN = MAIN_CHUNKS * 8192;            // 64 rows x 128 B per chunk
  static constexpr uint32_t STAGE_BYTES = STAGE_MAIN + 64 * ROPE_BYTES;
  static constexpr uint32_t P_OFF = STAGE0 + NS * STAGE_BYTES;
  static constexpr uint32_t SX_ROW = 64 * 4 + 16;                       // padded: no bank conflicts
  static constexpr uint32_t P_PLANE = 128 * P_ROW;                      // bytes of one P plane
  static constexpr uint32_t SX_OFF = P_OFF + P_PLANES * P_PLANE;
  static constexpr uint32_t ALPHA_OFF = SX_OFF + 64 * SX_ROW;
  static constexpr uint32_t FIN_OFF = ALPHA_OFF + 512;
  static constexpr uint32_t BAR_OFF = FIN_OFF + 512;
  static constexpr int NBARS = 2 * NS + 12;
  static constexpr uint32_t MISC_OFF = BAR_OFF + 8 * NBARS;
  static constexpr uint32_t SMEM_BYTES = MISC_OFF + 16 + 1024;  // + alignment slack

  static constexpr uint32_t Q_TILE_BYTES_PER_ROW = MAIN_CHUNKS * 128 + ROPE_BYTES;
  static constexpr uint32_t P_PEER_BYTES = 4 * (P_PLANES * 16 * P_ROW + 64);  // peer's P rows + factors
  static constexpr float TAU = (E == 2) ? 8.f : 2.f;               // lazy-rescale threshold (log2)
  static constexpr float SIGMA = (E == 2) ? 0.f : 6.f;             // P = 2^(x - m + SIGMA) <= 2^(TAU+SIGMA)

  static_assert(STAGE0 % 1024 == 0 && STAGE_BYTES % 1024 == 0 && P_OFF % 1024 == 0, "alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// barrier indices
template <int NS>
struct Bar {
  static constexpr int Q_FULL = 0;
  static constexpr int K_FULL = 1;            // + stage
  static constexpr int K_EMPTY = 1 + NS;      // + stage
  static constexpr int S_FULL = 1 + 2 * NS;   // + buffer (2)
  static constexpr int S_EMPTY = 3 + 2 * NS;  // + buffer (2)
  static constexpr int SX_FULL = 5 + 2 * NS;
  static constexpr int SX_EMPTY = 6 + 2 * NS;
  static constexpr int P_READY = 7 + 2 * NS;
  static constexpr int P_FULL = 8 + 2 * NS;
  static constexpr int P_EMPTY = 9 + 2 * NS;
  static constexpr int O_DONE = 10 + 2 * NS;
  static constexpr int FIN_FULL = 11 + 2 * NS;
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;      // O: columns [0, 256)
constexpr uint32_t kSCol = 256;    // S buffers: [256, 320) and [320, 384)

struct TcParams {
  CUtensorMap tm_q_main, tm_q_rope, tm_kv_main, tm_kv_rope;
  DecodeArgs a;
};

// P for 32 keys of a row, packed for the tensor core, plus two sums: the
// exact fp32 sum of the weights (for the LSE) and the sum of the weights as
// rounded into the MMA operand (for normalising O, so the weights that
// multiply V sum to one).
// 16-bit: 16 words of bf16 / fp16 pairs in w[0..15].
// FP8: P = 2^(x - m + SIGMA) as a sum of two E4M3 terms, hi = e4m3(P) in
// w[0..7] and lo = e4m3(P - hi) in w[8..15] (about 8 significant bits).
template <int DT>
__device__ __forceinline__ void pack_p(const float (&x)[32], float m_use, uint32_t (&w)[16], float& sum_q,
                                       float& sum_e) {
  float sq = 0.f, se = 0.f;
  if constexpr (DT == MLA_BF16 || DT == MLA_FP16) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p0 = exp2f(x[2 * i] - m_use), p1 = exp2f(x[2 * i + 1] - m_use);
      se += p0 + p1;
      float2 f;
      if constexpr (DT == MLA_BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
        f = __bfloat1622float2(h);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
      } else {
        __half2 h = __floats2half2_rn(p0, p1);
        f = __half22float2(h);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
      }
      sq += f.x + f.y;
    }
  } else {
    constexpr float SIGMA = Cfg<MLA_FP8_E4M3>::SIGMA;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t hi = 0, lo = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float p0 = exp2f(x[4 * i + 2 * k] - m_use + SIGMA);
        const float p1 = exp2f(x[4 * i + 2 * k + 1] - m_use + SIGMA);
        se += p0 + p1;
        const __nv_fp8x2_storage_t qh = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
        __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(qh, __NV_E4M3);
        const float2 fh = __half22float2(*reinterpret_cast<__half2*>(&hr));
        const __nv_fp8x2_storage_t ql =
            __nv_cvt_float2_to_fp8x2(make_float2(p0 - fh.x, p1 - fh.y), __NV_SATFINITE, __NV_E4M3);
        __half2_raw lr = __nv_cvt_fp8x2_to_halfraw2(ql, __NV_E4M3);
        const float2 fl = __half22float2(*reinterpret_cast<__half2*>(&lr));
        sq += (fh.x + fl.x) + (fh.y + fl.y);
        hi |= (uint32_t)qh << (16 * k);
        lo |= (uint32_t)ql << (16 * k);
      }
      w[i] = hi;
      w[8 + i] = lo;
    }
  }
  sum_q = sq;
  sum_e = se;
}

template <int DT>
__global__ void __launch_bounds__(192, 1) tc_partial_kernel(const __grid_constant__ TcParams prm) {
  using C = Cfg<DT>;
  using B = Bar<C::NS>;
  const DecodeArgs& a = prm.a;
  const mla_plan& p = a.plan;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::BAR_OFF + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = cluster_ctarank();
  const uint32_t peer = c ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int G = p.q_groups, S = p.split_kv, T = p.q_len, H = p.num_heads, M = p.rows_per_unit;
  const int g = pair % G;
  const int s = (pair / G) % S;
  const int b = pair / (G * S);
  const int n = effective_seq_len(a, b, c == 0 && s == 0 && g == 0 && threadIdx.x == 0);
  const int key0 = s * p.keys_per_split;
  const int64_t row0 = (int64_t)b * T * H + (int64_t)g * M;

  if (key0 >= n) {
    // No key in this split. With one split the outputs are final here.
    if (S == 1) {
      for (int r = threadIdx.x; r < M; r += blockDim.x) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + (row0 + r) * MLA_D_V + 256 * c);
        for (int i = 0; i < 32; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        if (c == 0 && a.lse) a.lse[row0 + r] = -INFINITY;
      }
    }
    return;  // the peer takes the same branch (same entry)
  }
  const int key1 = min(n, key0 + p.keys_per_split);
  const int n_tiles = (key1 - key0 + kTileKeys - 1) / kTileKeys;
  const int tile0 = key0 / kTileKeys;
  const int32_t* table = a.block_tables + (int64_t)b * a.max_pages_per_seq;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(bar(B::Q_FULL), 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar(B::K_FULL + i), 1);
      mbar_init(bar(B::K_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B::S_FULL + i), 1);
      mbar_init(bar(B::S_EMPTY + i), 4);
    }
    mbar_init(bar(B::SX_FULL), 1);
    mbar_init(bar(B::SX_EMPTY), 4);
    mbar_init(bar(B::P_READY), 4);
    mbar_init(bar(B::P_FULL), 1);
    mbar_init(bar(B::P_EMPTY), 2);
    mbar_init(bar(B::O_DONE), 1);
    mbar_init(bar(B::FIN_FULL), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (M < 128) {
    // Q rows the TMA box does not cover are zero (rows are independent).
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int ci = 0; ci < C::MAIN_CHUNKS; ++ci) {
      uint4* base = reinterpret_cast<uint4*>(smem + C::Q_MAIN + ci * 16384 + M * 128);
      for (int i = threadIdx.x; i < (128 - M) * 8; i += blockDim.x) base[i] = z;
    }
    uint4* rb = reinterpret_cast<uint4*>(smem + C::Q_ROPE + M * C::ROPE_BYTES);
    for (int i = threadIdx.x; i < (128 - M) * C::ROPE_BYTES / 16; i += blockDim.x) rb[i] = z;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any remote access
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
      const uint64_t pol_kv = policy_evict_first();
      mbar_arrive_expect_tx(bar(B::Q_FULL), C::Q_TILE_BYTES_PER_ROW * (uint32_t)M);
      for (int ci = 0; ci < C::MAIN_CHUNKS; ++ci)
        tma_load_2d(sb + C::Q_MAIN + ci * 16384, &prm.tm_q_main, 256 * (int)c + ci * C::CHUNK_ELEMS, (int)row0,
                    bar(B::Q_FULL), pol_q);
      tma_load_2d(sb + C::Q_ROPE, &prm.tm_q_rope, 512 + 32 * (int)c, (int)row0, bar(B::Q_FULL), pol_q);
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % C::NS;
        if (!bounded_wait(bar(B::K_EMPTY + st), ((j / C::NS) & 1) ^ 1, abort_flag, a.status)) break;
        int page = table[tile0 + j];
        if (page < 0 || (int64_t)page >= a.num_pages) page = 0;  // masked by the softmax warps
        const uint32_t stage = sb + C::STAGE0 + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar(B::K_FULL + st), C::STAGE_BYTES);
        for (int ci = 0; ci < C::MAIN_CHUNKS; ++ci)
          tma_load_2d(stage + ci * 8192, &prm.tm_kv_main, 256 * (int)c + ci * C::CHUNK_ELEMS, page * kTileKeys,
                      bar(B::K_FULL + st), pol_kv);
        tma_load_2d(stage + C::STAGE_MAIN, &prm.tm_kv_rope, 512 + 32 * (int)c, page * kTileKeys,
                    bar(B::K_FULL + st), pol_kv);
      }
      drain_loads(bar(B::K_FULL), C::NS, n_tiles);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idq = instr_desc(C::FMT, C::FMT, 0, 128, 64);
      constexpr uint32_t idp = instr_desc(C::FMT, C::FMT, 1, 128, 256);
      bool ok = bounded_wait(bar(B::Q_FULL), 0, abort_flag, a.status);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % C::NS, buf = j & 1;
        if (!bounded_wait(bar(B::K_FULL + st), (j / C::NS) & 1, abort_flag, a.status)) return false;
        if (!bounded_wait(bar(B::S_EMPTY + buf), ((j >> 1) & 1) ^ 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + 64u * buf;
        const uint32_t stage = sb + C::STAGE0 + st * C::STAGE_BYTES;
        uint32_t acc = 0;
#pragma unroll
        for (int ci = 0; ci < C::MAIN_CHUNKS; ++ci) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = smem_desc(sb + C::Q_MAIN + ci * 16384 + kk * 32, 16, 1024, kSw128);
            const uint64_t db = smem_desc(stage + ci * 8192 + kk * 32, 16, 1024, kSw128);
            if (C::E == 2) mma_f16(d, da, db, idq, acc); else mma_f8(d, da, db, idq, acc);
            acc = 1;
          }
        }
#pragma unroll
        for (int kk = 0; kk < C::ROPE_BYTES / 32; ++kk) {
          const uint64_t da = smem_desc(sb + C::Q_ROPE + kk * 32, 16, 8 * C::ROPE_BYTES, C::ROPE_SW);
          const uint64_t db = smem_desc(stage + C::STAGE_MAIN + kk * 32, 16, 8 * C::ROPE_BYTES, C::ROPE_SW);
          if (C::E == 2) mma_f16(d, da, db, idq, 1); else mma_f8(d, da, db, idq, 1);
        }
        mma_commit(bar(B::S_FULL + buf));
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && n_tiles > 1) ok = issue_qk(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        mbar_arrive_expect_tx(bar(B::P_FULL), C::P_PEER_BYTES);
        if (!bounded_wait(bar(B::P_READY), j & 1, abort_flag, a.status)) break;
        if (!bounded_wait(bar(B::P_FULL), j & 1, abort_flag, a.status)) break;
        tc_fence_after();
        const int st = j % C::NS;
        const uint32_t stage = sb + C::STAGE0 + st * C::STAGE_BYTES;
#pragma unroll
        for (int pl = 0; pl < C::P_PLANES; ++pl) {
#pragma unroll
          for (int kk = 0; kk < 64 / C::MMA_K; ++kk) {
            const uint64_t da = smem_desc(sb + C::P_OFF + pl * C::P_PLANE + kk * 32, 16, 8 * C::P_ROW, C::P_SW);
            const uint64_t db = smem_desc(stage + kk * C::MMA_K * 128, 8192, 1024, kSw128);
            const uint32_t acc = (j > 0 || pl > 0 || kk > 0) ? 1u : 0u;
            if (C::E == 2) mma_f16(tmem + kOCol, da, db, idp, acc); else mma_f8(tmem + kOCol, da, db, idp, acc);
          }
        }
        mma_commit(bar(B::K_EMPTY + st));
        mma_commit_multicast(bar(B::P_EMPTY), 0x3);
        mma_commit(bar(B::O_DONE));
        if (j + 2 < n_tiles) ok = issue_qk(j + 2);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const bool owner = ((lane >> 4) == (int)c);
    const int R = 32 * q + 16 * (int)c + (lane & 15);  // own row this thread works on
    const int h = owner ? 0 : 1;                       // its 32-key half
    const int lane_row = 32 * q + lane;                // its TMEM lane
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int own_idx = 16 * q + (lane & 15);          // row R in the 64-row exchange buffer
    const int limit = (R < M) ? n - T + g * p.fold + R / H : n - 1;
    const uint32_t sx_peer = mapa(sb + C::SX_OFF, peer);
    const uint32_t sx_full_peer = mapa(bar(B::SX_FULL), peer);
    const uint32_t sx_empty_peer = mapa(bar(B::SX_EMPTY), peer);
    const uint32_t p_peer = mapa(sb + C::P_OFF, peer);
    const uint32_t alpha_peer = mapa(sb + C::ALPHA_OFF, peer);
    const uint32_t p_full_peer = mapa(bar(B::P_FULL), peer);
    const uint32_t fin_peer = mapa(sb + C::FIN_OFF, peer);
    const uint32_t fin_full_peer = mapa(bar(B::FIN_FULL), peer);
    float* alpha_s = reinterpret_cast<float*>(smem + C::ALPHA_OFF);
    float* fin_s = reinterpret_cast<float*>(smem + C::FIN_OFF);
    const float sl2 = a.score_scale_log2;
    float m_ref = -INFINITY, lacc = 0.f, lexact = 0.f;
    bool ok = true;

    for (int j = 0; j < n_tiles; ++j) {
      const int buf = j & 1;
      if (!(ok = warp_wait(bar(B::S_FULL + buf), (j >> 1) & 1, abort_flag, a.status))) break;
      tc_fence_after();
      uint32_t v[64];
      {
        uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
        uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
        tmem_ld32(tmem + tl + kSCol + 64u * buf, v0);
        tmem_ld32(tmem + tl + kSCol + 64u * buf + 32u, v1);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B::S_EMPTY + buf));

      // helper lanes hold the partial of a row the peer owns: send it over
      if (!(ok = warp_wait(bar(B::SX_EMPTY), (j & 1) ^ 1, abort_flag, a.status))) break;
      if (!owner) {
        const uint32_t dst = sx_peer + (uint32_t)(16 * q + (lane & 15)) * C::SX_ROW;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          st_async_v4(dst + 16u * u, v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3], sx_full_peer);
      }
      // the owner passes keys 32..63 of its row to its helper
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t x = __shfl_xor_sync(0xffffffffu, v[32 + i], 16);
        if (!owner) v[i] = x;
      }
      if (warp == 2 && lane == 0) mbar_arrive_expect_tx(bar(B::SX_FULL), 64 * 64 * 4);
      if (!(ok = warp_wait(bar(B::SX_FULL), j & 1, abort_flag, a.status))) break;
      float x[32];
      {
        const float4* px = reinterpret_cast<const float4*>(smem + C::SX_OFF + own_idx * C::SX_ROW + h * 128);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 f = px[u];
          x[4 * u + 0] = (__uint_as_float(v[4 * u + 0]) + f.x) * sl2;
          x[4 * u + 1] = (__uint_as_float(v[4 * u + 1]) + f.y) * sl2;
          x[4 * u + 2] = (__uint_as_float(v[4 * u + 2]) + f.z) * sl2;
          x[4 * u + 3] = (__uint_as_float(v[4 * u + 3]) + f.w) * sl2;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(sx_empty_peer);

      // mask: causal limit of the row, end of sequence, invalid pages
      const int pg = table[tile0 + j];
      const bool page_ok = pg >= 0 && (int64_t)pg < a.num_pages;
      if (!page_ok && lane == 0 && q == 0) atomicOr(a.status, MLA_DEV_BAD_PAGE);
      const int kb = key0 + kTileKeys * j + 32 * h;
      float mloc = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (!page_ok || kb + i > limit) x[i] = -INFINITY;
        mloc = fmaxf(mloc, x[i]);
      }
      const float mt = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));
      float alpha = 1.f;
      if (mt > m_ref + C::TAU) {
        alpha = exp2f(m_ref - mt);
        m_ref = mt;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t w[16];
      float psum, pexact;
      pack_p<DT>(x, m_use, w, psum, pexact);
      lacc = fmaf(lacc, alpha, psum);
      lexact = fmaf(lexact, alpha, pexact);

      // P buffer is free once both CTAs finished the previous P.V
      if (j > 0 && !(ok = warp_wait(bar(B::P_EMPTY), (j - 1) & 1, abort_flag, a.status))) break;
      if constexpr (C::E == 2) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int phys = (4 * h + u) ^ (R & 7);
          *reinterpret_cast<uint4*>(smem + C::P_OFF + R * C::P_ROW + phys * 16) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      } else {
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int phys = (2 * h + u) ^ ((R >> 1) & 3);
            *reinterpret_cast<uint4*>(smem + C::P_OFF + pl * C::P_PLANE + R * C::P_ROW + phys * 16) =
                make_uint4(w[8 * pl + 4 * u], w[8 * pl + 4 * u + 1], w[8 * pl + 4 * u + 2], w[8 * pl + 4 * u + 3]);
          }
        }
      }
      if (owner) alpha_s[R] = alpha;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t r0 = (uint32_t)(32 * q + 16 * (int)c);
#pragma unroll
        for (int pl = 0; pl < C::P_PLANES; ++pl)
          bulk_copy_to_peer(p_peer + pl * C::P_PLANE + r0 * C::P_ROW, sb + C::P_OFF + pl * C::P_PLANE + r0 * C::P_ROW,
                            16 * C::P_ROW, p_full_peer);
        bulk_copy_to_peer(alpha_peer + r0 * 4, sb + C::ALPHA_OFF + r0 * 4, 64, p_full_peer);
      }
      // rescale this lane's half-row of O if its reference maximum moved
      float my_alpha = alpha;
      if (!(ok = warp_wait(bar(B::P_FULL), j & 1, abort_flag, a.status))) break;
      if (!owner) my_alpha = alpha_s[lane_row];
      if (j > 0 && __any_sync(0xffffffffu, my_alpha != 1.f)) {
        if (!(ok = warp_wait(bar(B::O_DONE), (j - 1) & 1, abort_flag, a.status))) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + kOCol + 32u * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * my_alpha);
          tmem_st32(tmem + tl + kOCol + 32u * cc, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B::P_READY));
    }

    // ------------------------------------------------------------ epilogue
    if (ok) {
      const float l_row = lacc + __shfl_xor_sync(0xffffffffu, lacc, 16);
      const float l_ex = lexact + __shfl_xor_sync(0xffffffffu, lexact, 16);
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      float lse_val = -INFINITY;
      if (owner) {
        fin_s[R] = (l_row > 0.f) ? a.v_scale / l_row : 0.f;
        if (l_ex > 0.f) lse_val = (m_use - C::SIGMA + log2f(l_ex)) * kLn2;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t r0 = (uint32_t)(32 * q + 16 * (int)c);
        bulk_copy_to_peer(fin_peer + r0 * 4, sb + C::FIN_OFF + r0 * 4, 64, fin_full_peer);
      }
      if (warp == 2 && lane == 0) mbar_arrive_expect_tx(bar(B::FIN_FULL), 256);
      ok = warp_wait(bar(B::FIN_FULL), 0, abort_flag, a.status);
      if (ok) ok = warp_wait(bar(B::O_DONE), (n_tiles - 1) & 1, abort_flag, a.status);
      if (ok) {
        tc_fence_after();
        const float inv = fin_s[lane_row];
        const bool live = lane_row < M;
        const int64_t rg = row0 + lane_row;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + kOCol + 32u * cc, o);
          tmem_wait_ld();
          if (!live) continue;
          if (S == 1) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + rg * MLA_D_V +
                                                  256 * c + 32 * cc);
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
            float4* dst = reinterpret_cast<float4*>(a.o_part + (rg * S + s) * MLA_D_V + 256 * c + 32 * cc);
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
        if (owner && R < M) {
          if (S == 1) {
            if (a.lse) a.lse[row0 + R] = lse_val;
          } else {
            a.lse_part[(row0 + R) * S + s] = lse_val;
          }
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
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();
}

template <int DT>
cudaError_t launch_dt(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<DT>;
  TcParams prm;
  prm.a = a;
  const mla_plan& p = a.plan;
  const uint64_t q_rows = (uint64_t)p.batch * p.q_len * p.num_heads;
  const uint64_t kv_rows = (uint64_t)a.num_pages * kTileKeys;
  const CUtensorMapSwizzle rope_sw = C::E == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!encode_rows_576(&prm.tm_q_main, a.q, C::E, q_rows, C::CHUNK_ELEMS, p.rows_per_unit, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_q_rope, a.q, C::E, q_rows, 32, p.rows_per_unit, rope_sw) ||
      !encode_rows_576(&prm.tm_kv_main, a.kv_cache, C::E, kv_rows, C::CHUNK_ELEMS, kTileKeys,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows_576(&prm.tm_kv_rope, a.kv_cache, C::E, kv_rows, 32, kTileKeys, rope_sw))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_max_dynamic_smem((const void*)tc_partial_kernel<DT>, (int)C::SMEM_BYTES, smem_set);
      e != cudaSuccess)
    return e;
  const uint64_t pairs = (uint64_t)p.batch * p.q_groups * p.split_kv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_partial_kernel<DT>, prm);
}

}  // namespace

cudaError_t launch_tc_partial(const DecodeArgs& a, cudaStream_t stream) {
  if ((uint64_t)a.plan.batch * a.plan.q_groups * a.plan.split_kv == 0) return cudaSuccess;
  switch (a.plan.dtype) {
    case MLA_BF16: return launch_dt<MLA_BF16>(a, stream);
    case MLA_FP16: return launch_dt<MLA_FP16>(a, stream);
    default: return cudaErrorInvalidValue;  // FP8 has its own kernel
  }
}

}  // namespace mla
