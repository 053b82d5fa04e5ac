// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "mla_decode.h"

// 1 in the bounds-checking build (libmla_decode_check.so), 0 otherwise.
#ifndef MLA_BOUNDS_CHECK
#define MLA_BOUNDS_CHECK 0
#endif

namespace mla {

constexpr uint32_t kPlanMagic = 0x4d4c4131u;  // "MLA1"
constexpr int kNumSMs = 148;                    // B200
constexpr int kHeaderBytes = 256;               // workspace header (status word at offset 0)
constexpr int kTileKeys = 64;                   // keys per tile = one cache page
constexpr int kPairTileKeys = 128;              // keys per CTA-pair tile (one page per CTA)
constexpr int kMaxBalancedUnits = 16384;        // decode units (entry x query group) the balanced schedule takes
constexpr int kMaxVarlenUnits = 1 << 16;        // units of a ragged-query (prefill) plan

// Balanced schedule table at the end of the workspace: int32 weighted start
// of every schedule slot (U + 1 entries, the last = W, the total weight; slot
// s holds unit sched_unit(s), see pair_schedule.cuh), then the number of pairs
// that have work. Written by the partial kernel, read by the combine.
// Balanced schedule: per-unit counts of finished partial pieces, then the
// unit table's ready flag; right after the status header, and cleared with it
// before every launch of the partial kernel.
constexpr int kPieceArrivals = 16;  // softmax warps of a CTA pair: counter arrivals per partial piece
inline uint64_t balanced_counter_bytes(int64_t units) {
  return ((uint64_t)(units + 1) * 4 + 255) & ~uint64_t(255);
}
inline uint64_t balanced_table_bytes(int64_t units) {
  return ((uint64_t)(units + 2) * 4 + 255) & ~uint64_t(255);
}
// FP8 rows that see fewer keys than this send P as two E4M3 terms (the P.V
// MMAs run twice); the balanced schedule weighs such tiles 3 against 2.
// Measured with one E4M3 term on N(0,1) inputs, the output's relative L2
// error is 2.3e-2 at 256 keys, 1.3e-2 at 4096, 1.0e-2 at 8192 and 7.7e-3 at
// 16384 (the bound is 3e-2), and the worst element uses 1.04, 0.26, 0.20 and
// 0.15 of its tolerance; with two terms both stay at 1.7e-3 and 0.11.
constexpr int kTwoTermKeys = 8192;
// A piece transition (a pair moving on to a new unit) costs about as much as
// 8 to 12 pair tiles: the cut piece's epilogue, the drain of its last MMAs
// before the next unit's query block can be loaded, and the refill. Measured
// on the 80K-key FP8 batch of 16 entries, pairs whose range crosses an entry
// boundary finished 8.3 us (~8 tiles) after the others; with a lead-in of 16
// they still finished 5 us later, and 24 was the fastest of 8, 16, 24 and 32
// on the 4-entry batch (74.1 against 76.1 us) and within 1% elsewhere. The balanced schedule therefore charges
// every unit with tiles a lead-in of this weight (a tile weighs 2 or 3) at its
// weighted start, ahead of its first tile, so that a pair whose range holds a
// unit start takes correspondingly fewer tiles. The first unit carries one
// too: with the group-major order of pair_schedule.cuh, the halves of the
// sequence then have equal weight and the pairs that read the same pages for
// the two query groups of an entry stay aligned.
constexpr int kPieceLeadWeight = 24;
__host__ __device__ inline int unit_lead_weight(int tiles) { return tiles > 0 ? kPieceLeadWeight : 0; }
// Piece lists too long for a CTA's shared memory go to a spill area right
// before the unit table: per CTA rank, U + P pieces of 3 int32 (a pair's
// pieces are the units its range meets, consecutive in the schedule's
// sequence; pair p's list starts at entry first_slot(p) + p, so the lists of
// consecutive pairs never overlap).
inline uint64_t balanced_spill_bytes(int64_t units, int pairs) {
  return ((uint64_t)2 * (units + pairs) * 12 + 255) & ~uint64_t(255);
}

// Everything a launch needs, validated by the ABI layer.
struct DecodeArgs {
  mla_plan plan;
  const void* q;
  const void* kv_cache;
  int64_t num_pages;
  const int32_t* block_tables;
  int max_pages_per_seq;
  const int32_t* seq_lens;
  float score_scale_log2;  // softmax_scale * q_scale * kv_scale * log2(e)
  float v_scale;           // kv_scale (FP8) or 1
  void* out;               // bf16 [B*T*H, 512]
  float* lse;              // fp32 [B*T*H] or null
  int32_t* status;         // device status word
  float* o_part;           // fp32 [B*T*H, S, 512] (split_kv > 1)
  float* lse_part;         // fp32 [B*T*H, S]       (split_kv > 1)
  int32_t* sched;          // balanced schedule table (MLA_SCHEDULE_BALANCED), else null
  int32_t* unit_done;      // balanced: [U] finished-piece counts, [U] table-ready flag; else null
  int32_t* pieces;         // balanced: piece-list spill area; else null
  const int32_t* cu_q;     // ragged queries: [B + 1] token offsets of the entries; decode: null
  int64_t total_q;         // query tokens in q (B * q_len for decode)
};

// Pair of the balanced schedule whose range holds pair tile x (0 <= x < W):
// pair p covers [floor(W p / np), floor(W (p + 1) / np)).
__host__ __device__ inline int balanced_pair_of(int64_t x, int64_t W, int np) {
  return (int)(((x + 1) * np + W - 1) / W) - 1;
}
__host__ __device__ inline int64_t balanced_lo(int p, int64_t W, int np) { return W * p / np; }

// Records `e` as this thread's last CUDA error (read by mla_last_cuda_error)
// and returns MLA_ERR_CUDA.
int cuda_failure(cudaError_t e);

// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device, once per device: the attribute belongs to each device's context, so
// a process that drives several GPUs needs it on every one. `done` is the
// caller's per-kernel bitmask of devices already set (devices >= 64 are set
// on every call).
cudaError_t set_max_dynamic_smem(const void* func, int bytes, std::atomic<uint64_t>& done);

int plan_impl(int batch, int q_len, int num_heads, int max_seq_len, int dtype, int split_kv,
              int fold, int kernel, int varlen, mla_plan* plan);

cudaError_t launch_simt_partial(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_tc_partial(const DecodeArgs& a, cudaStream_t stream);      // 16-bit inputs
cudaError_t launch_tc_fp8_partial(const DecodeArgs& a, cudaStream_t stream);  // FP8, per-CTA MMAs
cudaError_t launch_tc_fp8_pair_partial(const DecodeArgs& a, cudaStream_t stream);  // FP8, CTA-pair MMAs
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_tc16_pair_partial(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_kv_pack(const void* latent, const void* rope, int64_t n, const int64_t* slots, void* cache,
                           int64_t num_slots, int in_dtype, int cache_dtype, float kv_scale, int32_t* status,
                           cudaStream_t stream);
cudaError_t launch_kv_amax(const void* latent, const void* rope, int64_t n, int in_dtype, float* amax,
                           cudaStream_t stream);
cudaError_t launch_combine_balanced(const DecodeArgs& a, cudaStream_t stream);
// Zeroes `bytes` (a multiple of 16) at the 16-byte aligned `ws`, as a
// programmatic dependent of the previous kernel in the stream (see combine.cu).
cudaError_t launch_workspace_clear(void* ws, uint64_t bytes, cudaStream_t stream);

}  // namespace mla
