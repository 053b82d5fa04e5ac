// Split-KV combine kernel: LSE-weighted merge of the per-split partials.
//
// The second of the two decode kernels (TokenSpeed MLA article
// 最快MLA内核背后的秘密, section 二; the article's reducer avoids per-element
// loads, section 四). One warp per output row (b, t, h):
//   L   = ln sum_s exp(lse_s)          (max-shifted, warp-shuffle reductions)
//   out = sum_s exp(lse_s - L) * O_s   (BF16, round to nearest even)
// Each lane owns 16 consecutive output columns: four 16-byte fp32 loads per
// split and two 16-byte BF16 stores. Splits past the entry's last key were
// never written and are skipped; a split whose lse is -inf (no visible key)
// has weight 0; a row with no visible key at all gets out = 0, lse = -inf.
#include "device_common.cuh"
#include "pair_schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

// Batch entry of packed query token `tok` (ragged queries: the last entry
// whose first token is at most tok), or -1 when no entry holds the token.
__device__ int entry_of_token(const DecodeArgs& a, int64_t tok) {
  const mla_plan& p = a.plan;
  if (!a.cu_q) return (int)(tok / p.q_len);
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.cu_q[mid] <= tok) lo = mid; else hi = mid - 1;
  }
  const EntryQ e = entry_q(a, lo, false);
  return (tok >= e.q0 && tok < e.q0 + e.qlen) ? lo : -1;
}

__global__ void __launch_bounds__(256) combine_kernel(const DecodeArgs a) {
  const mla_plan& p = a.plan;
  const int64_t rows = a.total_q * p.num_heads;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int b = entry_of_token(a, row / p.num_heads);
  if (b < 0) return;  // a packed token outside every entry: no output
  const int n = effective_seq_len(a, b, false);
  const int S = p.split_kv;
  const int ns = min(S, (n + p.keys_per_split - 1) / p.keys_per_split);
  const float* lp = a.lse_part + row * S;

  float m = -INFINITY;
  for (int s = lane; s < ns; s += 32) m = fmaxf(m, lp[s]);
  m = warp_max(m);
  float L = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int s = lane; s < ns; s += 32) sum += expf(lp[s] - m);
    sum = warp_sum(sum);
    L = m + logf(sum);
  }
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  if (L != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float ls = lp[s];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - L);
      const float4* src = reinterpret_cast<const float4*>(a.o_part + (row * S + s) * MLA_D_V + lane * 16);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 x = src[v];
        acc[4 * v + 0] = fmaf(w, x.x, acc[4 * v + 0]);
        acc[4 * v + 1] = fmaf(w, x.y, acc[4 * v + 1]);
        acc[4 * v + 2] = fmaf(w, x.z, acc[4 * v + 2]);
        acc[4 * v + 3] = fmaf(w, x.w, acc[4 * v + 3]);
      }
    }
  }
  uint4 packed[2];
  uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    pw[i] = *reinterpret_cast<uint32_t*>(&h2);
  }
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V + lane * 16);
  dst[0] = packed[0];
  dst[1] = packed[1];
  if (a.lse && lane == 0) a.lse[row] = L;
}

}  // namespace

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t rows = a.total_q * a.plan.num_heads;
  if (rows == 0) return cudaSuccess;
  combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla

namespace mla {
namespace {

// Combine for the balanced CTA-pair schedule. Units a single pair covered
// whole were finished by the partial kernel and are left alone; units with
// no key get out = 0, lse = -inf; a unit cut between pairs p0 .. p1 merges
// the pieces in their slots (pair p0: slot 2p0 + 1; every later pair q:
// slot 2q). Slots are laid out [slot][16-byte column chunk][row]: thread
// (row i, warp w) of a block of 32 rows x 8 warps sums kC4 chunks (4 kC4
// output columns) of row i over the pieces, and the 32 threads of a warp read
// 32 consecutive rows (512 contiguous bytes) per load. The grid holds
// units x row blocks x 16 / kC4 column blocks, so that even a few long units
// that were cut into many pieces spread over the whole GPU. The grid must be
// resident at once while its units finish, so that no block waits for
// another's slot: kC4 = 2 runs at 64 registers a thread (four blocks an SM,
// grids of up to 592 blocks) and merges 3 pieces a batch; plans whose grid at
// kC4 = 1 is at most 296 blocks (few units, each cut into many pieces) take
// kC4 = 1 at up to 128 registers (two blocks an SM) and merge 20 pieces a
// batch, so that the ~20 pieces of a unit spread over all 74 pairs take one
// round of loads.
constexpr int kCombineNarrowResident = 2 * 148;
constexpr uint64_t kUnitWaitNs = 500ull * 1000 * 1000;  // per wait: 0.5 s

// Bounded wait (one thread) for a counter written by the partial kernel;
// sets MLA_DEV_TIMEOUT and returns false when the limit passes.
__device__ bool wait_count(const int32_t* ctr, int target, int32_t* status) {
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::ld_acquire_gpu(ctr) < target) {
    if (ptx::globaltimer() - t0 > kUnitWaitNs) {
      atomicOr(status, MLA_DEV_TIMEOUT);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}

// Merge of one unit's rows [32 rb, 32 rb + 32) x column block cb (block-
// uniform u, so every thread takes the same path through the barriers).
template <int kC4>
__device__ __forceinline__ void combine_unit(const DecodeArgs& a, int u, int rb, int cb, int* s_ok) {
  const mla_plan& p = a.plan;
  const int M = p.rows_per_unit;
  const int U = p.batch * p.q_groups;
  const int32_t* tbl = a.sched;
  const int sl = sched_slot(p, u);  // the unit's position in the schedule's sequence
  if (!in_bounds(a, sl, U)) return;  // block-uniform
  const int64_t start = tbl[sl], end = tbl[sl + 1], W = tbl[U];
  const int np = tbl[U + 1];
  const UnitGeom ug = unit_geom(a, u, false);
  // pairs holding the unit's first and last tiles (tile starts are weighted;
  // the first follows the unit's lead-in)
  const int lead = end > start ? unit_lead_weight(1) : 0;
  const int p0 = end > start ? balanced_pair_of(start + lead, W, np) : 0;
  const int p1 = end > start ? balanced_pair_of(end - tile_weight(p, ug), W, np) : 0;
  if (end > start && p0 == p1) return;  // a whole unit: written by its pair
  // (block-uniform: every thread leaves together)
  if (end > start && !(in_bounds(a, 2 * p0 + 1, balanced_slots(a)) && in_bounds(a, 2 * p1, balanced_slots(a)))) return;
  if (end > start) {
    __syncthreads();  // every thread has read s_ok
    if (threadIdx.x == 0) *s_ok = wait_count(a.unit_done + u, kPieceArrivals * (p1 - p0 + 1), a.status);
    __syncthreads();
    if (!*s_ok) return;
    (void)ptx::ld_acquire_gpu(a.unit_done + u);
  }
  const int r = rb * 32 + (threadIdx.x & 31);       // row within the unit
  const int c4_0 = (cb * 8 + (threadIdx.x >> 5)) * kC4;  // first of this thread's kC4 16-byte chunks
  if (r >= ug.rows) return;  // past the unit's rows (an entry's last group under ragged queries)
  if (!in_bounds(a, ug.row0 + r, out_rows(a)) || !in_bounds(a, r, M)) return;
  const bool lse_writer = a.lse && cb == 0 && (threadIdx.x >> 5) == 0;
  if (end == start) {  // no key at all
    const int64_t row = ug.row0 + r;
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V + c4_0 * 4;
    if constexpr (kC4 == 2)
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    else
      *reinterpret_cast<uint2*>(dst) = make_uint2(0, 0);
    if (lse_writer) a.lse[row] = -INFINITY;
    return;
  }
  // Pair p0's piece begins at the unit's start: slot 2p0 + 1. Every later
  // pair's piece begins inside the unit: slot 2q. Slots number
  // 2 * split_kv <= 148 of M <= MLA_MAX_ROWS rows: float offsets into the
  // partials fit an int.
  auto slot = [&](int q) -> int { return q == p0 ? 2 * p0 + 1 : 2 * q; };

  // One pass over the pieces with a running maximum (the sum and the
  // accumulators are rescaled when it grows). Pieces go in batches of kBatch
  // whose loads are all issued before any of them is used (no branch depends
  // on a loaded value), so their latencies overlap.
  constexpr int kBatch = kC4 == 2 ? 3 : 20;
  constexpr int kAcc = 4 * kC4;
  const float* base = a.o_part + (c4_0 * M + r) * 4;
  const int slot_stride = (MLA_D_V / 4) * M * 4;  // floats per partial slot
  float m = -INFINITY, sum = 0.f;
  float acc[kAcc];
#pragma unroll
  for (int i = 0; i < kAcc; ++i) acc[i] = 0.f;
  for (int q0 = p0; q0 <= p1; q0 += kBatch) {
    float ls[kBatch];
    float4 x0[kBatch], x1[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const bool in = q0 + i <= p1;
      const int sl = slot(in ? q0 + i : p0);
      const float* src = base + sl * slot_stride;
      // past p1: slot p0 is read again and weighs 0 (lse -inf)
      ls[i] = in ? a.lse_part[sl * M + r] : -INFINITY;
      x0[i] = *reinterpret_cast<const float4*>(src);
      if constexpr (kC4 == 2) x1[i] = *reinterpret_cast<const float4*>(src + M * 4);
    }
    float mb = m;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) mb = fmaxf(mb, ls[i]);
    if (mb == -INFINITY) continue;  // every piece so far is empty
    const float sc = m == -INFINITY ? 0.f : expf(m - mb);
    sum *= sc;
#pragma unroll
    for (int e = 0; e < kAcc; ++e) acc[e] *= sc;
    m = mb;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      // an empty piece (lse -inf) has weight 0 and may hold anything
      const bool live = ls[i] != -INFINITY;
      const float w = live ? expf(ls[i] - m) : 0.f;
      sum += w;
      acc[0] = fmaf(w, live ? x0[i].x : 0.f, acc[0]);
      acc[1] = fmaf(w, live ? x0[i].y : 0.f, acc[1]);
      acc[2] = fmaf(w, live ? x0[i].z : 0.f, acc[2]);
      acc[3] = fmaf(w, live ? x0[i].w : 0.f, acc[3]);
      if constexpr (kC4 == 2) {
        acc[4] = fmaf(w, live ? x1[i].x : 0.f, acc[4]);
        acc[5] = fmaf(w, live ? x1[i].y : 0.f, acc[5]);
        acc[6] = fmaf(w, live ? x1[i].z : 0.f, acc[6]);
        acc[7] = fmaf(w, live ? x1[i].w : 0.f, acc[7]);
      }
    }
  }
  const float L = m == -INFINITY ? -INFINITY : m + logf(sum);
  const float inv = m == -INFINITY ? 0.f : 1.f / sum;
#pragma unroll
  for (int i = 0; i < kAcc; ++i) acc[i] *= inv;
  uint32_t pk[kAcc / 2];
#pragma unroll
  for (int e = 0; e < kAcc / 2; ++e) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    pk[e] = *reinterpret_cast<uint32_t*>(&h2);
  }
  const int64_t row = ug.row0 + r;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V + c4_0 * 4;
  if constexpr (kC4 == 2)
    *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  else
    *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
  if (lse_writer) a.lse[row] = L;
}

template <int kC4>
__device__ __forceinline__ void combine_balanced_block(const DecodeArgs& a, int units_per_block);

template <int kC4>
__global__ void __launch_bounds__(256, kC4 == 2 ? 4 : 2) combine_balanced_kernel(const DecodeArgs a, int units_per_block) {
  // The next step's workspace clear may be launched now: it waits for this
  // grid's completion before touching the workspace.
  ptx::launch_dependents();
  combine_balanced_block<kC4>(a, units_per_block);
  // This grid completes only after the partial kernel it depends on: the
  // partial kernel's last writes (the rows of units one pair finished whole)
  // may come after every merge here, and work later in the stream relies on
  // the completion of this grid alone. One block waiting for it is enough (a
  // grid completes when its last block exits); the others leave as soon as
  // their merges are done and make room for the rest of the grid.
  if (blockIdx.x == 0) ptx::grid_dep_wait();
}

template <int kC4>
__device__ __forceinline__ void combine_balanced_block(const DecodeArgs& a, int units_per_block) {
  const mla_plan& p = a.plan;
  const int M = p.rows_per_unit;
  const int U = p.batch * p.q_groups;
  // Launched as the partial kernel's programmatic dependent, this block may
  // start while pairs still run: it waits for the unit table, then, per unit
  // of its share, for every piece of the unit (kPieceArrivals arrivals each).
  // Each thread then acquires the counter itself before reading what it
  // guards. A block takes units_per_block consecutive units (more than one
  // only for large unit counts, e.g. ragged prefill), so that blocks of whole
  // units, which have nothing to merge, do not dominate the grid.
  __shared__ int s_ok;
  if (threadIdx.x == 0) s_ok = wait_count(a.unit_done + U, 1, a.status);
  __syncthreads();
  if (!s_ok) return;
  (void)ptx::ld_acquire_gpu(a.unit_done + U);
  const int nb = (M + 31) / 32;
  constexpr int kColBlocks = 16 / kC4;
  const int cb = blockIdx.x % kColBlocks;
  const int blk = blockIdx.x / kColBlocks;
  const int rb = blk % nb;
  const int u0 = (blk / nb) * units_per_block;
  for (int u = u0; u < U && u < u0 + units_per_block; ++u) {
    combine_unit<kC4>(a, u, rb, cb, &s_ok);
    __syncthreads();
    if (!s_ok) return;  // a wait gave up (the same in every thread)
  }
}

}  // namespace

// Clears the status word, the unit counters and the table's ready flag of a
// balanced-schedule workspace before the partial kernel runs. Launched as a
// programmatic dependent of the previous kernel in the stream (normally the
// previous step's combine, which reads these counters): it lets the partial
// kernel start its set-up at once and waits for that kernel before writing.
__global__ void __launch_bounds__(256) workspace_clear_kernel(uint4* ws, int64_t n16) {
  ptx::launch_dependents();
  ptx::grid_dep_wait();
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n16; i += (int64_t)gridDim.x * 256)
    ws[i] = make_uint4(0, 0, 0, 0);
}

cudaError_t launch_workspace_clear(void* ws, uint64_t bytes, cudaStream_t stream) {
  const int64_t n16 = (int64_t)(bytes / 16);
  const int64_t blocks = (n16 + 255) / 256;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(blocks < 148 ? (blocks > 0 ? blocks : 1) : 148));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, workspace_clear_kernel, reinterpret_cast<uint4*>(ws), n16);
}

cudaError_t launch_combine_balanced(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t units = (int64_t)a.plan.batch * a.plan.q_groups;
  if (units == 0) return cudaSuccess;
  const int nb = (a.plan.rows_per_unit + 31) / 32;
  // programmatic dependent of the partial kernel: blocks take the SMs of
  // pairs that are done and wait for their own unit (the partial kernel
  // never waits for this grid)
  // about 4096 unit blocks at most: beyond that a block takes several units
  const int64_t per = (units + 4095) / 4096;
  const int64_t unit_blocks = (units + per - 1) / per;
  // one chunk per thread when that grid is still resident at once
  const bool narrow = unit_blocks * nb * 16 <= kCombineNarrowResident;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(unit_blocks * nb * (narrow ? 16 : 8)));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return narrow ? cudaLaunchKernelEx(&cfg, combine_balanced_kernel<1>, a, (int)per)
                : cudaLaunchKernelEx(&cfg, combine_balanced_kernel<2>, a, (int)per);
}

}  // namespace mla
