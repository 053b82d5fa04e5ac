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

namespace mla {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const DecodeArgs a) {
  const mla_plan& p = a.plan;
  const int64_t rows = (int64_t)p.batch * p.q_len * p.num_heads;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int b = (int)(row / ((int64_t)p.q_len * p.num_heads));
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
  const int64_t rows = (int64_t)a.plan.batch * a.plan.q_len * a.plan.num_heads;
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
// the pieces in their slots (pair p: slot 2p if the unit is its first, else
// 2p + 1), as above. One warp per output row.
__global__ void __launch_bounds__(256) combine_balanced_kernel(const DecodeArgs a) {
  const mla_plan& p = a.plan;
  const int64_t rows = (int64_t)p.batch * p.q_len * p.num_heads;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int TH = p.q_len * p.num_heads;
  const int b = (int)(row / TH);
  const int t = (int)(row % TH) / p.num_heads;
  const int h = (int)(row % TH) % p.num_heads;
  const int g = t / p.fold;
  const int r = (t - g * p.fold) * p.num_heads + h;  // row within the unit
  const int U = p.batch * p.q_groups;
  const int u = b * p.q_groups + g;
  const int32_t* tbl = a.sched;
  const int64_t start = tbl[u], end = tbl[u + 1], W = tbl[U];
  const int np = tbl[U + 1];
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V + lane * 16);
  if (end == start) {  // no key at all
    dst[0] = make_uint4(0, 0, 0, 0);
    dst[1] = make_uint4(0, 0, 0, 0);
    if (a.lse && lane == 0) a.lse[row] = -INFINITY;
    return;
  }
  const int p0 = balanced_pair_of(start, W, np), p1 = balanced_pair_of(end - 1, W, np);
  if (p0 == p1) return;  // written by its pair
  const int M = p.rows_per_unit;
  auto slot_of = [&](int q) { return balanced_lo(q, W, np) >= start ? 2 * q : 2 * q + 1; };
  const int npc = p1 - p0 + 1;

  float m = -INFINITY;
  for (int k = lane; k < npc; k += 32) m = fmaxf(m, a.lse_part[(int64_t)slot_of(p0 + k) * M + r]);
  m = warp_max(m);
  float L = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int k = lane; k < npc; k += 32) sum += expf(a.lse_part[(int64_t)slot_of(p0 + k) * M + r] - m);
    sum = warp_sum(sum);
    L = m + logf(sum);
  }
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  if (L != -INFINITY) {
    for (int k = 0; k < npc; ++k) {
      const int64_t sl = slot_of(p0 + k);
      const float ls = a.lse_part[sl * M + r];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - L);
      const float4* src = reinterpret_cast<const float4*>(a.o_part + (sl * M + r) * MLA_D_V + lane * 16);
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
  dst[0] = packed[0];
  dst[1] = packed[1];
  if (a.lse && lane == 0) a.lse[row] = L;
}

}  // namespace

cudaError_t launch_combine_balanced(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.plan.batch * a.plan.q_len * a.plan.num_heads;
  if (rows == 0) return cudaSuccess;
  combine_balanced_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
