// Split-KV partial kernel on CUDA cores: the simple cross-check kernel.
//
// One CTA per (batch entry, query group, split) -- the first of the two
// kernels of the split-KV decode (TokenSpeed MLA article 最快MLA内核背后的秘密,
// section 二). Each warp walks its rows one at a time over the split's keys:
// lanes split the 576 dims of the dot product, the score is reduced across
// the warp, and an online softmax (log2 domain) keeps the row's running
// maximum, sum and the 512-wide output (16 values per lane). Keys are read
// straight from the paged cache through the block table. It is slow by
// design; the tensor-core kernel is the product path.
#include "device_common.cuh"

namespace mla {
namespace {

template <int DT>
__global__ void __launch_bounds__(256) simt_partial_kernel(const DecodeArgs a) {
  const mla_plan& p = a.plan;
  const int S = p.split_kv, G = p.q_groups, H = p.num_heads;
  int idx = blockIdx.x;
  const int g = idx % G;
  idx /= G;
  const int s = idx % S;
  const int b = idx / S;
  const UnitGeom ug = unit_geom(a, b * G + g, s == 0 && threadIdx.x == 0);
  const int n = ug.n;
  const int key0 = s * p.keys_per_split;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (key0 >= n) {
    // Only split 0 can be empty-and-final: with one split the outputs are
    // written here, so an entry without keys still gets out = 0, lse = -inf.
    // (With several splits the combine kernel writes those rows.)
    if (S == 1) {
      for (int m = warp; m < ug.rows; m += 8) {
        const int64_t row = ug.row0 + m;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V;
        for (int i = lane; i < MLA_D_V; i += 32) out[i] = __float2bfloat16_rn(0.f);
        if (a.lse && lane == 0) a.lse[row] = -INFINITY;
      }
    }
    return;
  }
  const int key1 = min(n, key0 + p.keys_per_split);
  const int32_t* table = a.block_tables + (int64_t)b * a.max_pages_per_seq;

  for (int m = warp; m < ug.rows; m += 8) {
    const int last = ug.nq + m / H;  // causal: keys <= last
    const int64_t row = ug.row0 + m;
    const int jend = min(key1, last + 1);
    float qv[MLA_D_QK / 32];
#pragma unroll
    for (int i = 0; i < MLA_D_QK / 32; ++i) qv[i] = load_elem<DT>(a.q, row * MLA_D_QK + lane + 32 * i);
    float mx = -INFINITY, l = 0.f;
    float o[MLA_D_V / 32];
#pragma unroll
    for (int i = 0; i < MLA_D_V / 32; ++i) o[i] = 0.f;
    for (int j = max(key0, row_key_lo(p, last)); j < jend; ++j) {  // sliding window: the row's last keys
      const int page = table[j / kTileKeys];
      if (page < 0 || (int64_t)page >= a.num_pages) {
        if (lane == 0) atomicOr(a.status, MLA_DEV_BAD_PAGE);
        continue;
      }
      const int64_t base = ((int64_t)page * kTileKeys + (j % kTileKeys)) * MLA_D_QK;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < MLA_D_QK / 32; ++i) dot = fmaf(qv[i], load_elem<DT>(a.kv_cache, base + lane + 32 * i), dot);
      dot = warp_sum(dot);
      const float sc = dot * a.score_scale_log2;
      const float mn = fmaxf(mx, sc);
      const float alpha = exp2f(mx - mn);
      const float pj = exp2f(sc - mn);
      l = fmaf(l, alpha, pj);
#pragma unroll
      for (int i = 0; i < MLA_D_V / 32; ++i)
        o[i] = fmaf(o[i], alpha, pj * load_elem<DT>(a.kv_cache, base + lane + 32 * i));
      mx = mn;
    }
    const float inv = l > 0.f ? a.v_scale / l : 0.f;
    const float lse_v = l > 0.f ? (mx + log2f(l)) * kLn2 : -INFINITY;
    if (S == 1) {
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + row * MLA_D_V;
#pragma unroll
      for (int i = 0; i < MLA_D_V / 32; ++i) out[lane + 32 * i] = __float2bfloat16_rn(o[i] * inv);
      if (a.lse && lane == 0) a.lse[row] = lse_v;
    } else {
      float* op = a.o_part + (row * S + s) * MLA_D_V;
#pragma unroll
      for (int i = 0; i < MLA_D_V / 32; ++i) op[lane + 32 * i] = o[i] * inv;
      if (lane == 0) a.lse_part[row * S + s] = lse_v;
    }
  }
}

}  // namespace

cudaError_t launch_simt_partial(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t grid = (int64_t)a.plan.batch * a.plan.q_groups * a.plan.split_kv;
  if (grid == 0) return cudaSuccess;
  switch (a.plan.dtype) {
    case MLA_BF16: simt_partial_kernel<MLA_BF16><<<(unsigned)grid, 256, 0, stream>>>(a); break;
    case MLA_FP16: simt_partial_kernel<MLA_FP16><<<(unsigned)grid, 256, 0, stream>>>(a); break;
    default: simt_partial_kernel<MLA_FP8_E4M3><<<(unsigned)grid, 256, 0, stream>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace mla
