// Fused K/V pack + FP8 quantise: the step that writes new tokens into the
// paged latent cache the decode kernels read.
//
// tokenspeed-mla package card, "What it is and what it does": one fused
// kernel packs K/V and quantises to FP8 in place of separate cat and cast
// operations. TokenSpeed MLA article (最快MLA内核背后的秘密), section 一 (its
// kernel table: mla_kv_pack_quantize_fp8) and section 六 (the 576-wide cache
// row: 512 latent dims, then 64 rope dims).
//
// Token i's row [latent_i || rope_i] goes to cache row slot_mapping[i]
// (page * page_size + offset; a negative slot skips the token). With an FP8
// cache every element is E4M3(x / kv_scale): the quotient in fp32 (IEEE
// division, rounded to nearest), then cvt.rn.satfinite (nearest even,
// saturating to +-448, NaN kept). With a 16-bit cache of the inputs' type the
// row is a copy.
//
// One thread per 16-byte chunk of an output row: 36 chunks per FP8 row (32
// latent, 4 rope), 72 per 16-bit row; consecutive threads write consecutive
// chunks of a row and read consecutive 32-byte (or 16-byte) pieces of the
// input. HBM-bound: n * 1152 bytes read, n * 576 (FP8) written.
//
// The FP8 code of an element depends only on its 16 input bits (kv_scale is
// one value per call), so large calls first encode the 32768 non-negative bit
// patterns into a table in each CTA's shared memory, with the same division
// and conversion as the direct path, and then look every element up: the IEEE
// divisions, 16 per output chunk, otherwise bind the kernel to the ALU.
// Small calls (a decode step's few tokens) keep the direct path, whose CTAs
// do not pay for the table.
#include <atomic>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

__device__ __forceinline__ float bits_to_float(uint16_t h, bool bf16) {
  return bf16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

__global__ void __launch_bounds__(256) kv_pack_fp8_kernel(const uint16_t* __restrict__ latent,
                                                          const uint16_t* __restrict__ rope, int64_t n,
                                                          const int64_t* __restrict__ slots, int64_t num_slots,
                                                          float kv_scale, bool bf16, uint8_t* __restrict__ cache,
                                                          int32_t* status) {
  const int64_t total = n * 36;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / 36;
    const int c = (int)(idx - i * 36);
    const int64_t s = slots[i];
    if (s < 0) continue;
    if (s >= num_slots) {
      if (status) atomicOr(status, MLA_DEV_BAD_PAGE);
      continue;
    }
    const uint16_t* src = c < 32 ? latent + i * 512 + c * 16 : rope + i * 64 + (c - 32) * 16;
    const uint4 r0 = *reinterpret_cast<const uint4*>(src);
    const uint4 r1 = *reinterpret_cast<const uint4*>(src + 8);
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t b[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t word = w[2 * k + h];
        const float x0 = __fdiv_rn(bits_to_float((uint16_t)(word & 0xffffu), bf16), kv_scale);
        const float x1 = __fdiv_rn(bits_to_float((uint16_t)(word >> 16), bf16), kv_scale);
        b[h] = ptx::cvt_e4m3x2(x0, x1);  // x0 in the low byte
      }
      out[k] = b[0] | (b[1] << 16);
    }
    *reinterpret_cast<uint4*>(cache + s * 576 + c * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// FP8 codes of the 32768 non-negative 16-bit input patterns for this call's
// scale (x0 of each pair in the low byte, as the direct path packs them). A
// negative input's code is its magnitude's with the sign bit set: x / s is
// -(|x| / s) exactly for s > 0, and the conversion is symmetric (a NaN's sign
// is the one thing this changes, and a NaN's sign after division is
// unspecified).
constexpr int kE4m3TableBytes = 32768;
__device__ __forceinline__ void build_e4m3_table(uint8_t* table, float kv_scale, bool bf16) {
  for (int b = threadIdx.x; b < kE4m3TableBytes / 2; b += blockDim.x) {
    const float x0 = __fdiv_rn(bits_to_float((uint16_t)(2 * b), bf16), kv_scale);
    const float x1 = __fdiv_rn(bits_to_float((uint16_t)(2 * b + 1), bf16), kv_scale);
    reinterpret_cast<uint16_t*>(table)[b] = (uint16_t)ptx::cvt_e4m3x2(x0, x1);
  }
}
// codes of the two 16-bit inputs of word w, the low one in the low byte
__device__ __forceinline__ uint32_t table_codes(const uint8_t* table, uint32_t w) {
  return (uint32_t)table[w & 0x7fffu] | ((w >> 8) & 0x80u) | ((uint32_t)table[(w >> 16) & 0x7fffu] << 8) |
         ((w >> 16) & 0x8000u);
}

// Two output chunks a grid stride apart per thread and iteration, their
// input loads issued before the slots are read and before any lookup, so
// that enough bytes are in flight per SM for HBM.
__global__ void __launch_bounds__(256) kv_pack_fp8_table_kernel(const uint16_t* __restrict__ latent,
                                                                const uint16_t* __restrict__ rope, int64_t n,
                                                                const int64_t* __restrict__ slots,
                                                                int64_t num_slots, float kv_scale, bool bf16,
                                                                uint8_t* __restrict__ cache, int32_t* status) {
  extern __shared__ uint8_t table[];
  build_e4m3_table(table, kv_scale, bf16);
  __syncthreads();
  const int64_t total = n * 36;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += 2 * stride) {
    uint4 r[2][2];
    int64_t tok[2];
    int ch[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t id = idx + u * stride;
      tok[u] = id < total ? id / 36 : -1;
      ch[u] = tok[u] >= 0 ? (int)(id - tok[u] * 36) : 0;
      if (tok[u] >= 0) {
        const uint16_t* src = ch[u] < 32 ? latent + tok[u] * 512 + ch[u] * 16 : rope + tok[u] * 64 + (ch[u] - 32) * 16;
        r[u][0] = *reinterpret_cast<const uint4*>(src);
        r[u][1] = *reinterpret_cast<const uint4*>(src + 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (tok[u] < 0) continue;
      const int64_t s = slots[tok[u]];
      if (s < 0) continue;
      if (s >= num_slots) {
        if (status) atomicOr(status, MLA_DEV_BAD_PAGE);
        continue;
      }
      const uint32_t w[8] = {r[u][0].x, r[u][0].y, r[u][0].z, r[u][0].w, r[u][1].x, r[u][1].y, r[u][1].z, r[u][1].w};
      uint32_t out[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) out[k] = table_codes(table, w[2 * k]) | (table_codes(table, w[2 * k + 1]) << 16);
      *reinterpret_cast<uint4*>(cache + s * 576 + ch[u] * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

__global__ void __launch_bounds__(256) kv_pack_copy_kernel(const uint16_t* __restrict__ latent,
                                                           const uint16_t* __restrict__ rope, int64_t n,
                                                           const int64_t* __restrict__ slots, int64_t num_slots,
                                                           uint16_t* __restrict__ cache, int32_t* status) {
  const int64_t total = n * 72;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / 72;
    const int c = (int)(idx - i * 72);
    const int64_t s = slots[i];
    if (s < 0) continue;
    if (s >= num_slots) {
      if (status) atomicOr(status, MLA_DEV_BAD_PAGE);
      continue;
    }
    const uint16_t* src = c < 64 ? latent + i * 512 + c * 8 : rope + i * 64 + (c - 64) * 8;
    *reinterpret_cast<uint4*>(cache + s * 576 + c * 8) = *reinterpret_cast<const uint4*>(src);
  }
}

// Largest |x| over the non-NaN elements (fmaxf drops NaN): per-thread maxima,
// a warp and block reduction, then one atomicMax on the float's bits (valid
// for non-negative floats) per block into a zeroed result.
__global__ void __launch_bounds__(256) kv_amax_kernel(const uint16_t* __restrict__ latent,
                                                      const uint16_t* __restrict__ rope, int64_t n, bool bf16,
                                                      unsigned int* amax_bits) {
  float m = 0.f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n * 64; j += stride) {
    // 8 latent elements and 1 rope element per step
    const uint4 v = *reinterpret_cast<const uint4*>(latent + j * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = fmaxf(m, fabsf(bits_to_float((uint16_t)(w[k] & 0xffffu), bf16)));
      m = fmaxf(m, fabsf(bits_to_float((uint16_t)(w[k] >> 16), bf16)));
    }
    m = fmaxf(m, fabsf(bits_to_float(rope[j], bf16)));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b = fmaxf(b, wm[i]);
    atomicMax(amax_bits, __float_as_uint(b));
  }
}

int grid_for(int64_t work) {
  const int64_t blocks = (work + 255) / 256;
  const int64_t cap = 148 * 8;  // a few resident blocks per SM, grid-stride beyond
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_kv_pack(const void* latent, const void* rope, int64_t n, const int64_t* slots,
                           void* cache, int64_t num_slots, int in_dtype, int cache_dtype, float kv_scale,
                           int32_t* status, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const auto* l = static_cast<const uint16_t*>(latent);
  const auto* r = static_cast<const uint16_t*>(rope);
  if (cache_dtype == MLA_FP8_E4M3) {
    // the table path from 8 output chunks per thread of its grid (six CTAs an
    // SM) on: the table's 32768 divisions per CTA are then a small share of
    // the call's
    if (n * 36 >= (int64_t)kNumSMs * 6 * 256 * 8) {
      static std::atomic<uint64_t> smem_set{0};
      if (cudaError_t e = set_max_dynamic_smem((const void*)kv_pack_fp8_table_kernel, kE4m3TableBytes, smem_set);
          e != cudaSuccess)
        return e;
      kv_pack_fp8_table_kernel<<<kNumSMs * 6, 256, kE4m3TableBytes, stream>>>(
          l, r, n, slots, num_slots, kv_scale, in_dtype == MLA_BF16, static_cast<uint8_t*>(cache), status);
      return cudaGetLastError();
    }
    kv_pack_fp8_kernel<<<grid_for(n * 36), 256, 0, stream>>>(l, r, n, slots, num_slots, kv_scale,
                                                             in_dtype == MLA_BF16, static_cast<uint8_t*>(cache),
                                                             status);
  } else {
    kv_pack_copy_kernel<<<grid_for(n * 72), 256, 0, stream>>>(l, r, n, slots, num_slots,
                                                              static_cast<uint16_t*>(cache), status);
  }
  return cudaGetLastError();
}

cudaError_t launch_kv_amax(const void* latent, const void* rope, int64_t n, int in_dtype, float* amax,
                           cudaStream_t stream) {
  if (cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream); e != cudaSuccess) return e;
  if (n == 0) return cudaSuccess;
  kv_amax_kernel<<<grid_for(n * 64), 256, 0, stream>>>(static_cast<const uint16_t*>(latent),
                                                       static_cast<const uint16_t*>(rope), n, in_dtype == MLA_BF16,
                                                       reinterpret_cast<unsigned int*>(amax));
  return cudaGetLastError();
}

}  // namespace mla
