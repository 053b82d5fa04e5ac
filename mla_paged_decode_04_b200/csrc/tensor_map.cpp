// Tensor-map encoding for the TMA loads (driver entry point fetched at run
// time, so the library does not link libcuda).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "mla_decode.h"

namespace mla {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}
}  // namespace

bool encode_rows_576(CUtensorMap* m, const void* base, int esize, uint64_t rows, uint32_t box_x, uint32_t box_y,
                     CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {MLA_D_QK, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)MLA_D_QK * esize};
  const cuuint32_t box[2] = {box_x, box_y};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A 3-D view of a [rows, 576] array of esize-byte elements: (element within
// a 128-byte column chunk, row, chunk), chunks `chunk_stride` bytes apart
// from `base`. A box of (128 / esize, box_rows, box_chunks) lands as
// box_chunks SW128 tiles of box_rows x 128 bytes one after the other: several
// column chunks of a page in one TMA instruction.
bool encode_rows_576_chunks(CUtensorMap* m, const void* base, int esize, uint64_t rows, uint32_t nchunks,
                            uint64_t chunk_stride, uint32_t box_rows, uint32_t box_chunks) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)(128 / esize), rows, nchunks};
  const cuuint64_t strides[2] = {(cuuint64_t)MLA_D_QK * esize, chunk_stride};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / esize), box_rows, box_chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace mla
