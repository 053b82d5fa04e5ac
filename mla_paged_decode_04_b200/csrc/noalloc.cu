// Decode entry point for callers that cannot allocate device memory.
//
// mla_decode needs a workspace (status word plus the split-KV partials) that
// the caller allocates. Some callers cannot do that: a plugin inside a
// serving engine that has reserved all device memory for its own pool and
// offers its kernels no allocator, or code running where cudaMalloc is not
// allowed (it may synchronise the device, which a latency-critical decode loop
// or another library's critical section must not do). mla_decode_no_alloc
// serves them with a scratch buffer that lives in this library's own device
// memory: a file-scope array of MLA_NO_ALLOC_SCRATCH_BYTES, reserved on every
// GPU that loads the library and held until the process exits.
//
// The array's name is only a host-side stand-in. Its device address is looked
// up with cudaGetSymbolAddress on every call, with the calling device current,
// and then passed to the kernels like any workspace. The lookup is a host-side
// table query, so it costs little, and it always names the array of the
// current context: after a cudaDeviceReset the module is loaded again and the
// array may sit at another address. The first lookup on a device loads the
// module there (lazy loading), so the first call on a device should come
// before any stream capture on it. Nothing here calls cudaMalloc or cudaFree.
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_no_alloc_scratch[MLA_NO_ALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current device's context.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaError_t e = cudaGetSymbolAddress(&p, g_no_alloc_scratch); e != cudaSuccess) return mla::cuda_failure(e);
  if (p == nullptr) return mla::cuda_failure(cudaErrorInvalidSymbol);
  *out = p;
  return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_no_alloc(const mla_plan* plan, const void* q, const void* kv_cache,
                                   int64_t num_pages, int page_size, const int32_t* block_tables,
                                   int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                                   float q_scale, float kv_scale, void* out, float* lse, void* stream) {
  if (!plan) return MLA_ERR_PLAN_MISMATCH;
  if (plan->workspace_bytes > (uint64_t)MLA_NO_ALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != MLA_OK) return rc;
  return mla_decode(plan, q, kv_cache, num_pages, page_size, block_tables, max_pages_per_seq, seq_lens,
                    softmax_scale, q_scale, kv_scale, out, lse, scratch, (uint64_t)MLA_NO_ALLOC_SCRATCH_BYTES,
                    stream);
}

extern "C" int mla_decode_no_alloc_status(void* stream, int clear, int32_t* device_status) {
  if (!device_status) return MLA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != MLA_OK) return rc;
  return mla_decode_status(scratch, stream, clear, device_status);
}
