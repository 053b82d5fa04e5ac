// C ABI: argument validation, workspace layout and kernel launches.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace mla {

namespace {
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
}  // namespace

int cuda_failure(cudaError_t e) {
  g_last_cuda_error = e;
  return MLA_ERR_CUDA;
}

namespace {

constexpr float kLog2e = 1.4426950408889634f;

int check_device_arch() {
  static std::mutex mu;
  static int cached[64];
  static bool init = false;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_failure(e);
  if (dev < 0 || dev >= 64) return MLA_ERR_ARCH;
  std::lock_guard<std::mutex> lk(mu);
  if (!init) {
    for (int i = 0; i < 64; ++i) cached[i] = 1;  // 1 = unknown
    init = true;
  }
  if (cached[dev] == 1) {
    int major = 0, minor = 0;
    if (cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev); e != cudaSuccess)
      return cuda_failure(e);
    if (cudaError_t e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev); e != cudaSuccess)
      return cuda_failure(e);
    cached[dev] = (major == 10 && minor == 0) ? MLA_OK : MLA_ERR_ARCH;
  }
  return cached[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The current device can address `ptr`: its own device or managed memory, or
// host memory mapped into the device address space. A pageable host pointer
// (or another device's memory) would fault inside a kernel, so it is refused
// here. A host-side query; nothing is enqueued.
bool device_addressable(const void* ptr, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    (void)cudaGetLastError();  // not the caller's error to see later
    return false;
  }
  if (at.type == cudaMemoryTypeDevice) return at.device == dev;
  if (at.type == cudaMemoryTypeManaged) return true;
  if (at.type == cudaMemoryTypeHost) return at.devicePointer == ptr;
  return false;
}

// The plan must be one the planner could have produced for its own fields.
int check_plan(const mla_plan* p) {
  if (!p || p->magic != kPlanMagic) return MLA_ERR_PLAN_MISMATCH;
  if (p->batch < 0 || p->q_len < 1 || p->num_heads < 1 || p->num_heads > MLA_MAX_ROWS ||
      p->max_seq_len < 0)
    return MLA_ERR_PLAN_MISMATCH;
  if (p->dtype != MLA_BF16 && p->dtype != MLA_FP16 && p->dtype != MLA_FP8_E4M3) return MLA_ERR_PLAN_MISMATCH;
  if (p->varlen != 0 && p->varlen != 1) return MLA_ERR_PLAN_MISMATCH;
  // decode: F divides q_len; ragged queries: an entry's last group may be short
  if (p->fold < 1 || p->fold > p->q_len || (!p->varlen && p->q_len % p->fold != 0) ||
      p->q_groups != (p->q_len + p->fold - 1) / p->fold || p->rows_per_unit != p->num_heads * p->fold ||
      p->rows_per_unit > MLA_MAX_ROWS)
    return MLA_ERR_PLAN_MISMATCH;
  if (p->split_kv < 1 || p->keys_per_split < kTileKeys || p->keys_per_split % kTileKeys != 0)
    return MLA_ERR_PLAN_MISMATCH;
  if ((int64_t)p->split_kv * p->keys_per_split < (int64_t)p->max_seq_len) return MLA_ERR_PLAN_MISMATCH;
  if (p->kernel != MLA_KERNEL_TCGEN05 && p->kernel != MLA_KERNEL_SIMT && p->kernel != MLA_KERNEL_TCGEN05_SOLO)
    return MLA_ERR_PLAN_MISMATCH;
  if (p->kernel == MLA_KERNEL_TCGEN05_SOLO && p->dtype != MLA_FP8_E4M3) return MLA_ERR_PLAN_MISMATCH;
  if (p->schedule != MLA_SCHEDULE_SPLITS && p->schedule != MLA_SCHEDULE_BALANCED) return MLA_ERR_PLAN_MISMATCH;
  if (p->window < 0) return MLA_ERR_PLAN_MISMATCH;
  // the failure-detection test modes exist on the FP8 CTA-pair kernel only;
  // mode 2 (stores past the buffers, caught by the checks) in the checking
  // build only
  if (p->fault_test != 0 &&
      !((p->fault_test == 1 || (p->fault_test == 2 && MLA_BOUNDS_CHECK)) && p->dtype == MLA_FP8_E4M3 &&
        p->kernel == MLA_KERNEL_TCGEN05 && p->schedule == MLA_SCHEDULE_BALANCED))
    return MLA_ERR_PLAN_MISMATCH;
  // a window and ragged queries run on the CTA-pair kernels and the SIMT kernel
  if ((p->window > 0 || p->varlen) &&
      !(p->kernel == MLA_KERNEL_SIMT || (p->kernel == MLA_KERNEL_TCGEN05 && p->schedule == MLA_SCHEDULE_BALANCED)))
    return MLA_ERR_PLAN_MISMATCH;
  if (p->schedule == MLA_SCHEDULE_BALANCED) {
    // CTA-pair kernels only; slots [2P, M, 512] fp32 + [2P, M] + unit table
    if (p->kernel != MLA_KERNEL_TCGEN05 || p->split_kv > kNumSMs / 2)
      return MLA_ERR_PLAN_MISMATCH;
    const int64_t units = (int64_t)p->batch * p->q_groups;
    if (units > (p->varlen ? kMaxVarlenUnits : kMaxBalancedUnits)) return MLA_ERR_PLAN_MISMATCH;
    const uint64_t slot_rows = 2ull * p->split_kv * p->rows_per_unit;
    if (p->partial_offset < (uint64_t)kHeaderBytes + balanced_counter_bytes(units) || p->partial_offset % 256 != 0 ||
        p->lse_offset < p->partial_offset + slot_rows * MLA_D_V * 4 || p->lse_offset % 256 != 0 ||
        p->workspace_bytes < p->lse_offset + slot_rows * 4 + balanced_spill_bytes(units, p->split_kv) +
                                 balanced_table_bytes(units))
      return MLA_ERR_PLAN_MISMATCH;
    return MLA_OK;
  }
  const uint64_t rows = (uint64_t)p->batch * p->q_len * p->num_heads;
  if (p->split_kv > 1) {
    if (p->partial_offset < (uint64_t)kHeaderBytes || p->partial_offset % 256 != 0 ||
        p->lse_offset < p->partial_offset + rows * (uint64_t)p->split_kv * MLA_D_V * 4 ||
        p->lse_offset % 256 != 0 ||
        p->workspace_bytes < p->lse_offset + rows * (uint64_t)p->split_kv * 4)
      return MLA_ERR_PLAN_MISMATCH;
  } else if (p->workspace_bytes < (uint64_t)kHeaderBytes) {
    return MLA_ERR_PLAN_MISMATCH;
  }
  return MLA_OK;
}

}  // namespace

namespace {

// Validate the arguments and fill the launch description. Returns MLA_OK or
// an error code; nothing is enqueued here.
// cu_q: null for decode (every entry has the plan's q_len tokens); for a
// ragged-query plan the device [B + 1] token offsets, with total_q tokens in q.
int prepare(const mla_plan* plan, const void* q, const void* kv_cache, int64_t num_pages,
            int page_size, const int32_t* block_tables, int max_pages_per_seq,
            const int32_t* seq_lens, float softmax_scale, float q_scale, float kv_scale, void* out,
            float* lse, void* workspace, uint64_t workspace_bytes, const int32_t* cu_q, int64_t total_q,
            DecodeArgs* a) {
  int rc = check_plan(plan);
  if (rc != MLA_OK) return rc;
  const mla_plan& p = *plan;
  if ((cu_q != nullptr) != (p.varlen != 0)) return MLA_ERR_PLAN_MISMATCH;
  if (!p.varlen) total_q = (int64_t)p.batch * p.q_len;
  // the fixed-split workspace holds B * q_len * H rows
  if (total_q < 0 || total_q > (int64_t)p.batch * p.q_len) return MLA_ERR_INVALID_ARG;
  if (page_size != MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned(workspace, 256)) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < p.workspace_bytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (p.dtype == MLA_FP8_E4M3 &&
      (!std::isfinite(q_scale) || !std::isfinite(kv_scale) || q_scale <= 0.f || kv_scale <= 0.f))
    return MLA_ERR_INVALID_ARG;
  if (p.batch > 0) {
    if (!q || !kv_cache || !block_tables || !seq_lens || !out) return MLA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16) || !aligned(block_tables, 4) ||
        !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)) || (cu_q && !aligned(cu_q, 4)))
      return MLA_ERR_INVALID_ARG;
    if (num_pages < 1 || max_pages_per_seq < 1) return MLA_ERR_INVALID_ARG;
    if (num_pages > (int64_t(1) << 31) / MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_failure(e);
    if (!device_addressable(q, dev) || !device_addressable(kv_cache, dev) ||
        !device_addressable(block_tables, dev) || !device_addressable(seq_lens, dev) ||
        !device_addressable(out, dev) || (lse && !device_addressable(lse, dev)) ||
        !device_addressable(workspace, dev) || (cu_q && !device_addressable(cu_q, dev)))
      return MLA_ERR_INVALID_ARG;
  }
  rc = check_device_arch();
  if (rc != MLA_OK) return rc;

  *a = DecodeArgs{};
  a->plan = p;
  a->q = q;
  a->kv_cache = kv_cache;
  a->num_pages = num_pages;
  a->block_tables = block_tables;
  a->max_pages_per_seq = max_pages_per_seq;
  a->seq_lens = seq_lens;
  const bool fp8 = p.dtype == MLA_FP8_E4M3;
  a->score_scale_log2 =
      (float)((double)softmax_scale * (fp8 ? (double)q_scale * kv_scale : 1.0) * (double)kLog2e);
  a->v_scale = fp8 ? kv_scale : 1.f;
  a->out = out;
  a->lse = lse;
  a->status = reinterpret_cast<int32_t*>(workspace);
  char* ws = reinterpret_cast<char*>(workspace);
  const bool partials = p.split_kv > 1 || p.schedule == MLA_SCHEDULE_BALANCED;
  a->o_part = partials ? reinterpret_cast<float*>(ws + p.partial_offset) : nullptr;
  a->lse_part = partials ? reinterpret_cast<float*>(ws + p.lse_offset) : nullptr;
  const int64_t units = (int64_t)p.batch * p.q_groups;
  a->sched = p.schedule == MLA_SCHEDULE_BALANCED
                 ? reinterpret_cast<int32_t*>(ws + p.workspace_bytes - balanced_table_bytes(units))
                 : nullptr;
  a->pieces = p.schedule == MLA_SCHEDULE_BALANCED
                  ? reinterpret_cast<int32_t*>(ws + p.workspace_bytes - balanced_table_bytes(units) -
                                               balanced_spill_bytes(units, p.split_kv))
                  : nullptr;
  a->cu_q = cu_q;
  a->total_q = total_q;
  a->unit_done = p.schedule == MLA_SCHEDULE_BALANCED ? reinterpret_cast<int32_t*>(ws + kHeaderBytes) : nullptr;
  return MLA_OK;
}

int run_partial(const DecodeArgs& a, cudaStream_t st) {
  // The status word, and for the balanced schedule the unit counters after it.
  // The balanced schedule clears them with a small kernel launched as a
  // programmatic dependent, and the partial kernel after it is one too: both
  // start while the kernel before them in the stream finishes (normally the
  // previous step's combine), and wait for it before touching memory.
  if (a.unit_done) {
    const uint64_t clear = kHeaderBytes + balanced_counter_bytes((int64_t)a.plan.batch * a.plan.q_groups);
    if (cudaError_t e = launch_workspace_clear(a.status, clear, st); e != cudaSuccess) return cuda_failure(e);
  } else if (cudaError_t e = cudaMemsetAsync(a.status, 0, sizeof(int32_t), st); e != cudaSuccess) {
    return cuda_failure(e);
  }
  if (a.plan.batch == 0 || a.total_q == 0) return MLA_OK;
  cudaError_t e;
  if (a.plan.kernel == MLA_KERNEL_SIMT)
    e = launch_simt_partial(a, st);
  else if (a.plan.kernel == MLA_KERNEL_TCGEN05_SOLO)
    e = launch_tc_fp8_partial(a, st);
  else if (a.plan.schedule == MLA_SCHEDULE_BALANCED)
    e = a.plan.dtype == MLA_FP8_E4M3 ? launch_tc_fp8_pair_partial(a, st) : launch_tc16_pair_partial(a, st);
  else
    e = launch_tc_partial(a, st);
  return e == cudaSuccess ? MLA_OK : cuda_failure(e);
}

int run_combine(const DecodeArgs& a, cudaStream_t st) {
  if (a.plan.batch == 0 || a.total_q == 0) return MLA_OK;
  if (a.plan.schedule == MLA_SCHEDULE_BALANCED) {
    const cudaError_t e = launch_combine_balanced(a, st);
    return e == cudaSuccess ? MLA_OK : cuda_failure(e);
  }
  if (a.plan.split_kv == 1) return MLA_OK;
  const cudaError_t e = launch_combine(a, st);
  return e == cudaSuccess ? MLA_OK : cuda_failure(e);
}

}  // namespace
}  // namespace mla

#define MLA_ARGS_DECL                                                                            \
  const mla_plan *plan, const void *q, const void *kv_cache, int64_t num_pages, int page_size, \
      const int32_t *block_tables, int max_pages_per_seq, const int32_t *seq_lens,              \
      float softmax_scale, float q_scale, float kv_scale, void *out, float *lse, void *workspace, \
      uint64_t workspace_bytes, void *stream
#define MLA_ARGS_FWD                                                                            \
  plan, q, kv_cache, num_pages, page_size, block_tables, max_pages_per_seq, seq_lens,          \
      softmax_scale, q_scale, kv_scale, out, lse, workspace, workspace_bytes, nullptr, 0
#define MLA_PREFILL_ARGS_DECL                                                                   \
  const mla_plan *plan, const void *q, int64_t total_q, const int32_t *cu_seqlens_q,            \
      const void *kv_cache, int64_t num_pages, int page_size, const int32_t *block_tables,      \
      int max_pages_per_seq, const int32_t *seq_lens, float softmax_scale, float q_scale,       \
      float kv_scale, void *out, float *lse, void *workspace, uint64_t workspace_bytes, void *stream
#define MLA_PREFILL_ARGS_FWD                                                                    \
  plan, q, kv_cache, num_pages, page_size, block_tables, max_pages_per_seq, seq_lens,          \
      softmax_scale, q_scale, kv_scale, out, lse, workspace, workspace_bytes, cu_seqlens_q, total_q

using namespace mla;

extern "C" int mla_decode(MLA_ARGS_DECL) {
  DecodeArgs a;
  int rc = prepare(MLA_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = run_partial(a, st);
  if (rc != MLA_OK) return rc;
  return run_combine(a, st);
}

extern "C" int mla_decode_partial(MLA_ARGS_DECL) {
  DecodeArgs a;
  int rc = prepare(MLA_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  return run_partial(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int mla_decode_combine(MLA_ARGS_DECL) {
  DecodeArgs a;
  int rc = prepare(MLA_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  return run_combine(a, reinterpret_cast<cudaStream_t>(stream));
}

// Ragged-query (prefill) forms: the same kernels, entries' tokens given by
// cu_seqlens_q. A null cu_seqlens_q is refused (it would select the decode
// geometry).
extern "C" int mla_prefill(MLA_PREFILL_ARGS_DECL) {
  if (!cu_seqlens_q) return MLA_ERR_INVALID_ARG;
  DecodeArgs a;
  int rc = prepare(MLA_PREFILL_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = run_partial(a, st);
  if (rc != MLA_OK) return rc;
  return run_combine(a, st);
}

extern "C" int mla_prefill_partial(MLA_PREFILL_ARGS_DECL) {
  if (!cu_seqlens_q) return MLA_ERR_INVALID_ARG;
  DecodeArgs a;
  int rc = prepare(MLA_PREFILL_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  return run_partial(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int mla_prefill_combine(MLA_PREFILL_ARGS_DECL) {
  if (!cu_seqlens_q) return MLA_ERR_INVALID_ARG;
  DecodeArgs a;
  int rc = prepare(MLA_PREFILL_ARGS_FWD, &a);
  if (rc != MLA_OK) return rc;
  return run_combine(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int mla_decode_status(void* workspace, void* stream, int clear, int32_t* device_status) {
  if (!workspace || !device_status) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaStreamSynchronize(st); e != cudaSuccess) return cuda_failure(e);
  int32_t v = 0;
  if (cudaError_t e = cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost); e != cudaSuccess)
    return cuda_failure(e);
  if (clear) {
    if (cudaError_t e = cudaMemset(workspace, 0, sizeof v); e != cudaSuccess) return cuda_failure(e);
  }
  *device_status = v;
  return MLA_OK;
}

extern "C" const char* mla_status_string(int code) {
  switch (code) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED_SHAPE: return "MLA_ERR_UNSUPPORTED_SHAPE";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_ARCH: return "MLA_ERR_ARCH";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_PLAN_MISMATCH: return "MLA_ERR_PLAN_MISMATCH";
    default: return "MLA_ERR_UNKNOWN";
  }
}

extern "C" const char* mla_version(void) { return "0.1.0"; }

extern "C" int mla_bounds_checked(void) { return MLA_BOUNDS_CHECK ? 1 : 0; }

extern "C" int mla_last_cuda_error(const char** name) {
  if (name) *name = cudaGetErrorName(g_last_cuda_error);
  return (int)g_last_cuda_error;
}

extern "C" int mla_kv_pack(const void* latent, const void* rope, int64_t n_tokens, const int64_t* slot_mapping,
                           void* kv_cache, int64_t num_pages, int page_size, int in_dtype, int cache_dtype,
                           float kv_scale, int32_t* device_status, void* stream) {
  if (n_tokens < 0 || num_pages < 0) return MLA_ERR_INVALID_ARG;
  if (page_size != MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED_SHAPE;
  if (in_dtype != MLA_BF16 && in_dtype != MLA_FP16) return MLA_ERR_INVALID_ARG;
  if (cache_dtype != MLA_FP8_E4M3 && cache_dtype != in_dtype) return MLA_ERR_INVALID_ARG;
  if (cache_dtype == MLA_FP8_E4M3 && (!std::isfinite(kv_scale) || kv_scale <= 0.f)) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!latent || !rope || !slot_mapping || !kv_cache) return MLA_ERR_INVALID_ARG;
  if (!aligned(latent, 16) || !aligned(rope, 16) || !aligned(kv_cache, 16) || !aligned(slot_mapping, 8) ||
      (device_status && !aligned(device_status, 4)))
    return MLA_ERR_INVALID_ARG;
  if (num_pages > (int64_t(1) << 40) / MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_failure(e);
  if (!device_addressable(latent, dev) || !device_addressable(rope, dev) || !device_addressable(slot_mapping, dev) ||
      !device_addressable(kv_cache, dev) || (device_status && !device_addressable(device_status, dev)))
    return MLA_ERR_INVALID_ARG;
  if (int rc = check_device_arch(); rc != MLA_OK) return rc;
  const cudaError_t e = launch_kv_pack(latent, rope, n_tokens, slot_mapping, kv_cache, num_pages * MLA_PAGE_SIZE,
                                       in_dtype, cache_dtype, kv_scale, device_status,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_failure(e);
}

extern "C" int mla_kv_amax(const void* latent, const void* rope, int64_t n_tokens, int in_dtype, float* amax,
                           void* stream) {
  if (n_tokens < 0 || !amax) return MLA_ERR_INVALID_ARG;
  if (in_dtype != MLA_BF16 && in_dtype != MLA_FP16) return MLA_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!latent || !rope)) return MLA_ERR_INVALID_ARG;
  if (!aligned(amax, 4) || (n_tokens > 0 && (!aligned(latent, 16) || !aligned(rope, 2)))) return MLA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_failure(e);
  if (!device_addressable(amax, dev) ||
      (n_tokens > 0 && (!device_addressable(latent, dev) || !device_addressable(rope, dev))))
    return MLA_ERR_INVALID_ARG;
  if (int rc = check_device_arch(); rc != MLA_OK) return rc;
  const cudaError_t e = launch_kv_amax(latent, rope, n_tokens, in_dtype, amax, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_failure(e);
}

namespace mla {
cudaError_t set_max_dynamic_smem(const void* func, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}
}  // namespace mla

extern "C" int mla_decode_plan_window(mla_plan* plan, int window) {
  if (!plan || window < 0) return MLA_ERR_INVALID_ARG;
  mla_plan p = *plan;
  p.window = 0;
  if (int rc = check_plan(&p); rc != MLA_OK) return rc;
  if (window > 0 && !(p.kernel == MLA_KERNEL_SIMT ||
                      (p.kernel == MLA_KERNEL_TCGEN05 && p.schedule == MLA_SCHEDULE_BALANCED)))
    return MLA_ERR_UNSUPPORTED_SHAPE;
  plan->window = window;
  return MLA_OK;
}
