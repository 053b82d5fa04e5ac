/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) MLA paged-decode library.
 *
 * Multi-head Latent Attention decode over a paged latent KV cache: every
 * batch entry's q_len x H query rows (576 = 512 latent + 64 rope dims) attend
 * through a block table to one per-token latent cache shared by all heads
 * (K = all 576 dims of a cached row, V = its first 512 dims), causally among
 * the q_len tokens of the step. Output: BF16 rows plus an fp32 per-row LSE.
 *
 * Sources (prose only; the pages print no formulas or code):
 *   - tokenspeed-mla package card, "What it is and what it does": a decode
 *     path over FP16, BF16 or FP8 inputs that always writes BF16 output, run
 *     as two kernels (split-KV partials, then a reduction) with the split
 *     count and workspace size derived at run time.
 *   - TokenSpeed MLA article (最快MLA内核背后的秘密), section 二: split_kv and
 *     the workspace size follow from batch_size, q_len and max_seq_len;
 *     section 三: query-token folding (largest F with q_len % F == 0 and
 *     H * F <= 128); section 四: causal and LSE outputs; section 六: tensor
 *     layouts query [B, q_len, H, D_qk], kv_cache [num_pages, page_size,
 *     D_total] plus block_tables.
 *
 * Conventions for every entry point:
 *   - Return 0 (MLA_OK) on success, a negative mla_status otherwise. Host-side
 *     argument errors are detected before anything is enqueued.
 *   - Device pointers are raw CUDA device addresses owned by the caller (in
 *     practice allocated by PyTorch). The library allocates no device memory
 *     and never synchronises the stream in mla_decode. A pointer the current
 *     device cannot address (pageable host memory, another device's memory)
 *     is refused with MLA_ERR_INVALID_ARG before anything is enqueued;
 *     mapped pinned host memory and managed memory are accepted.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream. All device work is enqueued on it, asynchronously.
 *   - Problems only the device can see (a block-table entry outside
 *     [0, num_pages), a seq_len above the planned maximum, a pipeline wait
 *     that ran out) are recorded as bits of a status word in the workspace
 *     header and never trap; read them with mla_decode_status. The affected
 *     rows' outputs are then unspecified but finite; no memory outside the
 *     arguments is touched.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_D_QK 576        /* latent (512) + rope (64) dims of q and of a cached row */
#define MLA_D_V 512         /* V = first 512 dims of the cached row */
#define MLA_PAGE_SIZE 64    /* tokens per cache page (the only page size supported) */
#define MLA_MAX_ROWS 128    /* rows (heads x folded tokens) one CTA pair processes */
#define MLA_NO_ALLOC_SCRATCH_BYTES (48u << 20) /* scratch of mla_decode_no_alloc, per device */

typedef enum { MLA_BF16 = 0, MLA_FP16 = 1, MLA_FP8_E4M3 = 2 } mla_dtype;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,       /* null pointer, negative size, bad dtype, ... */
  MLA_ERR_UNSUPPORTED_SHAPE = -2, /* e.g. page_size != 64, H > 128 */
  MLA_ERR_WORKSPACE_TOO_SMALL = -3,
  MLA_ERR_ARCH = -4,              /* current device is not sm_100 */
  MLA_ERR_CUDA = -5,              /* a CUDA runtime call failed */
  MLA_ERR_PLAN_MISMATCH = -6      /* plan fields inconsistent or not from mla_decode_plan */
} mla_status;

/* Work schedules of a plan (mla_plan.schedule). */
#define MLA_SCHEDULE_SPLITS 0u
#define MLA_SCHEDULE_BALANCED 1u

/* Bits of the device status word (workspace header). */
#define MLA_DEV_BAD_PAGE 0x1     /* block-table entry outside [0, num_pages): keys masked */
#define MLA_DEV_SEQ_TOO_LONG 0x2 /* seq_len above max_seq_len or the table width: clamped */
#define MLA_DEV_TIMEOUT 0x4      /* a bounded pipeline wait gave up; outputs unspecified */
#define MLA_DEV_BAD_QLEN 0x8     /* ragged queries: a cu_seqlens_q range decreasing, longer than the
                                    plan's max_q_len or past total_q; that entry gets no output */
#define MLA_DEV_BOUNDS 0x10      /* bounds-checking build only (mla_bounds_checked): a global
                                    index of the CTA-pair or combine kernels fell outside its
                                    buffer; that access was skipped, outputs unspecified */

typedef enum {
  MLA_KERNEL_AUTO = 0,         /* MLA_KERNEL_TCGEN05 */
  MLA_KERNEL_TCGEN05 = 1,      /* sm_100a tensor-core split-KV kernel (TMA + tcgen05 + TMEM); for FP8 the
                                  CTA-pair form whose MMAs span both CTAs (cta_group::2) */
  MLA_KERNEL_SIMT = 2,         /* plain CUDA-core kernel: a slow, simple cross-check */
  MLA_KERNEL_TCGEN05_SOLO = 3  /* FP8 only: tensor-core kernel whose two CTAs per unit each compute all
                                  scores and keep half of the output columns (no cross-CTA MMA) */
} mla_kernel;

/*
 * Plan of one decode shape. Filled by mla_decode_plan; treat as read-only.
 * Two work schedules exist (field `schedule`):
 *   MLA_SCHEDULE_SPLITS: every unit is cut into split_kv chunks of
 *     keys_per_split keys, one CTA (pair) each; partials [B*q_len*H, S, 512].
 *   MLA_SCHEDULE_BALANCED (CTA-pair kernels): split_kv = P CTA pairs stay
 *     resident; the units' 128-key tiles, counted from the device seq_lens,
 *     are dealt out as equal contiguous ranges. A unit a pair covers whole
 *     is written to out/lse directly; a unit cut between pairs leaves
 *     partials in slots (pair p: slot 2p for its first unit, 2p+1 for its
 *     last) that the combine merges: fp32 O as [2P][128 chunks of 4
 *     columns][M rows][4] at partial_offset, fp32 LSE as [2P][M] at
 *     lse_offset. Between the 256-byte status header and partial_offset
 *     lie B*G + 1 int32 counters (finished pieces per unit, then a flag for
 *     the unit table at the end of the workspace; before that table, a
 *     spill area for piece lists longer than a pair keeps in shared
 *     memory), cleared with the status
 *     word before every launch: the combine kernel is launched as the
 *     partial kernel's programmatic dependent and merges each unit as soon
 *     as its counter is complete. keys_per_split then only
 *     bounds seq_len (>= max_seq_len).
 *   fold            F: query tokens folded into the row dimension
 *   q_groups        G = q_len / F; each (batch entry, group) is one unit
 *   rows_per_unit   M = H * F <= 128 query rows that share each K tile
 *   split_kv        S: key chunks per unit processed in parallel
 *   keys_per_split  chunk length in keys (multiple of 64); split s covers
 *                   keys [s * keys_per_split, (s + 1) * keys_per_split)
 *   num_ctas        CTAs of the partial kernel
 *   workspace_bytes bytes the caller must pass as workspace (>= 256)
 *   partial_offset, lse_offset  byte offsets of the fp32 partial O
 *                   [B*q_len*H, S, 512] and partial LSE [B*q_len*H, S]
 *                   inside the workspace (used when split_kv > 1)
 */
typedef struct {
  int32_t batch, q_len, num_heads, max_seq_len, dtype;
  int32_t fold, q_groups, rows_per_unit;
  int32_t split_kv, keys_per_split;
  int32_t kernel, num_ctas;
  uint64_t workspace_bytes, partial_offset, lse_offset;
  uint32_t magic;    /* set by the planner; checked by mla_decode */
  uint32_t schedule; /* MLA_SCHEDULE_* below */
  int32_t window;    /* sliding window in keys (0 = none); set with mla_decode_plan_window */
  int32_t varlen;    /* 1: ragged query lengths (mla_prefill_plan / mla_prefill), q_len = the longest */
  int32_t fault_test; /* 0, as the planner sets it. Tests of failure detection only: 1 makes the
                         FP8 CTA-pair kernel leave the first tile of every pair unloaded, so that
                         the wait for it runs out (MLA_DEV_TIMEOUT after its 0.5 s limit, no
                         fault); 2, accepted by the bounds-checking build only, moves every
                         output row and partial slot of that kernel past its buffer, so that
                         the checks skip each store and set MLA_DEV_BOUNDS; refused on other
                         plans */
} mla_plan;

/*
 * mla_decode_plan: choose F, split_kv and the workspace size for a shape
 * (TokenSpeed MLA article, section 二 for split_kv and workspace sizing from
 * batch, q_len and max_seq_len; section 三 for the fold factor).
 * Pure host arithmetic on the 148-SM B200, deterministic and memoised; no
 * device calls. batch >= 0, 1 <= q_len, 1 <= num_heads <= 128,
 * max_seq_len >= 0, dtype an mla_dtype. Errors: MLA_ERR_INVALID_ARG,
 * MLA_ERR_UNSUPPORTED_SHAPE. `plan` is written only on success.
 */
int mla_decode_plan(int batch, int q_len, int num_heads, int max_seq_len, int dtype,
                    mla_plan* plan);

/*
 * mla_decode_plan_custom: as mla_decode_plan, with overrides for tests and
 * tuning: split_kv > 0 forces S (clamped to the number of 64-key tiles),
 * fold > 0 forces F (must divide q_len with H * F <= 128), kernel selects an
 * mla_kernel. Zero means "choose automatically".
 */
int mla_decode_plan_custom(int batch, int q_len, int num_heads, int max_seq_len, int dtype,
                           int split_kv, int fold, int kernel, mla_plan* plan);

/*
 * mla_decode_plan_window: restrict every query row to its last `window`
 * visible keys (sliding-window decode, a decode option the TokenSpeed MLA
 * article lists among its tests, section 六): a row with n visible keys
 * attends to keys [max(0, n - window), n). window = 0 restores full
 * attention. Supported by the CTA-pair kernels (balanced schedule) and the
 * SIMT kernel; other plans return MLA_ERR_UNSUPPORTED_SHAPE. The plan's
 * workspace size does not change. Errors: MLA_ERR_INVALID_ARG (null plan,
 * window < 0), MLA_ERR_PLAN_MISMATCH (plan not from mla_decode_plan*).
 */
int mla_decode_plan_window(mla_plan* plan, int window);

/*
 * mla_decode: one decode step (tokenspeed-mla package card, "Quickstart":
 * query, kv_cache, workspace, block_tables, seq_lens, max_seq_len,
 * softmax_scale; layouts from the TokenSpeed MLA article, section 六).
 *
 *   plan            from mla_decode_plan for this batch/q_len/H/max_seq_len/dtype
 *   q               device, [B, q_len, H, 576] of plan->dtype, contiguous,
 *                   16-byte aligned
 *   kv_cache        device, [num_pages, page_size, 576] of plan->dtype,
 *                   contiguous, 16-byte aligned; page_size must be 64
 *   block_tables    device int32 [B, max_pages_per_seq]; entry j of row b is
 *                   the page holding keys 64j .. 64j+63 of entry b; entries
 *                   past ceil(seq_len/64) are never read
 *   seq_lens        device int32 [B]: keys in the cache for entry b, counting
 *                   this step's q_len tokens; token t of the step sees keys
 *                   0 .. seq_len - q_len + t (no key: out 0, lse -inf)
 *   softmax_scale   applied to q.k (e.g. 576^-0.5)
 *   q_scale, kv_scale  FP8 dequantisation: values are code * scale; the
 *                   cache's one scale serves K and V. Ignored (1) for 16-bit
 *   out             device bf16 [B, q_len, H, 512]
 *   lse             device fp32 [B, q_len, H], natural log of the sum of
 *                   exp(scaled scores); may be NULL
 *   workspace       device buffer of >= plan->workspace_bytes, 256-byte
 *                   aligned; holds the status word and the split partials.
 *                   Calls that share a workspace must not overlap on the GPU.
 *   stream          cudaStream_t as void*
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED_SHAPE,
 * MLA_ERR_WORKSPACE_TOO_SMALL, MLA_ERR_PLAN_MISMATCH, MLA_ERR_ARCH,
 * MLA_ERR_CUDA (launch failure). Nothing is enqueued when an error is
 * returned before the first launch. Capturable in a CUDA graph.
 */
int mla_decode(const mla_plan* plan, const void* q, const void* kv_cache, int64_t num_pages,
               int page_size, const int32_t* block_tables, int max_pages_per_seq,
               const int32_t* seq_lens, float softmax_scale, float q_scale, float kv_scale,
               void* out, float* lse, void* workspace, uint64_t workspace_bytes, void* stream);

/*
 * mla_decode_partial / mla_decode_combine: the two kernels of mla_decode,
 * enqueued separately (TokenSpeed MLA article, section 二: a split-KV kernel
 * writing partial outputs and LSEs, then a reduction kernel merging them).
 * Same arguments, validation and errors as mla_decode; calling
 * mla_decode_partial then mla_decode_combine on one stream equals one
 * mla_decode. mla_decode_partial resets the status word and, when
 * plan->split_kv == 1, writes out/lse itself; mla_decode_combine is then a
 * no-op. Exposed so that each kernel can be timed on its own.
 */
int mla_decode_partial(const mla_plan* plan, const void* q, const void* kv_cache,
                       int64_t num_pages, int page_size, const int32_t* block_tables,
                       int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                       float q_scale, float kv_scale, void* out, float* lse, void* workspace,
                       uint64_t workspace_bytes, void* stream);
int mla_decode_combine(const mla_plan* plan, const void* q, const void* kv_cache,
                       int64_t num_pages, int page_size, const int32_t* block_tables,
                       int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                       float q_scale, float kv_scale, void* out, float* lse, void* workspace,
                       uint64_t workspace_bytes, void* stream);

/*
 * Ragged-query (prefill) forms: chunked prefill of several sequences with
 * different numbers of new tokens, packed without padding (tokenspeed-mla
 * package card, "What it is and what it does": the prefill path handles
 * ragged variable-length sequences without padding and takes FP8 inputs;
 * TokenSpeed MLA article, section 一, its kernel table). The attention is
 * the decode's, in the latent form over the same paged cache: entry b has
 * q_len_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b] new tokens, already
 * written to the cache, and seq_lens[b] keys in all; its token t sees keys
 * 0 .. seq_lens[b] - q_len_b + t.
 *
 * mla_prefill_plan: as mla_decode_plan with max_q_len = the most new tokens
 * an entry may have. F is the largest fold with H * F <= 128 (need not
 * divide max_q_len); every entry gets ceil(max_q_len / F) query groups, the
 * ones past its tokens empty. Runs on the CTA-pair kernels (balanced
 * schedule, at most 65536 groups in all, else MLA_ERR_UNSUPPORTED_SHAPE);
 * mla_prefill_plan_custom also takes kernel = MLA_KERNEL_SIMT and forced
 * split_kv / fold, like mla_decode_plan_custom. The plan's `varlen` is 1.
 */
int mla_prefill_plan(int batch, int max_q_len, int num_heads, int max_seq_len, int dtype, mla_plan* plan);
int mla_prefill_plan_custom(int batch, int max_q_len, int num_heads, int max_seq_len, int dtype,
                            int split_kv, int fold, int kernel, mla_plan* plan);

/*
 * mla_prefill: one ragged prefill step. Arguments as mla_decode, except:
 *   plan          from mla_prefill_plan (varlen = 1)
 *   q             device, [total_q, H, 576]: the entries' new tokens, packed
 *   total_q       tokens in q, 0 <= total_q <= batch * max_q_len
 *   cu_seqlens_q  device int32 [B + 1], non-decreasing, cu[0] >= 0,
 *                 cu[B] <= total_q, each q_len_b <= max_q_len; a range that
 *                 breaks this sets MLA_DEV_BAD_QLEN and that entry gets no
 *                 output. Packed tokens outside every entry are not written.
 *   out           device bf16 [total_q, H, 512]; lse fp32 [total_q, H] or NULL
 * mla_prefill_partial / mla_prefill_combine: its two kernels, as
 * mla_decode_partial / mla_decode_combine. A decode plan, or a null
 * cu_seqlens_q, is refused (MLA_ERR_PLAN_MISMATCH / MLA_ERR_INVALID_ARG).
 */
int mla_prefill(const mla_plan* plan, const void* q, int64_t total_q, const int32_t* cu_seqlens_q,
                const void* kv_cache, int64_t num_pages, int page_size, const int32_t* block_tables,
                int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale, float q_scale,
                float kv_scale, void* out, float* lse, void* workspace, uint64_t workspace_bytes, void* stream);
int mla_prefill_partial(const mla_plan* plan, const void* q, int64_t total_q, const int32_t* cu_seqlens_q,
                        const void* kv_cache, int64_t num_pages, int page_size, const int32_t* block_tables,
                        int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale, float q_scale,
                        float kv_scale, void* out, float* lse, void* workspace, uint64_t workspace_bytes,
                        void* stream);
int mla_prefill_combine(const mla_plan* plan, const void* q, int64_t total_q, const int32_t* cu_seqlens_q,
                        const void* kv_cache, int64_t num_pages, int page_size, const int32_t* block_tables,
                        int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale, float q_scale,
                        float kv_scale, void* out, float* lse, void* workspace, uint64_t workspace_bytes,
                        void* stream);

/*
 * mla_decode_status: synchronise `stream`, copy the device status word of
 * `workspace` (MLA_DEV_* bits from the last mla_decode that used it) into
 * *device_status, and clear it if `clear` is non-zero. For tests and debug
 * tooling; it blocks. Errors: MLA_ERR_INVALID_ARG, MLA_ERR_CUDA.
 */
int mla_decode_status(void* workspace, void* stream, int clear, int32_t* device_status);

/*
 * mla_decode_no_alloc: mla_decode without a caller-provided workspace, for
 * callers that cannot allocate device memory (no counterpart on the pages:
 * an addition of this library). Examples: a plugin inside a serving engine
 * that has reserved all device memory for its own pool and gives its kernels
 * no allocator, or code where cudaMalloc is not allowed because it may
 * synchronise the device. The workspace is instead a scratch array of
 * MLA_NO_ALLOC_SCRATCH_BYTES in this library's own device memory, reserved on
 * every GPU that loads the library and held until the process exits; the
 * call itself allocates nothing (no cudaMalloc, no cudaFree).
 *   - Arguments, layouts and errors as mla_decode, minus workspace and
 *     workspace_bytes. A plan whose workspace_bytes exceeds
 *     MLA_NO_ALLOC_SCRATCH_BYTES is rejected with MLA_ERR_WORKSPACE_TOO_SMALL
 *     before anything is enqueued (use fewer splits or mla_decode).
 *   - Every call looks up the scratch array's device address in the current
 *     device's context (cudaGetSymbolAddress, a host-side query), so a
 *     context that was reset and created again gets the array's new address.
 *     The first lookup on a device loads the library's device code there:
 *     make the first call on a device before any stream capture on it.
 *   - Every call on a device shares the one scratch array and it keeps the
 *     last call's contents: calls that overlap on the GPU (different streams
 *     without ordering) race on it and must not be issued. The status word
 *     it holds is reset by each call; read it with
 *     mla_decode_no_alloc_status.
 */
int mla_decode_no_alloc(const mla_plan* plan, const void* q, const void* kv_cache,
                        int64_t num_pages, int page_size, const int32_t* block_tables,
                        int max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                        float q_scale, float kv_scale, void* out, float* lse, void* stream);

/*
 * mla_decode_no_alloc_status: mla_decode_status for the scratch array of
 * mla_decode_no_alloc on the current device (no counterpart on the pages).
 * Synchronises `stream`, copies the status word (MLA_DEV_* bits of the last
 * mla_decode_no_alloc on this device) into *device_status and clears it when
 * `clear` is non-zero. A caller of mla_decode_no_alloc never sees the
 * scratch address, so this is its only way to learn of bad pages, over-long
 * sequences or a wait that ran out. MLA_ERR_INVALID_ARG for a null
 * device_status; MLA_ERR_CUDA if the synchronise or the copy fails.
 */
int mla_decode_no_alloc_status(void* stream, int clear, int32_t* device_status);

/* Human-readable name of an mla_status code (static storage, never NULL). */
const char* mla_status_string(int code);

/* Library version string, e.g. "0.1.0". */
const char* mla_version(void);

/*
 * The CUDA runtime error behind this thread's most recent MLA_ERR_CUDA
 * (cudaError_t value; 0 if none yet). If `name` is not NULL it receives the
 * error's name (static storage, e.g. "cudaErrorInvalidValue"). Host only; no
 * CUDA call is made.
 */
int mla_last_cuda_error(const char** name);

/*
 * 1 in the bounds-checking build of this library (libmla_decode_check.so,
 * compiled with MLA_BOUNDS_CHECK=1), 0 in the normal one. The checking build
 * tests, on the device, every global index of the CTA-pair partial kernels,
 * their on-device schedule and the balanced combine against the extent of
 * its buffer (block-table rows, the piece spill area, the schedule table, the
 * unit counters, the partial slots, out and lse); an index outside sets
 * MLA_DEV_BOUNDS in the status word and the access is skipped instead of
 * made. It is slower and meant for debugging, not for production. Host only.
 */
int mla_bounds_checked(void);

/*
 * mla_kv_pack: write new tokens into the paged latent cache, fused with the
 * FP8 quantisation (tokenspeed-mla package card, "What it is and what it
 * does": one kernel packs K/V and quantises to FP8 in place of separate cat
 * and cast operations; TokenSpeed MLA article, section 一, kernel table
 * entry mla_kv_pack_quantize_fp8, and section 六 for the 576-wide row).
 *
 *   latent        [n_tokens, 512] in_dtype, contiguous, 16-byte aligned: the
 *                 latent (compressed K/V) part of each new token
 *   rope          [n_tokens, 64] in_dtype, contiguous, 16-byte aligned: the
 *                 rope key part
 *   slot_mapping  [n_tokens] int64, device: cache row page * 64 + offset of
 *                 token i; negative = skip the token; a slot at or past
 *                 num_pages * 64 skips the token and sets MLA_DEV_BAD_PAGE
 *                 in *device_status (when given)
 *   kv_cache      [num_pages, 64, 576] cache_dtype: row s becomes
 *                 [latent_i || rope_i]; other rows are untouched
 *   in_dtype      MLA_BF16 or MLA_FP16
 *   cache_dtype   MLA_FP8_E4M3: each element is E4M3FN(x / kv_scale), the
 *                 quotient formed in fp32 (IEEE division, round to nearest)
 *                 and rounded to nearest even, saturating to +-448, NaN
 *                 kept; or in_dtype: the row is copied
 *   kv_scale      finite, > 0 (the per-tensor dequantisation scale decode
 *                 takes; ignored for a 16-bit cache)
 *   device_status optional int32 device word (e.g. a decode workspace's
 *                 status word); may be NULL
 *
 * All pointers are device-addressable from the current device and owned by
 * the caller; nothing is allocated or synchronised. Argument errors return
 * MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED_SHAPE (page_size != 64) before
 * any launch. n_tokens = 0 is a no-op.
 */
int mla_kv_pack(const void* latent, const void* rope, int64_t n_tokens, const int64_t* slot_mapping,
                void* kv_cache, int64_t num_pages, int page_size, int in_dtype, int cache_dtype,
                float kv_scale, int32_t* device_status, void* stream);

/*
 * mla_kv_amax: largest |x| over the non-NaN elements of latent [n_tokens,
 * 512] and rope [n_tokens, 64] (in_dtype MLA_BF16 or MLA_FP16), written as
 * one fp32 to the device pointer `amax` (zeroed first, on `stream`): the
 * per-tensor scale amax / 448 of the FP8 cache recipe follows from it.
 * Same pointer rules and errors as mla_kv_pack.
 */
int mla_kv_amax(const void* latent, const void* rope, int64_t n_tokens, int in_dtype, float* amax,
                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
