/*
 * MLA paged-decode oracle: plain fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link or
 * call this file; only the tests, the package smoke check and the bench's
 * CPU-baseline leg use it. It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (the plain definition; no blocking, no splitting, no
 * online softmax):
 *   For every batch entry b, query token t < q_len and head h:
 *     n      = seq_len[b] - q_len + t + 1           visible keys (causal,
 *                                                    aligned to the end)
 *     k_j    = cache[block_table[b][j / page], j % page, 0:576]   j < n
 *     v_j    = k_j[0:512]
 *     s_j    = softmax_scale * <q[b,t,h,0:576], k_j>
 *     lse    = ln sum_j exp(s_j)
 *     out    = sum_j exp(s_j - lse) * v_j
 *   Rows with n <= 0 get out = 0 and lse = -inf.
 * Sources: tokenspeed-mla package card, "What it is and what it does"
 * (decode over a paged cache, FP16/BF16/FP8 inputs, BF16 output); TokenSpeed
 * MLA article (最快MLA内核背后的秘密), section 六 (query [B, q_len, H, D_qk],
 * kv_cache [num_pages, page_size, D_total], block_tables) and section 一
 * (the latent cache shared by all heads: K is the whole 576-wide latent+rope
 * row, V its first 512 entries). Causal masking among the q_len tokens and
 * the per-row LSE are the options named in section 四. The pages do not say
 * whether seq_len counts this step's q_len tokens; this oracle takes that it
 * does (token t of q_len sees keys up to seq_len - q_len + t).
 *
 * Also here: the same decode restricted to a sliding window (each row's last
 * W visible keys), and the fused K/V pack with the E4M3 encoder it uses.
 * Ragged prefill, in the Python wrapper, calls this decode once per entry
 * with that entry's query length.
 *
 * Inputs are the raw element bytes the GPU path also receives; this file
 * decodes them itself from the published encodings (IEEE 754 binary16,
 * bfloat16 = upper half of binary32, OCP OFP8 E4M3FN). FP8 values are
 * dequantised as code * scale with one fp32 scale for q and one for the
 * cache, and everything after decoding is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_FP16 = 1, ORACLE_FP8_E4M3 = 2 };

enum {
  ORACLE_OK = 0,
  ORACLE_EINVAL = -1,
  ORACLE_EPAGE = -2, /* block table entry outside [0, num_pages) */
  ORACLE_ENOMEM = -3
};

/* Mutations for the pin-sensitivity tests: each plants one plausible
 * mistake so a test can show that some pin catches it. 0 = none. */
enum {
  MUT_NONE = 0,
  MUT_DROP_ROPE = 1,      /* score ignores dims 512..575 */
  MUT_V_OFFSET = 2,       /* V taken from dims 64..575 instead of 0..511 */
  MUT_NO_CAUSAL = 3,      /* every token sees all seq_len keys */
  MUT_NO_SCALE = 4,       /* softmax_scale dropped */
  MUT_LSE_LOG2 = 5,       /* LSE reported in log2 units */
  MUT_PAGE_INDEX = 6,     /* block table skipped: slot j / page used as the page id */
  MUT_WRONG_SIGN = 7      /* exp(+lse - s) instead of exp(s - lse), renormalised */
};

double oracle_decode_bf16(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double oracle_decode_fp16(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int e = (bits >> 10) & 0x1f;
  int m = bits & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-10 * 2^-14 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp(1.0 + (double)m / 1024.0, e - 15);
  }
  return sign ? -v : v;
}

/* OCP OFP8 E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; largest finite 448. */
double oracle_decode_e4m3(uint8_t bits) {
  int sign = (bits >> 7) & 1;
  int e = (bits >> 3) & 0xf;
  int m = bits & 0x7;
  double v;
  if (e == 0xf && m == 0x7) return NAN;
  if (e == 0) {
    v = ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
  } else {
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  }
  return sign ? -v : v;
}

static double decode_elem(int dtype, const void* base, size_t idx) {
  switch (dtype) {
    case ORACLE_BF16: return oracle_decode_bf16(((const uint16_t*)base)[idx]);
    case ORACLE_FP16: return oracle_decode_fp16(((const uint16_t*)base)[idx]);
    default: return oracle_decode_e4m3(((const uint8_t*)base)[idx]);
  }
}

/* Decode a whole buffer to fp64 (used by the tests to pin the decoders). */
void oracle_decode_buffer(int dtype, const void* src, size_t n, double* dst) {
  for (size_t i = 0; i < n; ++i) dst[i] = decode_elem(dtype, src, i);
}

/*
 * oracle_mla_decode_range: attention of the selected rows restricted to the
 * visible keys j with key_lo <= j < key_hi (key_hi < 0 means no upper bound).
 * With key_lo = 0, key_hi = -1 this is the full decode. A window W > 0
 * (sliding-window decode, a decode option the TokenSpeed MLA article lists
 * among its tests in section 六) further limits a row with n visible keys to
 * its last W: keys j >= n - W. Rows are flat indices
 * r = (b * q_len + t) * H + h; rows == NULL means all B*q_len*H rows in order.
 * out is [n_rows, Dv] and lse [n_rows]; a row whose range holds no visible
 * key gets out = 0, lse = -inf.
 */
int oracle_mla_decode_range_w(int dtype, int B, int q_len, int H, int D, int Dv,
                              const void* q, const void* cache, int64_t num_pages,
                              int page_size, const int32_t* block_tables,
                              int max_pages_per_seq, const int32_t* seq_lens,
                              double softmax_scale, double q_scale, double kv_scale,
                              int64_t n_rows, const int64_t* rows, int64_t key_lo,
                              int64_t key_hi, int64_t window, int mutation, double* out, double* lse) {
  if (B < 0 || q_len <= 0 || H <= 0 || D <= 0 || Dv <= 0 || Dv > D || page_size <= 0)
    return ORACLE_EINVAL;
  if (dtype != ORACLE_BF16 && dtype != ORACLE_FP16 && dtype != ORACLE_FP8_E4M3)
    return ORACLE_EINVAL;
  const int64_t total_rows = (int64_t)B * q_len * H;
  if (rows == NULL) n_rows = total_rows;
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= total_rows) return ORACLE_EINVAL;
  }
  const double qs = (dtype == ORACLE_FP8_E4M3) ? q_scale : 1.0;
  const double ks = (dtype == ORACLE_FP8_E4M3) ? kv_scale : 1.0;
  const double scale = (mutation == MUT_NO_SCALE) ? 1.0 : softmax_scale;
  const int v_off = (mutation == MUT_V_OFFSET) ? D - Dv : 0;
  const int d_score = (mutation == MUT_DROP_ROPE) ? Dv : D;
  int status = ORACLE_OK;

  for (int b = 0; b < B && status == ORACLE_OK; ++b) {
    /* Which requested rows belong to this batch entry? */
    int64_t cnt = 0;
    for (int64_t i = 0; i < n_rows; ++i) {
      int64_t r = rows ? rows[i] : i;
      if (r / ((int64_t)q_len * H) == b) ++cnt;
    }
    if (cnt == 0) continue;
    const int64_t nb = seq_lens[b] > 0 ? seq_lens[b] : 0;

    /* Gather and decode this entry's keys through the block table. */
    double* K = NULL;
    if (nb > 0) {
      K = (double*)malloc((size_t)nb * D * sizeof(double));
      if (!K) return ORACLE_ENOMEM;
    }
    int bad_page = 0;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nb; ++j) {
      int64_t slot = j / page_size, within = j % page_size;
      int64_t page;
      if (mutation == MUT_PAGE_INDEX)
        page = slot % num_pages;
      else
        page = (slot < max_pages_per_seq) ? block_tables[(int64_t)b * max_pages_per_seq + slot] : -1;
      if (page < 0 || page >= num_pages) {
        bad_page = 1;
        continue;
      }
      size_t base = ((size_t)page * page_size + (size_t)within) * D;
      for (int d = 0; d < D; ++d) K[(size_t)j * D + d] = decode_elem(dtype, cache, base + d) * ks;
    }
    if (bad_page) {
      free(K);
      return ORACLE_EPAGE;
    }

    int64_t* sel = (int64_t*)malloc((size_t)cnt * 2 * sizeof(int64_t));
    if (!sel) {
      free(K);
      return ORACLE_ENOMEM;
    }
    int64_t c = 0;
    for (int64_t i = 0; i < n_rows; ++i) {
      int64_t r = rows ? rows[i] : i;
      if (r / ((int64_t)q_len * H) == b) {
        sel[2 * c] = i;
        sel[2 * c + 1] = r;
        ++c;
      }
    }

    int alloc_fail = 0;
#pragma omp parallel
    {
      double* qv = (double*)malloc((size_t)D * sizeof(double));
      double* s = (double*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(double));
      if (!qv || !s) {
#pragma omp atomic write
        alloc_fail = 1;
      }
#pragma omp for schedule(dynamic, 1)
      for (int64_t ii = 0; ii < cnt; ++ii) {
        if (!qv || !s) continue;
        const int64_t oi = sel[2 * ii], r = sel[2 * ii + 1];
        const int t = (int)((r / H) % q_len);
        double* o = out + (size_t)oi * Dv;
        for (int d = 0; d < Dv; ++d) o[d] = 0.0;
        /* visible keys of this row */
        int64_t n = (mutation == MUT_NO_CAUSAL) ? nb : nb - q_len + t + 1;
        if (n > nb) n = nb;
        int64_t lo = key_lo > 0 ? key_lo : 0;
        if (window > 0 && n - window > lo) lo = n - window;
        int64_t hi = (key_hi >= 0 && key_hi < n) ? key_hi : n;
        if (hi <= lo) {
          lse[oi] = -INFINITY;
          continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = decode_elem(dtype, q, (size_t)r * D + d) * qs;
        /* pass 1: scores and their maximum */
        double m = -INFINITY;
        for (int64_t j = lo; j < hi; ++j) {
          const double* kj = K + (size_t)j * D;
          double dot = 0.0;
          for (int d = 0; d < d_score; ++d) dot += qv[d] * kj[d];
          s[j - lo] = scale * dot;
          if (s[j - lo] > m) m = s[j - lo];
        }
        /* pass 2: log-sum-exp, then the weighted sum of V */
        double sum = 0.0;
        for (int64_t j = lo; j < hi; ++j) sum += exp(s[j - lo] - m);
        double L = m + log(sum);
        double wsum = 0.0;
        for (int64_t j = lo; j < hi; ++j) {
          double w = (mutation == MUT_WRONG_SIGN) ? exp(L - s[j - lo]) : exp(s[j - lo] - L);
          wsum += w;
          const double* vj = K + (size_t)j * D + v_off;
          for (int d = 0; d < Dv; ++d) o[d] += w * vj[d];
        }
        if (mutation == MUT_WRONG_SIGN && wsum > 0)
          for (int d = 0; d < Dv; ++d) o[d] /= wsum;
        lse[oi] = (mutation == MUT_LSE_LOG2) ? L / log(2.0) : L;
      }
      free(qv);
      free(s);
    }
    free(sel);
    free(K);
    if (alloc_fail) status = ORACLE_ENOMEM;
  }
  return status;
}

int oracle_mla_decode_range(int dtype, int B, int q_len, int H, int D, int Dv,
                            const void* q, const void* cache, int64_t num_pages,
                            int page_size, const int32_t* block_tables,
                            int max_pages_per_seq, const int32_t* seq_lens,
                            double softmax_scale, double q_scale, double kv_scale,
                            int64_t n_rows, const int64_t* rows, int64_t key_lo,
                            int64_t key_hi, int mutation, double* out, double* lse) {
  return oracle_mla_decode_range_w(dtype, B, q_len, H, D, Dv, q, cache, num_pages, page_size, block_tables,
                                   max_pages_per_seq, seq_lens, softmax_scale, q_scale, kv_scale, n_rows, rows,
                                   key_lo, key_hi, 0, mutation, out, lse);
}

/* Full decode: all visible keys. */
int oracle_mla_decode(int dtype, int B, int q_len, int H, int D, int Dv, const void* q,
                      const void* cache, int64_t num_pages, int page_size,
                      const int32_t* block_tables, int max_pages_per_seq,
                      const int32_t* seq_lens, double softmax_scale, double q_scale,
                      double kv_scale, int64_t n_rows, const int64_t* rows, int mutation,
                      double* out, double* lse) {
  return oracle_mla_decode_range(dtype, B, q_len, H, D, Dv, q, cache, num_pages, page_size,
                                 block_tables, max_pages_per_seq, seq_lens, softmax_scale,
                                 q_scale, kv_scale, n_rows, rows, 0, -1, mutation, out, lse);
}

/*
 * LSE merge of partial results for one row (the reduction step of the
 * two-kernel split-KV decode, TokenSpeed MLA article section 二):
 *   L   = ln sum_s exp(lse_s)
 *   out = sum_s exp(lse_s - L) * o_s
 * Parts with lse = -inf carry no weight; if all are -inf, out = 0, L = -inf.
 */
void oracle_lse_merge(int n_parts, int Dv, const double* o_parts, const double* lse_parts,
                      double* out, double* lse) {
  double m = -INFINITY;
  for (int s = 0; s < n_parts; ++s)
    if (lse_parts[s] > m) m = lse_parts[s];
  for (int d = 0; d < Dv; ++d) out[d] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int s = 0; s < n_parts; ++s) sum += exp(lse_parts[s] - m);
  double L = m + log(sum);
  for (int s = 0; s < n_parts; ++s) {
    if (lse_parts[s] == -INFINITY) continue;
    double w = exp(lse_parts[s] - L);
    for (int d = 0; d < Dv; ++d) out[d] += w * o_parts[(size_t)s * Dv + d];
  }
  *lse = L;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the parallel loops use from now on (n >= 1; timing only, the
   results do not depend on it: every row is computed by one thread). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/*
 * Fused K/V pack + FP8 quantise (the cache-writing step before decode).
 * Sources: tokenspeed-mla package card, "What it is and what it does" (a
 * fused kernel packs K/V and quantises to FP8 in place of separate cat and
 * cast operations); TokenSpeed MLA article (最快MLA内核背后的秘密), section
 * 一 (its kernel table: mla_kv_pack_quantize_fp8) and section 六 (the
 * 576-wide cache row). Token i's cache row is [latent_i (512) || rope_i (64)]
 * written at row slot_mapping[i] of [num_pages * page_size, 576] (slots < 0
 * are skipped). With an FP8 cache each element is E4M3FN(x / kv_scale); the
 * pages fix no precision for the quotient, so it is formed in fp32, the
 * precision the CUDA kernel takes the same decision in, and rounded to
 * E4M3 from that exact fp32 value.
 */

/* OCP OFP8 E4M3FN encoding: round to nearest, ties to even; finite values
 * past the largest code and infinities saturate to +-448 (S.1111.110); NaN
 * encodes as S.1111.111. */
uint8_t oracle_encode_e4m3(float v) {
  const int sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (isnan(v)) return (uint8_t)(sign | 0x7f);
  if (a > 448.0) return (uint8_t)(sign | 0x7e);
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: steps of 2^-9; rounding up to 8 steps gives the
     * smallest normal code 0x08 */
    const double q = nearbyint(a * 512.0);
    return (uint8_t)(sign | (int)q);
  }
  int e = ilogb(a);                         /* 2^e <= a < 2^(e+1), e in [-6, 8] */
  double q = nearbyint(ldexp(a, 3 - e));    /* 8 + 3 mantissa bits, in [8, 16] */
  if (q == 16.0) {
    q = 8.0;
    e += 1;
  }
  if (e > 8) return (uint8_t)(sign | 0x7e); /* rounded past 448 */
  return (uint8_t)(sign | ((e + 7) << 3) | ((int)q - 8));
}

void oracle_encode_e4m3_buffer(const float* src, size_t n, uint8_t* dst) {
  for (size_t i = 0; i < n; ++i) dst[i] = oracle_encode_e4m3(src[i]);
}

/* Pack n tokens into the cache. in_dtype: ORACLE_BF16 or ORACLE_FP16;
 * cache_dtype: ORACLE_FP8_E4M3 (quantise with kv_scale) or in_dtype (copy of
 * the 16-bit bits). Returns ORACLE_EPAGE if a slot is >= num_slots. */
int oracle_kv_pack(int in_dtype, int cache_dtype, const void* latent, const void* rope, int64_t n,
                   const int64_t* slots, float kv_scale, void* cache, int64_t num_slots) {
  if (in_dtype != ORACLE_BF16 && in_dtype != ORACLE_FP16) return ORACLE_EINVAL;
  if (cache_dtype != ORACLE_FP8_E4M3 && cache_dtype != in_dtype) return ORACLE_EINVAL;
  for (int64_t i = 0; i < n; ++i) {
    const int64_t s = slots[i];
    if (s < 0) continue;
    if (s >= num_slots) return ORACLE_EPAGE;
    for (int d = 0; d < 576; ++d) {
      const uint16_t bits = d < 512 ? ((const uint16_t*)latent)[i * 512 + d]
                                    : ((const uint16_t*)rope)[i * 64 + (d - 512)];
      if (cache_dtype == ORACLE_FP8_E4M3) {
        const float x = (float)decode_elem(in_dtype, &bits, 0); /* exact: 16-bit values fit fp32 */
        const float quot = x / kv_scale;                         /* fp32 division, rounded to nearest */
        ((uint8_t*)cache)[s * 576 + d] = oracle_encode_e4m3(quot);
      } else {
        ((uint16_t*)cache)[s * 576 + d] = bits;
      }
    }
  }
  return ORACLE_OK;
}

/* Largest |x| over the non-NaN elements of n tokens' latent and rope parts. */
double oracle_kv_amax(int in_dtype, const void* latent, const void* rope, int64_t n) {
  double m = 0.0;
  for (int64_t i = 0; i < n * 512; ++i) {
    const double x = fabs(decode_elem(in_dtype, latent, (size_t)i));
    if (!isnan(x) && x > m) m = x;
  }
  for (int64_t i = 0; i < n * 64; ++i) {
    const double x = fabs(decode_elem(in_dtype, rope, (size_t)i));
    if (!isnan(x) && x > m) m = x;
  }
  return m;
}
