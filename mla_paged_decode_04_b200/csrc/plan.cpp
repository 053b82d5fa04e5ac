// Host-side decode plan: fold factor, split_kv and workspace layout.
//
// Fold (TokenSpeed MLA article 最快MLA内核背后的秘密, section 三): the largest
// F with q_len % F == 0 and H * F <= 128, so that the F tokens x H heads of a
// query group fill the 128-row tensor-core tile; the q_len / F groups become
// separate work units.
//
// split_kv (same article, section 二): derived at run time from batch, q_len
// and max_seq_len. The pages do not print the rule; this planner takes the
// plain reading of "keep the whole GPU busy": enumerate the split counts,
// model the makespan of the partial kernel in 64-key tiles as
//   waves * (tiles per split + fixed CTA cost) + combine cost,
// with one CTA pair per two SMs (74 pairs per wave on 148 SMs), and take the
// cheapest. The result is memoised per shape.
//
// The CTA-pair kernels instead keep all 74 pairs resident and balance the
// work on the device (MLA_SCHEDULE_BALANCED): the plan only fixes the number
// of pairs and sizes the partial slots, the piece spill and the schedule
// table.
//
// Ragged queries (prefill; tokenspeed-mla package card, "What it is and what
// it does": variable-length sequences without padding): q_len is the longest
// entry's token count, F the largest fold with H * F <= 128 (it need not
// divide q_len, an entry's last group holds the remainder) and every entry
// gets ceil(q_len / F) groups; groups past an entry's tokens are empty.
#include <climits>
#include <map>
#include <mutex>
#include <tuple>

#include "internal.h"

namespace mla {
namespace {

constexpr double kFixedTiles = 4.0;       // prologue (Q load, TMEM alloc) + epilogue, in tiles
constexpr double kCombinePerSplit = 4.0;  // partial write + combine read per split, in tiles

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

void choose_split(int64_t units, int64_t tiles, int64_t slots_per_wave, int forced,
                  int* split_out, int* chunk_tiles_out) {
  if (tiles <= 0) {
    *split_out = 1;
    *chunk_tiles_out = 1;
    return;
  }
  if (forced > 0) {
    int64_t s = forced < tiles ? forced : tiles;
    int64_t ct = ceil_div(tiles, s);
    *split_out = (int)ceil_div(tiles, ct);
    *chunk_tiles_out = (int)ct;
    return;
  }
  double best = 1e300;
  int best_s = 1;
  int64_t best_ct = tiles;
  int64_t max_s = tiles < 256 ? tiles : 256;
  for (int64_t s = 1; s <= max_s; ++s) {
    int64_t ct = ceil_div(tiles, s);
    if (ceil_div(tiles, ct) != s) continue;  // same chunking as a smaller s
    int64_t waves = ceil_div(units * s, slots_per_wave);
    double cost = (double)waves * ((double)ct + kFixedTiles);
    if (s > 1) cost += kCombinePerSplit * (double)(s * units) / (double)slots_per_wave;
    if (cost < best - 1e-9) {
      best = cost;
      best_s = (int)s;
      best_ct = ct;
    }
  }
  *split_out = best_s;
  *chunk_tiles_out = (int)best_ct;
}

std::mutex g_mu;
std::map<std::tuple<int, int, int, int, int, int, int, int, int>, mla_plan> g_memo;

}  // namespace

int plan_impl(int batch, int q_len, int num_heads, int max_seq_len, int dtype, int split_kv,
              int fold, int kernel, int varlen, mla_plan* plan) {
  if (!plan) return MLA_ERR_INVALID_ARG;
  if (batch < 0 || q_len < 1 || num_heads < 1 || max_seq_len < 0 || split_kv < 0 || fold < 0)
    return MLA_ERR_INVALID_ARG;
  if (dtype != MLA_BF16 && dtype != MLA_FP16 && dtype != MLA_FP8_E4M3) return MLA_ERR_INVALID_ARG;
  if (kernel != MLA_KERNEL_AUTO && kernel != MLA_KERNEL_TCGEN05 && kernel != MLA_KERNEL_SIMT &&
      kernel != MLA_KERNEL_TCGEN05_SOLO)
    return MLA_ERR_INVALID_ARG;
  if (kernel == MLA_KERNEL_TCGEN05_SOLO && dtype != MLA_FP8_E4M3) return MLA_ERR_INVALID_ARG;
  if (num_heads > MLA_MAX_ROWS) return MLA_ERR_UNSUPPORTED_SHAPE;
  if (max_seq_len > (1 << 30)) return MLA_ERR_UNSUPPORTED_SHAPE;

  if (varlen && kernel == MLA_KERNEL_TCGEN05_SOLO) return MLA_ERR_UNSUPPORTED_SHAPE;
  auto key = std::make_tuple(batch, q_len, num_heads, max_seq_len, dtype, split_kv, fold, kernel, varlen);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_memo.find(key);
    if (it != g_memo.end()) {
      *plan = it->second;
      return MLA_OK;
    }
  }

  // Ragged queries (prefill): q_len is the longest entry, and an entry's last
  // group may hold fewer than F tokens, so F need not divide q_len.
  int F = 0;
  if (fold > 0) {
    if (fold > q_len || (!varlen && q_len % fold != 0) || num_heads * fold > MLA_MAX_ROWS)
      return MLA_ERR_UNSUPPORTED_SHAPE;
    F = fold;
  } else {
    for (int f = q_len; f >= 1; --f)
      if ((varlen || q_len % f == 0) && num_heads * f <= MLA_MAX_ROWS) {
        F = f;
        break;
      }
  }
  const int G = (q_len + F - 1) / F;
  const int M = num_heads * F;
  int kern = kernel == MLA_KERNEL_AUTO ? MLA_KERNEL_TCGEN05 : kernel;
  const int64_t units = (int64_t)batch * G;
  const int64_t tiles = ceil_div(max_seq_len, kTileKeys);
  // The tcgen05 kernel runs one CTA pair per two SMs; the SIMT kernel uses
  // the same split so that both produce the same partial layout.
  const int64_t slots = kNumSMs / 2;
  int S = 1, chunk_tiles = 1;
  choose_split(units > 0 ? units : 1, tiles, slots, split_kv, &S, &chunk_tiles);

  mla_plan p{};
  p.batch = batch;
  p.q_len = q_len;
  p.num_heads = num_heads;
  p.max_seq_len = max_seq_len;
  p.dtype = dtype;
  p.fold = F;
  p.q_groups = G;
  p.rows_per_unit = M;
  const uint64_t rows = (uint64_t)batch * q_len * num_heads;
  // Every CTA of the balanced schedule (CTA-pair kernels) scans all units at
  // start; decode batches of more units than kMaxBalancedUnits take fixed
  // splits instead (FP8: the solo kernel; 16-bit: the exchange kernel).
  p.varlen = varlen ? 1 : 0;
  // the balanced schedule's int32 weights (3 per 64 keys at most, plus a unit's
  // lead-in) must fit
  const bool weights_fit = units * (tiles * 3 + kPieceLeadWeight) < (int64_t)INT32_MAX;
  const int64_t max_units = weights_fit ? (varlen ? kMaxVarlenUnits : kMaxBalancedUnits) : 0;
  if (kern == MLA_KERNEL_TCGEN05 && units > max_units) {
    // ragged queries run only on the balanced schedule (or the SIMT kernel)
    if (varlen) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (dtype == MLA_FP8_E4M3) kern = MLA_KERNEL_TCGEN05_SOLO;
  }
  p.kernel = kern;
  if (kern == MLA_KERNEL_TCGEN05 && units <= max_units) {
    const int P = split_kv > 0 ? (split_kv < kNumSMs / 2 ? split_kv : kNumSMs / 2) : kNumSMs / 2;
    p.schedule = MLA_SCHEDULE_BALANCED;
    p.split_kv = P;
    p.keys_per_split = (int32_t)(ceil_div(max_seq_len > 0 ? max_seq_len : 1, kTileKeys) * kTileKeys);
    p.num_ctas = 2 * P;
    const uint64_t slots = 2 * (uint64_t)P;
    uint64_t off = kHeaderBytes + balanced_counter_bytes(units);  // status, then the unit counters
    p.partial_offset = off;
    off += slots * (uint64_t)M * MLA_D_V * sizeof(float);
    off = (off + 255) & ~uint64_t(255);
    p.lse_offset = off;
    off += slots * (uint64_t)M * sizeof(float);
    off = (off + 255) & ~uint64_t(255);
    off += balanced_spill_bytes(units, P);  // piece lists too long for shared memory
    off += balanced_table_bytes(units);     // unit start table, at the end of the workspace
    p.workspace_bytes = off;
  } else {
    p.schedule = MLA_SCHEDULE_SPLITS;
    p.split_kv = S;
    p.keys_per_split = chunk_tiles * kTileKeys;
    p.num_ctas = (int32_t)(units * S * (kern == MLA_KERNEL_TCGEN05 || kern == MLA_KERNEL_TCGEN05_SOLO ? 2 : 1));
    uint64_t off = kHeaderBytes;
    p.partial_offset = off;
    p.lse_offset = off;
    if (S > 1) {
      p.partial_offset = off;
      off += rows * (uint64_t)S * MLA_D_V * sizeof(float);
      off = (off + 255) & ~uint64_t(255);
      p.lse_offset = off;
      off += rows * (uint64_t)S * sizeof(float);
      off = (off + 255) & ~uint64_t(255);
    }
    p.workspace_bytes = off;
  }
  p.magic = kPlanMagic;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_memo.size() > 4096) g_memo.clear();
    g_memo[key] = p;
  }
  *plan = p;
  return MLA_OK;
}

}  // namespace mla

extern "C" int mla_decode_plan(int batch, int q_len, int num_heads, int max_seq_len, int dtype,
                               mla_plan* plan) {
  return mla::plan_impl(batch, q_len, num_heads, max_seq_len, dtype, 0, 0, MLA_KERNEL_AUTO, 0, plan);
}

extern "C" int mla_decode_plan_custom(int batch, int q_len, int num_heads, int max_seq_len,
                                      int dtype, int split_kv, int fold, int kernel,
                                      mla_plan* plan) {
  return mla::plan_impl(batch, q_len, num_heads, max_seq_len, dtype, split_kv, fold, kernel, 0, plan);
}

extern "C" int mla_prefill_plan(int batch, int max_q_len, int num_heads, int max_seq_len, int dtype,
                                mla_plan* plan) {
  return mla::plan_impl(batch, max_q_len, num_heads, max_seq_len, dtype, 0, 0, MLA_KERNEL_AUTO, 1, plan);
}

extern "C" int mla_prefill_plan_custom(int batch, int max_q_len, int num_heads, int max_seq_len, int dtype,
                                       int split_kv, int fold, int kernel, mla_plan* plan) {
  return mla::plan_impl(batch, max_q_len, num_heads, max_seq_len, dtype, split_kv, fold, kernel, 1, plan);
}
