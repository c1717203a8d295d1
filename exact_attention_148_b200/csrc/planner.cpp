#include "planner.h"

#include <algorithm>

#include "../../include/exact_attention.h"

namespace fa {

namespace {
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
}  // namespace

int make_decode_plan(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                     int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                     int num_sms, int num_splits_override, DecodePlan* plan) {
  if (plan == nullptr || cache_seqlens_host == nullptr) return FA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || num_q_heads < 1 || num_kv_heads < 1 ||
      max_pages_per_seq < 1 || num_sms < 1 || num_splits_override < 0)
    return FA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (page_size != 64) return FA_ERR_UNSUPPORTED;
  const int64_t capacity = static_cast<int64_t>(max_pages_per_seq) * page_size;
  if (capacity > (int64_t{1} << 30)) return FA_ERR_INVALID_ARG;

  DecodePlan pl;
  pl.batch = batch;
  pl.num_q_heads = num_q_heads;
  pl.num_kv_heads = num_kv_heads;
  pl.head_dim = head_dim;
  pl.page_size = page_size;
  pl.max_pages_per_seq = max_pages_per_seq;
  pl.num_sms = num_sms;
  pl.group = num_q_heads / num_kv_heads;
  for (int gc : {8, 4, 2, 1})
    if (pl.group % gc == 0) {
      pl.heads_per_cta = gc;
      break;
    }
  pl.subgroups = pl.group / pl.heads_per_cta;
  if (static_cast<int64_t>(num_kv_heads) * pl.subgroups > 65535) return FA_ERR_UNSUPPORTED;

  pl.seqlens.assign(cache_seqlens_host, cache_seqlens_host + batch);
  int64_t total = 0;
  int max_len = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t L = pl.seqlens[b];
    // Cache-overflow check: a length the block table cannot address is an error.
    if (L < 0 || L > capacity) return FA_ERR_INVALID_ARG;
    total += L;
    max_len = std::max(max_len, static_cast<int>(L));
  }
  pl.max_seqlen = max_len;
  const int64_t units = static_cast<int64_t>(num_kv_heads) * pl.subgroups;   // CTAs per split

  int64_t chunk;
  if (num_splits_override > 0) {
    chunk = round_up(std::max<int64_t>(1, ceil_div(max_len, num_splits_override)), page_size);
  } else {
    // Aim for about kItemsPerSlot items per resident CTA slot so the hardware
    // scheduler's greedy assignment leaves a short tail, but never split below
    // kMinChunkTokens keys (each CTA must amortise its pipeline fill).
    const int64_t slots = static_cast<int64_t>(num_sms) * kDecodeCtasPerSm;
    const int64_t target = ceil_div(total * units, slots * kItemsPerSlot);
    chunk = round_up(std::max<int64_t>(target, kMinChunkTokens), page_size);
  }
  if (max_len > 0 && ceil_div(max_len, chunk) > kMaxSplits)
    chunk = round_up(ceil_div(max_len, kMaxSplits), page_size);
  chunk = std::max<int64_t>(chunk, page_size);
  pl.chunk_tokens = static_cast<int>(chunk);
  pl.max_splits = static_cast<int>(std::max<int64_t>(1, ceil_div(max_len, chunk)));

  int64_t items = 0;
  for (int b = 0; b < batch; ++b) items += std::max<int64_t>(1, ceil_div(pl.seqlens[b], chunk));
  pl.num_work_items = static_cast<int>(items * units);

  if (pl.max_splits > 1) {
    const size_t rows = static_cast<size_t>(batch) * num_q_heads;
    pl.ws_o_offset = 0;
    pl.ws_lse_offset = align256(static_cast<size_t>(pl.max_splits) * rows * head_dim * 4);
    pl.workspace_bytes = align256(pl.ws_lse_offset + static_cast<size_t>(pl.max_splits) * rows * 4);
  } else {
    pl.workspace_bytes = 0;
  }
  *plan = std::move(pl);
  return FA_OK;
}

}  // namespace fa
