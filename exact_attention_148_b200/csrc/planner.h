// Host-side decode planner: chooses how each request's cached context is split
// across CTAs (Flash-Decoding's split along the sequence, sized from the SM
// count as the "plan" stage of wsisp.com "FIA / FlashAttention", section 二
// describes: preprocess the variable lengths, balance the load, assign blocks).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <vector>

namespace fa {

constexpr uint32_t kPlanMagic = 0xFA148D0Cu;
constexpr int kMaxSplits = 128;
constexpr int kMinChunkTokens = 512;
constexpr int kItemsPerSlot = 8;   // the many-small-items candidate: items per resident CTA slot
// Decode-time simulation: last splits kept in per-request queues up to this
// many (batch x units) entries, one heap of all running ones beyond.
constexpr int64_t kMaxQueuedLast = int64_t{1} << 21;

struct DecodePlan {
  uint32_t magic = kPlanMagic;
  int batch = 0, num_q_heads = 0, num_kv_heads = 0, head_dim = 0;
  int page_size = 0, max_pages_per_seq = 0, num_sms = 0;
  int group = 1;          // Hq / Hkv
  int kv_elem_bytes = 2;  // 2 = bf16 cache, 1 = E4M3 cache
  int q_len = 1;          // query tokens per request (multi-token decode on tensor cores)
  bool tensor_cores = false;  // tcgen05 split kernel (all G heads of a kv head per CTA)
  int heads_per_cta = 1;  // GC: G on tensor cores, else largest of 8, 4, 2, 1 dividing the group
  int subgroups = 1;      // group / GC
  int chunk_tokens = 0;
  int max_splits = 1;
  int max_seqlen = 0;
  int num_work_items = 0;
  size_t ws_o_offset = 0, ws_lse_offset = 0, workspace_bytes = 0;
  std::vector<int32_t> seqlens;   // planned cache lengths
};

// kernel: 0 = choose, 1 = CUDA-core split kernel, 2 = tensor-core split kernel.
constexpr int kDecodeKernelAuto = 0, kDecodeKernelCudaCores = 1, kDecodeKernelTensorCores = 2;
constexpr int kTensorCoreMaxGroup = 16;   // q_len * G operand rows per CTA

// Returns an fa_status.  Pure host code (no CUDA calls).
int make_decode_plan(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                     int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                     int num_sms, int num_splits_override, int kv_elem_bytes, int kernel,
                     int q_len, DecodePlan* plan);

}  // namespace fa
