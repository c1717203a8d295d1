// KV-cache append: writes each request's new K/V rows into its pages.
//
// Prefill computes K and V for the whole prompt (or chunk) and stores them in
// the KV cache for the decode steps that follow ("Flash Attention & Paged
// Attention", section "FA对Prefill阶段的影响"); the cache is a pool of
// fixed-size pages reached through a logical-to-physical page table (same
// page, section 2).  Request b's n_b new rows take logical positions
// cache_seqlens[b] - n_b ... cache_seqlens[b] - 1 (cache_seqlens counts the
// tokens after the append), position t landing in page block_table[b][t / 64],
// slot t % 64.
//
// A pure copy, bound by HBM bandwidth: one warp per new token moves that
// token's K and V rows of every kv head with 16-byte loads and stores (the
// source row is contiguous; in the NHD page layout so is the destination).
#pragma once

#include "ptx_sm100.cuh"

namespace fa {

constexpr int kAppendPage = 64;
constexpr int kAppendThreads = 256;

struct AppendParams {
  const uint4* k_new;           // [T_new, Hkv, d] bf16
  const uint4* v_new;
  const int32_t* cu_seqlens;    // [B+1] offsets of the new rows
  const int32_t* cache_seqlens; // [B] lengths after the append
  const int32_t* block_table;   // [B, max_pages]
  __nv_bfloat16* k_pages;
  __nv_bfloat16* v_pages;
  int64_t page_stride, token_stride, head_stride;   // elements
  int64_t pool_elems;           // elements from the pool's base to one past its last one
  int total_new;
  int batch;
  int num_kv_heads;
  int max_pages;
  int num_pages;
};

template <int D>
__global__ void __launch_bounds__(kAppendThreads) fa_append_kv_kernel(const AppendParams p) {
  constexpr int VEC = D * 2 / 16;   // 16-byte pieces per (token, head) row
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kAppendThreads / 32);
  for (int t = blockIdx.x * (kAppendThreads / 32) + (threadIdx.x >> 5); t < p.total_new; t += warps) {
    // request owning row t: the last b with cu_seqlens[b] <= t
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cu_seqlens[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int first = p.cu_seqlens[b];
    const int n = p.cu_seqlens[b + 1] - first;
    const int len = p.cache_seqlens[b];
    if (t < first || t - first >= n) continue;   // past cu_seqlens[batch]
    if (n > len || len > p.max_pages * kAppendPage) {
      if (lane == 0) record_status(FA_ERR_PLAN_MISMATCH);
      continue;
    }
    const int pos = len - n + (t - first);
    if (!FA_DBG_OK(pos >= 0 && pos / kAppendPage < p.max_pages)) continue;
    const int phys = p.block_table[static_cast<size_t>(b) * p.max_pages + pos / kAppendPage];
    if (phys < 0 || phys >= p.num_pages) {
      if (lane == 0) record_status(FA_ERR_BAD_PAGE);
      continue;
    }
    const int64_t dst_row = static_cast<int64_t>(phys) * p.page_stride +
                            static_cast<int64_t>(pos % kAppendPage) * p.token_stride;
    const size_t src_row = static_cast<size_t>(t) * p.num_kv_heads * VEC;
    const int pieces = p.num_kv_heads * VEC;
    // Up to four 16-byte pieces of K and of V per lane in flight before the
    // stores (the sources are read-only for the whole kernel).
    for (int e0 = lane; e0 < pieces; e0 += 4 * 32) {
      uint4 kv[4], vv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + 32 * u;
        if (e < pieces) {
          kv[u] = __ldg(p.k_new + src_row + e);
          vv[u] = __ldg(p.v_new + src_row + e);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + 32 * u;
        if (e < pieces) {
          const int64_t dst = dst_row + (e / VEC) * p.head_stride + (e % VEC) * 8;   // elements
          if (!FA_DBG_OK(dst >= 0 && dst + 8 <= p.pool_elems)) continue;
          *reinterpret_cast<uint4*>(p.k_pages + dst) = kv[u];
          *reinterpret_cast<uint4*>(p.v_pages + dst) = vv[u];
        }
      }
    }
  }
}

}  // namespace fa
