// Persistent form of the ping-pong prefill (packed Q/K/V, bf16 or E4M3).
//
// Same roles, tiles, TMEM columns and per-tile math as fa_prefill_pp_kernel;
// the difference is what happens between work items.  In the grid form every
// (q tile pair, head pair) item is its own CTA, and each CTA pays for its
// launch, barrier and TMEM set-up, the latency of its first Q and K tiles,
// a first softmax with no second slot to overlap, and its last P V and
// epilogue with the tensor core idle.  Here one CTA per SM takes items from a
// global counter in launch order (heaviest first, so the greedy fill of the
// grid form is kept) and every pipeline runs on across items:
//
//   * the K/V ring, its barrier phases and the MMA stream never drain: the
//     producer loads K_0 of the next item as soon as a ring slot frees;
//   * a slot's Q tile is reloaded once the last S MMA of its previous item
//     has completed (q_empty, committed by the MMA warp after that MMA);
//   * the MMA warp issues S(i+1, 0) of a slot right after PV(i, last) of that
//     slot (the P columns it overwrites are consumed by then: the tcgen05
//     MMAs of one thread run in order), so the tensor core computes the next
//     item's first scores while the softmax warps write the current O;
//   * the softmax warps write O(i) and only then read S(i+1, 0) and arrive for
//     PV(i+1, 0), which overwrites O, so the O columns need no new barrier.
//
// Items pass from the producer warp (which takes their ids from the counter
// and decodes them) to the other roles, decoded, through a small
// shared-memory queue guarded by item_full / item_empty mbarriers, so no role
// but the producer reads global memory between items.  Every role takes every
// item, so all per-role counters (ring entries, Q loads, tiles per slot, f16
// V tiles) advance identically.  Once the last load of an item is issued, the
// producer claims the next one and asks L2 for its Q tiles and first K/V
// tiles.  The counter pair {next item, CTAs finished} is reset by the last CTA
// to finish, ready for the next launch on the same stream;
// the host gives each stream its own pair.
#pragma once

#include "prefill_pp_sm100.cuh"

namespace fa {

constexpr int kPersistQueue = 4;     // item ids in flight between the producer and the others
constexpr int kSchedSlots = 256;     // counter pairs: one per stream that launches this kernel

// One work item: two 128-row query slots of one sequence that read the same
// K/V tiles (two heads of a kv head at one q tile when the GQA group is even,
// else two consecutive q tiles of one head).  Same numbering as the grid
// form's CTA index: groups in launch order, heaviest q tiles first in a group.
struct PrefillItem {
  int id;          // item number, or -1: no more work
  int s0;          // first query of the sequence in the packed rows
  int L;           // its queries
  int Lk;          // its keys (= L for packed K/V; the cached length when paged)
  int seq;         // sequence (row of the block table when paged)
  int kv_head;
  int qtile[2];
  int head[2];
  int n_kv[2];     // key tiles of each slot (0: slot unused)
};

template <int D, bool F8 = false, bool PAGED = false>
struct PrefillPersistCfg {
  using B = PrefillPPCfg<D, F8>;
  // B's barriers, then q_empty[2], item_full[kPersistQueue], item_empty[kPersistQueue]
  static constexpr int NUM_BARS = B::NUM_BARS + 2 + 2 * kPersistQueue;
  static constexpr int QUEUE_OFF = (B::BAR_OFF + NUM_BARS * 8 + 15) & ~15;
  static constexpr int MISC_OFF = QUEUE_OFF + static_cast<int>(sizeof(PrefillItem)) * kPersistQueue;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int THREADS = B::THREADS;
  // roles that take each item from the queue: the MMA thread, 8 softmax warps,
  // and with E4M3 inputs the 2 converter warps
  static constexpr int CONSUMERS = 1 + 8 + (F8 ? 2 : 0);
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(!F8 || B::NS % 2 == 0, "E4M3: V tiles must stay on odd ring slots");
  static_assert(!(F8 && PAGED), "E4M3 inputs: packed K/V only");
};

// Launch arguments: the grid form's, plus the work counter.
struct PrefillPersistParams {
  PrefillParams p;
  uint32_t* sched;     // {next item, CTAs finished}; zero at launch, zero again at exit
  int total_items;     // work items of this launch
};

// Decode item idx.  The sequence bounds come from the device cu_seqlens; a
// sequence that leaves the T packed rows, or whose tile count differs from
// what the host planned for its group (cu_seqlens_dev != cu_seqlens_host), is
// recorded as FA_ERR_PLAN_MISMATCH and becomes an empty item.  PAGED: the
// keys are the sequence's cached length (cache_seqlens_dev); one below the
// query count or above the block table's capacity is recorded the same way
// and clamped, as in the grid form.
template <bool PAGED = false>
__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int idx, int BM, int BN) {
  int lo = 0, hi = p.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.group_start[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  PrefillItem w;
  w.id = idx;
  const int seq = static_cast<int>(p.group_id[lo] >> 16);
  w.kv_head = static_cast<int>(p.group_id[lo] & 0xFFFFu);
  const int rank = idx - p.group_start[lo];
  const bool seq_ok = FA_DBG_OK(seq < p.batch);
  w.seq = seq;
  w.s0 = seq_ok ? p.cu_seqlens[seq] : -1;
  w.L = seq_ok ? p.cu_seqlens[seq + 1] - w.s0 : 0;
  w.Lk = w.L;
  if constexpr (PAGED) {
    if (seq_ok) {
      int Lk = p.cache_seqlens[seq];
      const int cap = p.max_pages * kPrefillPage;
      if ((p.causal && Lk < w.L) || Lk > cap || Lk < 0) {
        if (rank == 0) record_status(FA_ERR_PLAN_MISMATCH);
        Lk = min(max(Lk, p.causal ? w.L : 0), cap);
      }
      w.Lk = Lk;
    }
  }
  const bool in_rows = w.s0 >= 0 && w.L >= 1 && w.s0 <= p.total_q - w.L;
  const int n_qtiles = in_rows ? (w.L + BM - 1) / BM : 0;
  const int n_ktiles = in_rows ? (w.Lk + BN - 1) / BN : 0;
  const int off = p.causal ? w.Lk - w.L : 0;   // query i sits at key position i + off
  const int G = p.group;
  const int planned = p.group_start[lo + 1] - p.group_start[lo];
  const int derived = ((G & 1) == 0) ? n_qtiles * (G >> 1) : ((n_qtiles + 1) >> 1) * G;
  if (!in_rows || derived != planned) {
    if (rank == 0) record_status(FA_ERR_PLAN_MISMATCH);
    w.s0 = 0;
    w.L = 0;
    w.Lk = 0;
    w.qtile[0] = w.qtile[1] = -1;
    w.head[0] = w.head[1] = 0;
    w.n_kv[0] = w.n_kv[1] = 0;
    return w;
  }
  if ((G & 1) == 0) {
    const int half = G >> 1;
    const int t = n_qtiles - 1 - rank / half;
    w.qtile[0] = w.qtile[1] = t;
    w.head[0] = w.kv_head * G + 2 * (rank % half);
    w.head[1] = w.head[0] + 1;
  } else {
    const int npairs = (n_qtiles + 1) >> 1;
    const int pr = npairs - 1 - rank / G;
    w.qtile[0] = 2 * pr;
    w.qtile[1] = 2 * pr + 1;
    w.head[0] = w.head[1] = w.kv_head * G + rank % G;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool active = w.qtile[k] >= 0 && w.qtile[k] < n_qtiles;
    w.n_kv[k] = !active ? 0 : (p.causal ? min(n_ktiles, (w.qtile[k] * BM + BM - 1 + off) / BN + 1) : n_ktiles);
  }
  return w;
}

template <int D, bool F8 = false, bool PAGED = false>
__global__ void __launch_bounds__(PrefillPersistCfg<D, F8, PAGED>::THREADS, 1)
    fa_prefill_persist_kernel(const __grid_constant__ PrefillPersistParams pp) {
  const PrefillParams& p = pp.p;
  using B = PrefillPPCfg<D, F8>;
  using C = PrefillPersistCfg<D, F8, PAGED>;
  constexpr int NS = B::NS;
  constexpr int QD = kPersistQueue;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t q_s = base + B::Q_OFF;
  auto kv_s = [&](uint32_t e) { return base + B::KV_OFF + (e % NS) * B::TILE_BYTES; };
  const uint32_t bars = base + B::BAR_OFF;
  const uint32_t bar_q = bars;
  auto bar_kv_full = [&](uint32_t e) { return bars + 8 * (1 + e % NS); };
  auto bar_kv_empty = [&](uint32_t e) { return bars + 8 * (1 + NS + e % NS); };
  auto bar_s_full = [&](int k) { return bars + 8 * (1 + 2 * NS + k); };
  auto bar_p_full = [&](int k) { return bars + 8 * (3 + 2 * NS + k); };
  auto bar_o_done = [&](int k) { return bars + 8 * (5 + 2 * NS + k); };
  const uint32_t bar_final = bars + 8 * (7 + 2 * NS);
  const uint32_t bar_vtail = bars + 8 * (8 + 2 * NS);   // PAGED: a V tile whose last page ends early
  const uint32_t bar_q1 = bars + 8 * (9 + 2 * NS);
  auto bar_vh_full = [&](int sl) { return bars + 8 * (10 + 2 * NS + sl); };
  auto bar_vh_empty = [&](int sl) { return bars + 8 * (12 + 2 * NS + sl); };
  auto bar_p_half = [&](int k) { return bars + 8 * (B::P_HALF_BAR + k); };
  auto bar_q_empty = [&](int k) { return bars + 8 * (B::NUM_BARS + k); };
  auto bar_item_full = [&](int i) { return bars + 8 * (B::NUM_BARS + 2 + i); };
  auto bar_item_empty = [&](int i) { return bars + 8 * (B::NUM_BARS + 2 + QD + i); };
  PrefillItem* queue = reinterpret_cast<PrefillItem*>(smem + C::QUEUE_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_q1, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar_kv_full(i), 1);
      // E4M3: the V tiles (odd ring entries, odd slots since NS is even and
      // every item has an even number of entries) are released by the two
      // converter warps, the K tiles by the MMA thread
      mbar_init(bar_kv_empty(i), (F8 && (i & 1)) ? 2 : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s_full(k), 1);
      mbar_init(bar_p_full(k), 4);
      mbar_init(bar_p_half(k), 4);
      mbar_init(bar_o_done(k), 1);
      mbar_init(bar_q_empty(k), 1);
      if constexpr (F8) {
        mbar_init(bar_vh_full(k), 2);
        mbar_init(bar_vh_empty(k), 1);
      }
    }
    for (int i = 0; i < QD; ++i) {
      mbar_init(bar_item_full(i), 1);
      mbar_init(bar_item_empty(i), C::CONSUMERS);
    }
    mbar_init(bar_final, 1);
    mbar_init(bar_vtail, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(tmem_slot), B::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  // A consumer warp's next item (id -1: no more work; -2: aborted).  All
  // lanes wait; lane 0 releases the queue entry once the item is in registers.
  auto take_item_warp = [&](int n) -> PrefillItem {
    const int qi = n % QD;
    PrefillItem w;
    if (!__all_sync(0xffffffffu, mbar_wait(bar_item_full(qi), (n / QD) & 1, abort_flag))) {
      w.id = -2;
      return w;
    }
    w = queue[qi];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_item_empty(qi));
    return w;
  };

  if (PAGED && warp == 8) {
    // ------------------------------------------ TMA producer + scheduler, paged K/V
    // The packed producer's order, with the grid form's paged loads: key tile
    // jt is logical pages 2jt and 2jt+1, whose physical ids the whole warp
    // reads 32 at a time; a page past the cache end or outside the pool loads
    // from page index num_pages (TMA zero fill, the bad id recorded).  The V
    // tile holding the cache's last page, when that page ends early, lands on
    // bar_vtail; once the item's loads are issued the warp zeroes the rows
    // past the end (0 * NaN would otherwise reach O) and marks the tile full.
    // Lane 0 claims the items and issues every copy and barrier operation.
    auto load_q = [&](int k, int h, int row0, uint32_t bar) {
      mbar_arrive_expect_tx(bar, B::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < B::CHUNKS; ++c)
        tma_load_3d(q_s + k * B::TILE_BYTES + c * B::CHUNK_BYTES, &p.tm_q, bar, c * 64, h, row0);
    };
    auto claim = [&]() -> PrefillItem {   // lane 0
      const int id = static_cast<int>(atomicAdd(pp.sched, 1u));
      PrefillItem w;
      if (id >= pp.total_items) {
        w.id = -1;
        return w;
      }
      w = prefill_item<true>(p, id, B::BM, B::BN);
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (w.n_kv[k] > 0)
#pragma unroll
          for (int c = 0; c < B::CHUNKS; ++c)
            tma_prefetch_l2_3d(&p.tm_q, c * 64, w.head[k], w.s0 + w.qtile[k] * B::BM);
      return w;
    };
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    uint32_t issued = 0;          // ring entries issued
    int qc0 = 0, qc1 = 0;         // Q loads of each slot
    int tails = 0;                // tail V tiles zeroed (bar_vtail phases)
    int tail_R = -1;              // ring entry of the tail V tile not yet marked full
    PrefillItem next;
    if (lane == 0) next = claim();
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int qi = n % QD;
      if (lane == 0) {
        ok = mbar_wait(bar_item_empty(qi), ((n / QD) & 1) ^ 1, abort_flag);
        if (ok) {
          queue[qi] = next;
          mbar_arrive(bar_item_full(qi));
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      const PrefillItem w = queue[qi];   // rewritten only QD items later
      if (w.id < 0) break;
      const int n_max = max(w.n_kv[0], w.n_kv[1]);
      const int32_t* bt_row = p.block_table + static_cast<size_t>(w.seq) * p.max_pages;
      const int tail_tile = (w.Lk % kPrefillPage != 0) ? (w.Lk - 1) / B::BN : -1;
      int pg_base = -1, pg_mine = 0;
      // ring entries K_0, V_0, K_1, V_1, ...; both Q tiles right after K_0
      for (int e = 0; e < 2 * n_max; ++e) {
        const int jt = e >> 1;
        const int lp0 = 2 * jt;
        if ((lp0 & ~31) != pg_base) {
          pg_base = lp0 & ~31;
          const int lp = pg_base + lane;
          int id = p.num_pages;
          if (lp * kPrefillPage < w.Lk && FA_DBG_OK(lp < p.max_pages)) {
            id = bt_row[lp];
            if (id < 0 || id >= p.num_pages) {
              record_status(FA_ERR_BAD_PAGE);
              id = p.num_pages;
            }
          }
          pg_mine = id;
        }
        const int ph0 = __shfl_sync(0xffffffffu, pg_mine, lp0 & 31);
        const int ph1 = __shfl_sync(0xffffffffu, pg_mine, (lp0 + 1) & 31);
        if (lane == 0) {
          const uint32_t R = issued;
          if (mbar_wait(bar_kv_empty(R), ((R / NS) & 1) ^ 1, abort_flag)) {
            const bool vtail = (e & 1) && jt == tail_tile;
            const uint32_t bar = vtail ? bar_vtail : bar_kv_full(R);
            mbar_arrive_expect_tx(bar, B::TILE_BYTES);
            const CUtensorMap* map = (e & 1) ? &p.tm_v : &p.tm_k;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int phys = h ? ph1 : ph0;
              const int c1 = (p.head_coord == 1) ? w.kv_head : (p.page_coord == 1 ? phys : 0);
              const int c2 = (p.head_coord == 2) ? w.kv_head : (p.page_coord == 2 ? phys : 0);
              const int c3 = (p.head_coord == 3) ? w.kv_head : (p.page_coord == 3 ? phys : 0);
#pragma unroll
              for (int c = 0; c < B::CHUNKS; ++c)
                tma_load_4d(kv_s(R) + c * B::CHUNK_BYTES + h * (B::CHUNK_BYTES / 2), map, bar, c * 64, c1, c2,
                            c3);
            }
            ++issued;
            if (vtail) tail_R = static_cast<int>(R);
            if (e == 0) {
              // a slot's Q tile is free once the last S MMA of its previous item completed
              if (w.n_kv[0] > 0) {
                ok = mbar_wait(bar_q_empty(0), (qc0 & 1) ^ 1, abort_flag);
                if (ok) {
                  load_q(0, w.head[0], w.s0 + w.qtile[0] * B::BM, bar_q);
                  ++qc0;
                }
              }
              if (ok && w.n_kv[1] > 0) {
                ok = mbar_wait(bar_q_empty(1), (qc1 & 1) ^ 1, abort_flag);
                if (ok) {
                  load_q(1, w.head[1], w.s0 + w.qtile[1] * B::BM, bar_q1);
                  ++qc1;
                }
              }
            }
          } else {
            ok = false;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      tail_R = __shfl_sync(0xffffffffu, tail_R, 0);
      if (ok && tail_R >= 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_vtail, tails & 1, abort_flag));
        if (ok) {
          // rows [Lk, end of its page) of the tile, in every 64-column chunk
          const int r0 = w.Lk - tail_tile * B::BN;
          const int r1 = ((w.Lk + kPrefillPage - 1) / kPrefillPage) * kPrefillPage - tail_tile * B::BN;
          uint4* tile = reinterpret_cast<uint4*>(smem + B::KV_OFF + (tail_R % NS) * B::TILE_BYTES);
          const int per_chunk = (r1 - r0) * 8;   // 16-byte stores per chunk
          for (int i = lane; i < B::CHUNKS * per_chunk; i += 32) {
            const int c = i / per_chunk, u = i % per_chunk;
            tile[(c * B::CHUNK_BYTES + r0 * 128) / 16 + u] = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_kv_full(tail_R));
          ++tails;
          tail_R = -1;
        }
      }
      // the next item is claimed once this one's loads are issued (see below)
      if (ok && lane == 0) next = claim();
    }
    if (lane == 0) {
      if (*abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes away
        volatile int never = 0;
        for (uint32_t i = (issued > static_cast<uint32_t>(NS) ? issued - NS : 0u); i < issued; ++i) {
          if (static_cast<int>(i) == tail_R) mbar_wait(bar_vtail, tails & 1, &never);
          else mbar_wait(bar_kv_full(i), (i / NS) & 1, &never);
        }
        if (qc0 > 0) mbar_wait(bar_q, (qc0 - 1) & 1, &never);
        if (qc1 > 0) mbar_wait(bar_q1, (qc1 - 1) & 1, &never);
      }
      __threadfence();   // this thread's counter updates precede the CTA's finish count
    }
  } else if (warp == 8) {
    // ---------------------------------------------------------------- TMA producer + scheduler
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      auto load_q = [&](int k, int h, int row0, uint32_t bar) {
        mbar_arrive_expect_tx(bar, B::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < B::CHUNKS; ++c)
          tma_load_3d(q_s + k * B::TILE_BYTES + c * B::CHUNK_BYTES, &p.tm_q, bar, c * 64, h, row0);
      };
      // Claim an item, decode it and ask L2 for its Q tiles and first K/V
      // tiles, which the TMA loads of the next item then find there.
      auto claim = [&]() -> PrefillItem {
        const int id = static_cast<int>(atomicAdd(pp.sched, 1u));
        PrefillItem w;
        if (id >= pp.total_items) {
          w.id = -1;
          return w;
        }
        w = prefill_item(p, id, B::BM, B::BN);
#pragma unroll
        for (int k = 0; k < 2; ++k)
          if (w.n_kv[k] > 0)
#pragma unroll
            for (int c = 0; c < B::CHUNKS; ++c)
              tma_prefetch_l2_3d(&p.tm_q, c * 64, w.head[k], w.s0 + w.qtile[k] * B::BM);
        const int pre = min(max(w.n_kv[0], w.n_kv[1]), 2);
        for (int j = 0; j < pre; ++j)
#pragma unroll
          for (int c = 0; c < B::CHUNKS; ++c) {
            tma_prefetch_l2_3d(&p.tm_k, c * 64, w.kv_head, w.s0 + j * B::BN);
            tma_prefetch_l2_3d(&p.tm_v, c * 64, w.kv_head, w.s0 + j * B::BN);
          }
        return w;
      };
      uint32_t issued = 0;          // ring entries issued
      int qc0 = 0, qc1 = 0;         // Q loads of each slot
      PrefillItem next = claim();
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const PrefillItem w = next;
        const int qi = n % QD;
        if (!mbar_wait(bar_item_empty(qi), ((n / QD) & 1) ^ 1, abort_flag)) break;
        queue[qi] = w;
        mbar_arrive(bar_item_full(qi));
        if (w.id < 0) break;
        const int n_max = max(w.n_kv[0], w.n_kv[1]);
        // ring entries K_0, V_0, K_1, V_1, ...; both Q tiles right after K_0
        for (int e = 0; e < 2 * n_max; ++e) {
          const uint32_t R = issued;
          if (!mbar_wait(bar_kv_empty(R), ((R / NS) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar_kv_full(R), B::TILE_BYTES);
          const CUtensorMap* map = (e & 1) ? &p.tm_v : &p.tm_k;
          const int row = w.s0 + (e >> 1) * B::BN;
#pragma unroll
          for (int c = 0; c < B::CHUNKS; ++c)
            tma_load_3d(kv_s(R) + c * B::CHUNK_BYTES, map, bar_kv_full(R), c * 64, w.kv_head, row);
          ++issued;
          if (e == 0) {
            // a slot's Q tile is free once the last S MMA of its previous item completed
            if (w.n_kv[0] > 0) {
              if (!mbar_wait(bar_q_empty(0), (qc0 & 1) ^ 1, abort_flag)) { ok = false; break; }
              load_q(0, w.head[0], w.s0 + w.qtile[0] * B::BM, bar_q);
              ++qc0;
            }
            if (w.n_kv[1] > 0) {
              if (!mbar_wait(bar_q_empty(1), (qc1 & 1) ^ 1, abort_flag)) { ok = false; break; }
              load_q(1, w.head[1], w.s0 + w.qtile[1] * B::BM, bar_q1);
              ++qc1;
            }
          }
        }
        // The next item is claimed (and its first tiles asked of L2) only once
        // every load of this one is issued, about NS ring entries before this
        // item's last MMA: a CTA holds at most one item it has not started, so
        // near the end of the launch the last items go to the CTAs that free
        // up first.
        if (ok) next = claim();
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes away
        volatile int never = 0;
        for (uint32_t i = (issued > static_cast<uint32_t>(NS) ? issued - NS : 0u); i < issued; ++i)
          mbar_wait(bar_kv_full(i), (i / NS) & 1, &never);
        if (qc0 > 0) mbar_wait(bar_q, (qc0 - 1) & 1, &never);
        if (qc1 > 0) mbar_wait(bar_q1, (qc1 - 1) & 1, &never);
      }
      __threadfence();   // this thread's counter updates precede the CTA's finish count
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_k(B::BM, B::BN) : idesc_bf16_f32(B::BM, B::BN, false);
      constexpr uint32_t idesc_pv = F8 ? idesc_f16_f32(B::BM, D, true) : idesc_bf16_f32(B::BM, D, true);
      const uint64_t q_desc = sdesc_sw128(q_s, 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(base + B::KV_OFF, 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(base + (F8 ? B::VH_OFF : B::KV_OFF), B::CHUNK_BYTES, 1024);
      auto ring_off = [&](uint32_t e) { return static_cast<uint64_t>((e % NS) * (B::TILE_BYTES >> 4)); };
      auto issue_qk = [&](int k, uint32_t R) {
        const uint64_t qd = q_desc + (k ? (B::TILE_BYTES >> 4) : 0);
        const uint64_t kd = k_desc0 + ring_off(R);
        const uint32_t d_tmem = tmem + (k ? 128u : 0u);
#pragma unroll
        for (int kk = 0; kk < D * B::ELEM / 32; ++kk) {   // 32-byte K steps
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * B::CHUNK_BYTES + (kk & 3) * 32) >> 4);
          if constexpr (F8) mma_f8_ss(d_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
          else mma_bf16_ss(d_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // V operand: ring entry R (bf16) or f16 tile vslot (E4M3)
      // keys 64h .. 64h+63 (the P columns of half h)
      auto issue_pv_half = [&](int k, uint32_t R, int vslot, bool accumulate, int h) {
        const uint32_t o_tmem = tmem + 256u + (k ? D : 0);
        const uint32_t p_tmem = tmem + (k ? 128u : 0u);
        const uint64_t vd = F8 ? v_desc0 + static_cast<uint64_t>((vslot * B::VH_TILE) >> 4)
                               : v_desc0 + ring_off(R);
#pragma unroll
        for (int kk = h * B::BN / 32; kk < (h + 1) * B::BN / 32; ++kk)
          mma_bf16_ts(o_tmem, p_tmem + kk * 8, vd + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                      (accumulate || kk > 0) ? 1u : 0u);
      };
      uint32_t ring = 0;      // first ring entry of the current item
      int qc0 = 0, qc1 = 0;   // Q tiles consumed per slot
      int t0 = 0, t1 = 0;     // key tiles done per slot before the current item
      int vcount = 0;         // f16 V tiles consumed (E4M3)
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int qi = n % QD;
        if (!mbar_wait(bar_item_full(qi), (n / QD) & 1, abort_flag)) break;
        const PrefillItem w = queue[qi];
        mbar_arrive(bar_item_empty(qi));
        if (w.id < 0) break;
        const int nk0 = w.n_kv[0], nk1 = w.n_kv[1];
        const int n_max = max(nk0, nk1);
        if (n_max == 0) continue;   // nothing loaded for an empty item
        // first scores of both slots (K_0 is entry `ring`)
        if (!mbar_wait(bar_kv_full(ring), (ring / NS) & 1, abort_flag)) break;
        if (nk0 > 0) {
          if (!mbar_wait(bar_q, qc0 & 1, abort_flag)) break;
          tc_fence_after_sync();
          issue_qk(0, ring);
          tc_commit(bar_s_full(0));
          if (nk0 == 1) tc_commit(bar_q_empty(0));
          ++qc0;
        }
        if (nk1 > 0) {
          if (!mbar_wait(bar_q1, qc1 & 1, abort_flag)) break;
          tc_fence_after_sync();
          issue_qk(1, ring);
          tc_commit(bar_s_full(1));
          if (nk1 == 1) tc_commit(bar_q_empty(1));
          ++qc1;
        }
        tc_commit(bar_kv_empty(ring));
        // One slot's step at key tile j: O_k += P_k V_j, then S_k(j+1).
        auto slot_step = [&](int k, int nk, int tb, int j, uint32_t v_R, int vslot, uint32_t k_R) -> bool {
          if (j >= nk) return true;
          // the first half of P V starts while the softmax finishes the second half
          if (!mbar_wait(bar_p_half(k), (tb + j) & 1, abort_flag)) return false;
          tc_fence_after_sync();
          issue_pv_half(k, v_R, vslot, j > 0, 0);
          if (!mbar_wait(bar_p_full(k), (tb + j) & 1, abort_flag)) return false;
          tc_fence_after_sync();
          issue_pv_half(k, v_R, vslot, true, 1);
          tc_commit(bar_o_done(k));
          if (j + 1 < nk) {
            issue_qk(k, k_R);
            tc_commit(bar_s_full(k));
            if (j + 2 == nk) tc_commit(bar_q_empty(k));   // that was the slot's last S of this item
          }
          return true;
        };
        for (int j = 0; j < n_max; ++j) {
          const uint32_t v_R = ring + 2 * j + 1, k_R = ring + 2 * j + 2;
          const int vslot = vcount & 1;
          const bool need_k = (j + 1 < nk0) || (j + 1 < nk1);
          if (F8 ? !mbar_wait(bar_vh_full(vslot), (vcount >> 1) & 1, abort_flag)
                 : !mbar_wait(bar_kv_full(v_R), (v_R / NS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (need_k && !mbar_wait(bar_kv_full(k_R), (k_R / NS) & 1, abort_flag)) { ok = false; break; }
          if (!slot_step(0, nk0, t0, j, v_R, vslot, k_R) || !slot_step(1, nk1, t1, j, v_R, vslot, k_R)) {
            ok = false;
            break;
          }
          if constexpr (F8) tc_commit(bar_vh_empty(vslot));
          else tc_commit(bar_kv_empty(v_R));
          if (need_k) tc_commit(bar_kv_empty(k_R));
          ++vcount;
        }
        ring += 2 * n_max;
        t0 += nk0;
        t1 += nk1;
      }
      tc_commit(bar_final);
      volatile int never = 0;
      mbar_wait(bar_final, 0, &never);
    }
  } else if (F8 && warp >= 10) {
    // ---------------------------------------------------------------- V converters (E4M3 -> f16)
    // Warp 10 widens keys 0-63 of V_j, warp 11 keys 64-127 (layouts as in
    // fa_prefill_pp_kernel's converter warps).
    const int half = warp - 10;
    uint32_t ring = 0;
    int vcount = 0;
    for (int n = 0;; ++n) {
      const PrefillItem w = take_item_warp(n);
      if (w.id < 0) break;
      const int n_max = max(w.n_kv[0], w.n_kv[1]);
      bool ok = true;
      for (int j = 0; j < n_max; ++j, ++vcount) {
        const uint32_t v_R = ring + 2 * j + 1;
        const int vslot = vcount & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_kv_full(v_R), (v_R / NS) & 1, abort_flag)) ||
            !__all_sync(0xffffffffu, mbar_wait(bar_vh_empty(vslot), ((vcount >> 1) & 1) ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + B::KV_OFF + (v_R % NS) * B::TILE_BYTES;
        uint8_t* dst = smem + B::VH_OFF + vslot * B::VH_TILE;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int e = lane + 32 * i;             // 0..511
          const int key = half * 64 + (e >> 3), u = e & 7, sw = key & 7;
          const uint4 b = *reinterpret_cast<const uint4*>(src + key * 128 + ((u ^ sw) << 4));
          uint4 lo4, hi4;
          e4m3x4_to_f16x4(b.x, lo4.x, lo4.y);
          e4m3x4_to_f16x4(b.y, lo4.z, lo4.w);
          e4m3x4_to_f16x4(b.z, hi4.x, hi4.y);
          e4m3x4_to_f16x4(b.w, hi4.z, hi4.w);
          const int c = u >> 2, w0 = 2 * (u & 3);
          uint8_t* row = dst + c * B::CHUNK_BYTES + key * 128;
          *reinterpret_cast<uint4*>(row + ((w0 ^ sw) << 4)) = lo4;
          *reinterpret_cast<uint4*>(row + (((w0 + 1) ^ sw) << 4)) = hi4;
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar_vh_full(vslot));
          mbar_arrive(bar_kv_empty(v_R));
        }
      }
      if (!ok) break;
      ring += 2 * n_max;
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- softmax warpgroups
    const int k = warp >> 2;                       // slot
    const int r = threadIdx.x & 127;               // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sc = tmem + lane_base + (k ? 128u : 0u);
    const uint32_t oc = tmem + lane_base + 256u + (k ? D : 0);
    int tiles = 0;                                 // key tiles of this slot before the item
    for (int n = 0;; ++n) {
      const PrefillItem w = take_item_warp(n);
      if (w.id < 0) break;
      const int nk = k ? w.n_kv[1] : w.n_kv[0];   // (k is not a compile-time index)
      if (nk == 0) continue;
      const int my_qtile = k ? w.qtile[1] : w.qtile[0];
      const int my_head = k ? w.head[1] : w.head[0];
      const int q_row = my_qtile * B::BM + r;
      // query q_row sees keys up to q_row + off (bottom-right aligned when
      // paged; off = 0 for packed K/V); key tiles past tile_last need the mask
      const int off = p.causal ? w.Lk - w.L : 0;
      const int row_last = p.causal ? min(q_row + off, w.Lk - 1) : w.Lk - 1;
      const int tile_last = p.causal ? min(my_qtile * B::BM + off, w.Lk - 1) : w.Lk - 1;
      float m_ref = 0.0f, l_sum = 0.0f;
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        const int g = tiles + j;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(k), g & 1, abort_flag))) { ok = false; break; }
        tc_fence_after_sync();
        // key tiles reaching past tile_last need the mask
        const bool masked = j * B::BN + B::BN - 1 > tile_last;
        if (!prefill_softmax_tile<D, F8>(sc, oc, j == 0, masked, row_last - j * B::BN,
                                                       p.scale_log2, m_ref, l_sum, bar_o_done(k),
                                                       (g - 1) & 1, bar_p_half(k), abort_flag)) {
          ok = false;
          break;
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full(k));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done(k), (tiles + nk - 1) & 1, abort_flag))) break;
      tc_fence_after_sync();
      const float inv_l = F8 ? p.v_scale / l_sum : 1.0f / l_sum;
      const bool valid = q_row < w.L && FA_DBG_OK(w.s0 + q_row < p.total_q && my_head < p.num_q_heads);
      __nv_bfloat16* orow = p.out + (static_cast<size_t>(w.s0 + q_row) * p.num_q_heads + my_head) * D;
      // all of O's columns in flight at once, one wait
      uint32_t o[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_x32(oc + c * 32, o[c]);
      tmem_ld_wait(o[0]);
#pragma unroll
      for (int c = 1; c < D / 32; ++c) reg_dep(o[c]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[c][2 * i]) * inv_l, __uint_as_float(o[c][2 * i + 1]) * inv_l);
        if (valid) store_o_chunk(orow + c * 32, pk, p.out_v8);
      }
      if (valid && p.lse != nullptr)
        p.lse[static_cast<size_t>(w.s0 + q_row) * p.num_q_heads + my_head] =
            (m_ref + log2f(l_sum)) * 0.69314718055994530942f;
      // O is read out: the next item's first P V may overwrite it (the
      // p_full arrival of its first tile follows this in program order)
      tc_fence_before_sync();
      tiles += nk;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, B::TMEM_COLS);
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish resets the counters for the next launch
    __threadfence();
    if (atomicAdd(pp.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(pp.sched, 0u);
      atomicExch(pp.sched + 1, 0u);
    }
  }
}

}  // namespace fa
