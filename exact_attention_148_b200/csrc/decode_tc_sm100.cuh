// Flash-Decoding split kernel on the tcgen05 tensor cores (head_dim 128).
//
// Same work split as fa_decode_split_kernel (one CTA per request, kv head and
// split of the cached context; "Flash Attention & Paged Attention", section
// "FA对decode阶段的影响"), but all G query heads that share the kv head are
// served by two small matrix products per 128-key tile, computed transposed so
// that the key dimension fills the MMA's 128 rows:
//
//   S^T (128 keys x N) = K_tile (128 x d) . Q^T (d x N)          SS, K-major
//   O^T (d x N)       += V_tile^T (d x 128) . P^T (128 x N)      SS, A MN-major
//
// N = the q_len * G (token, head) rows of the request's queries padded to NPAD
// (a multiple of 8, which an SS MMA with 128 rows accepts); with q_len > 1
// (multi-token decode) token t of the chunk sees keys up to
// cache_seqlens - q_len + t.  The CUDA cores then only run the online softmax: thread i
// of the four softmax warps owns key i of the tile (TMEM lane i of S^T) and,
// at the end, dimension i of O^T.  A K/V element is never touched by a CUDA
// core, so the loop is bound by the TMA stream, not by per-element FMAs.
//
// FP8 (E4M3) cache: K and V tiles feed kind::f8f6f4 MMAs exactly as stored.
// Q and P must then be E4M3 as well; each is carried as two E4M3 terms
// (hi = E4M3(x), lo = E4M3(x - hi)), stacked as 2*NPAD operand rows.  Q is
// scaled per head by a power of two into the E4M3 range, so each bf16 element
// (8 significant bits) is held exactly by the pair unless its residual falls
// below E4M3's normal range; P in [0, 1] (about 8 bits kept) is scaled by 256 (the running
// maximum here is exact, so P <= 1), which keeps probabilities down to 2^-14
// in E4M3's normal range.  Scores and outputs add the hi and lo columns.
//
// Roles (6 warps): warp 0 TMA producer (Q for bf16, then K and V of each
// 128-key tile: two 64-token pages through the block table, as separate ring
// items), warp 1 TMEM owner and MMA issuer, warps 2-5 softmax and epilogue.
#pragma once

#include "decode_sm100.cuh"
#include "ptx_sm100.cuh"

namespace fa {

constexpr int kDecodeTcThreads = 192;

template <bool KV8, int NPAD>
struct DecodeTcCfg {
  static_assert(NPAD == 8 || NPAD == 16, "8 or 16 padded heads per CTA");
  static constexpr int D = 128;
  static constexpr int KEYS = 128;                       // keys per tile (two pages)
  static constexpr int ELEM = KV8 ? 1 : 2;
  static constexpr int NB = KV8 ? 2 * NPAD : NPAD;       // operand rows / accumulator columns
  static constexpr int CHUNKS = D * ELEM / 128;          // 128-byte column chunks per K/V row
  static constexpr int KV_BYTES = KEYS * D * ELEM;       // one K or V tile
  // Ring of K and V tiles as separate items (K_0, V_0, K_1, ...).  With 8
  // padded rows: 96 KB for either type, two CTAs per SM hiding each other's
  // fill/drain.  With 16 the softmax of a tile takes longer and needs the
  // deeper look-ahead of a 192 KB ring (one CTA per SM); measured on B200.
  static constexpr int CTAS_PER_SM = NPAD == 8 ? 2 : 1;
  static constexpr int ITEMS = (CTAS_PER_SM == 2 ? 96 : 192) * 1024 / KV_BYTES;
  static constexpr int Q_BYTES = NB * 128 * CHUNKS;      // Q^T operand
  static constexpr int P_CHUNKS = KEYS * ELEM / 128;     // 128-byte key chunks per P^T row
  static constexpr int P_BYTES = NB * 128 * P_CHUNKS;    // one P^T operand
  static constexpr int RING_OFF = 0;
  static constexpr int Q_OFF = ITEMS * KV_BYTES;
  static constexpr int P_OFF = Q_OFF + ((Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int P_STRIDE = ((P_BYTES + 1023) / 1024) * 1024;
  static constexpr int RED_OFF = P_OFF + 2 * P_STRIDE;   // [2][NPAD][4] tile maxima
  static constexpr int SCL_OFF = RED_OFF + 2 * NPAD * 4 * 4;   // [NPAD] per-head score multipliers
  static constexpr int LRED_OFF = SCL_OFF + NPAD * 4;    // [NPAD][4] normaliser partials
  static constexpr int BAR_OFF = LRED_OFF + NPAD * 4 * 4;
  // q_full, kv_full[ITEMS], kv_empty[ITEMS], s_full[2], p_full[2], o_done[2], v_tail, final
  static constexpr int NUM_BARS = 1 + 2 * ITEMS + 8;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 128;             // S^T x2 + O^T: 3 * NB <= 96
  static_assert(3 * NB <= static_cast<int>(TMEM_COLS), "TMEM budget");
  static_assert(SMEM_BYTES <= (CTAS_PER_SM == 2 ? 113 : 227) * 1024, "shared memory per CTA");
};

__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major) {
  // c_format F32 (bit 4), a/b formats E4M3 (0), A major bit 15, N>>3, M>>4
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(int M, int N, bool a_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    static_assert(N == 32, "8, 16 or 32 columns");
    tmem_ld_x32(taddr, r);
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_n_wait(uint32_t (&r)[N]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                 "r"(r[6]), "r"(r[7])
                 : "memory");
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
  } else {
    static_assert(N == 32, "8, 16 or 32 columns");
    tmem_st_x32(taddr, r);
  }
}

// E4M3 code of x (round to nearest even, saturating at +-448), in the low
// byte (x goes to both bytes of the pair, so the pair's byte order is moot).
__device__ __forceinline__ uint32_t to_e4m3(float x) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(x), "f"(x));
  return static_cast<uint32_t>(h) & 0xFFu;
}

// Add to a barrier's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Value of the E4M3 code in the low byte of c.
__device__ __forceinline__ float from_e4m3(uint32_t c) { return e4m3_scaled<0>(c) * kTwo120; }

// Reduce N values per lane across the 32 lanes of a warp with op (max or
// add), transposed: each round keeps half of the values and adds/maxes in the
// partner's other half, so afterwards a lane holds the result for value
// index xpose32_base<N>(lane) (N < 32: replicated over 32/N lanes).
template <int N, int MASK, bool MAX>
__device__ __forceinline__ void xpose32(float* v, int lane) {
  if constexpr (MASK > 0) {
    if constexpr (N >= 2) {
      const bool upper = (lane & MASK) != 0;
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        const float send = upper ? v[k] : v[k + N / 2];
        const float keep = upper ? v[k + N / 2] : v[k];
        const float got = __shfl_xor_sync(0xffffffffu, send, MASK);
        v[k] = MAX ? fmaxf(keep, got) : keep + got;
      }
      xpose32<N / 2, MASK / 2, MAX>(v, lane);
    } else {
      const float got = __shfl_xor_sync(0xffffffffu, v[0], MASK);
      v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
      xpose32<1, MASK / 2, MAX>(v, lane);
    }
  }
}

template <int N>
__device__ __forceinline__ int xpose32_base(int lane) {
  int base = 0, n = N;
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    if (n >= 2) {
      if (lane & m) base += n / 2;
      n /= 2;
    }
  }
  return base;
}

template <bool KV8, int NPAD>
__global__ void __launch_bounds__(kDecodeTcThreads, NPAD == 8 ? 2 : 1)
    fa_decode_tc_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecodeTcCfg<KV8, NPAD>;
  constexpr int D = C::D;
  constexpr int NB = C::NB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int kv_head = blockIdx.y;
  const int b = blockIdx.z;
  const int G = p.group;                       // heads of the kv head
  const int QL = p.q_len;                      // query tokens per request
  const int R = QL * G;                        // real operand rows (<= NPAD): row = t * G + h
  const int qh0 = kv_head * G;

  int seqlen = p.cache_seqlens[b];
  if (seqlen > p.max_pages * kDecodePage || seqlen < 0) {
    if (split == 0 && threadIdx.x == 0) record_status(FA_ERR_PLAN_MISMATCH);
    seqlen = seqlen < 0 ? 0 : p.max_pages * kDecodePage;
  }
  int nsplit = (seqlen + p.chunk_tokens - 1) / p.chunk_tokens;
  if (nsplit > p.max_splits) {
    if (split == 0 && threadIdx.x == 0) record_status(FA_ERR_PLAN_MISMATCH);
    nsplit = p.max_splits;
    seqlen = p.max_splits * p.chunk_tokens;
  }
  const int nsplit_eff = nsplit > 0 ? nsplit : 1;
  if (split >= nsplit_eff) return;   // uniform; nothing initialised yet
  const int t_begin = split * p.chunk_tokens;
  const int t_end = min(seqlen, t_begin + p.chunk_tokens);
  const int page_begin = t_begin / kDecodePage;
  const int num_pg = t_end > t_begin ? (t_end - t_begin + kDecodePage - 1) / kDecodePage : 0;
  const int n_tiles = (num_pg + 1) / 2;
  const bool direct = (nsplit_eff == 1);

  // Multi-token decode: the chunk's own tokens must be in the cache.
  if (QL > 1 && seqlen < QL && split == 0 && threadIdx.x == 0) record_status(FA_ERR_PLAN_MISMATCH);
  if (n_tiles == 0) {   // empty cache: O = 0, LSE = -inf (only reachable with one split)
    for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
      const int rr = e / D;
      const size_t row = (static_cast<size_t>(b) * QL + rr / G) * p.num_q_heads + qh0 + rr % G;
      if (!FA_DBG_OK(row < static_cast<size_t>(p.batch) * QL * p.num_q_heads)) continue;
      p.out[row * D + e % D] = __float2bfloat16_rn(0.0f);
      if (e % D == 0 && p.lse != nullptr) p.lse[row] = -INFINITY;
    }
    return;
  }

  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t bar_q = bars;
  // ring item it = 2 * tile + (0: K, 1: V), slot it % ITEMS
  auto bar_kv_full = [&](int it) { return bars + 8 * (1 + it % C::ITEMS); };
  auto bar_kv_empty = [&](int it) { return bars + 8 * (1 + C::ITEMS + it % C::ITEMS); };
  auto item_par = [&](int it) { return static_cast<uint32_t>((it / C::ITEMS) & 1); };
  auto item_s = [&](int it) { return base + C::RING_OFF + (it % C::ITEMS) * C::KV_BYTES; };
  auto bar_s_full = [&](int k) { return bars + 8 * (1 + 2 * C::ITEMS + k); };
  auto bar_p_full = [&](int k) { return bars + 8 * (3 + 2 * C::ITEMS + k); };
  auto bar_o_done = [&](int k) { return bars + 8 * (5 + 2 * C::ITEMS + k); };
  const uint32_t bar_vtail = bars + 8 * (7 + 2 * C::ITEMS);
  const uint32_t bar_final = bars + 8 * (8 + 2 * C::ITEMS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, KV8 ? 4 : 1);
    for (int i = 0; i < C::ITEMS; ++i) {
      mbar_init(bar_kv_full(i), 1);
      mbar_init(bar_kv_empty(i), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s_full(k), 1);
      mbar_init(bar_p_full(k), 4);
      mbar_init(bar_o_done(k), 1);
    }
    mbar_init(bar_vtail, 1);
    mbar_init(bar_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      if constexpr (!KV8) {
        // R = q_len * G rows (token-major), 128 bytes each, per 64-column chunk;
        // rows R..NPAD-1 of the operand are never read back (their S^T
        // columns are masked and their P^T rows are zero).
        tma_prefetch_desc(&p.tm_q);
        mbar_arrive_expect_tx(bar_q, C::CHUNKS * R * 128);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_4d(base + C::Q_OFF + c * NPAD * 128, &p.tm_q, bar_q, c * 64, qh0, 0, b);
      }
    }
    const int32_t* bt_row = p.block_table + static_cast<size_t>(b) * p.max_pages + page_begin;
    // The split's last page ends inside the page only at the cache end; that
    // tile's V item lands on its own barrier, the warp zeroes its rows past
    // the cache end (0 * NaN would otherwise reach O), then marks it full.
    const int tail_tile = (t_end % kDecodePage != 0) ? n_tiles - 1 : -1;
    int pg_base = -1, pg_mine = 0, issued = 0, tail_item = -1;
    bool ok = true;
    for (int it = 0; it < 2 * n_tiles; ++it) {
      const int i = it >> 1;
      const int lp0 = 2 * i;                        // split-relative logical page
      if ((lp0 & ~31) != pg_base) {
        pg_base = lp0 & ~31;
        const int lp = pg_base + lane;
        int id = p.num_pages;                       // past the split: zero fill
        if (lp < num_pg && FA_DBG_OK(page_begin + lp < p.max_pages)) {
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
        if (mbar_wait(bar_kv_empty(it), item_par(it) ^ 1, abort_flag)) {
          const bool vtail = (it & 1) && i == tail_tile;
          const uint32_t bar = vtail ? bar_vtail : bar_kv_full(it);
          mbar_arrive_expect_tx(bar, C::KV_BYTES);
          const CUtensorMap* map = (it & 1) ? &p.tm_v : &p.tm_k;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int phys = h ? ph1 : ph0;
            const int c1 = (p.head_coord == 1) ? kv_head : (p.page_coord == 1 ? phys : 0);
            const int c2 = (p.head_coord == 2) ? kv_head : (p.page_coord == 2 ? phys : 0);
            const int c3 = (p.head_coord == 3) ? kv_head : (p.page_coord == 3 ? phys : 0);
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c)
              tma_load_4d(item_s(it) + c * (C::KEYS * 128) + h * (kDecodePage * 128), map, bar,
                          c * (128 / C::ELEM), c1, c2, c3);
          }
          ++issued;
          if (vtail) tail_item = it;
        } else {
          ok = false;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    tail_item = __shfl_sync(0xffffffffu, tail_item, 0);
    bool tail_landed = true;
    if (tail_item >= 0) {
      tail_landed = __all_sync(0xffffffffu, mbar_wait(bar_vtail, 0, abort_flag));
      if (tail_landed) {
        const int i = tail_item >> 1;
        const int r0 = t_end - (t_begin + i * C::KEYS);
        const int r1 = ((t_end + kDecodePage - 1) / kDecodePage) * kDecodePage - (t_begin + i * C::KEYS);
        uint4* tile = reinterpret_cast<uint4*>(smem + C::RING_OFF + (tail_item % C::ITEMS) * C::KV_BYTES);
        const int per_chunk = (r1 - r0) * 8;
        for (int e = lane; e < C::CHUNKS * per_chunk; e += 32) {
          const int c = e / per_chunk, w = e % per_chunk;
          tile[(c * C::KEYS * 128 + r0 * 128) / 16 + w] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_kv_full(tail_item));
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int never = 0;
      for (int it = (issued > C::ITEMS ? issued - C::ITEMS : 0); it < issued; ++it) {
        if (it == tail_item) {
          if (!tail_landed) mbar_wait(bar_vtail, 0, &never);
        } else {
          mbar_wait(bar_kv_full(it), item_par(it), &never);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = KV8 ? idesc_e4m3_f32(128, NB, false) : idesc_bf16_f32_ab(128, NB, false);
      constexpr uint32_t idesc_o = KV8 ? idesc_e4m3_f32(128, NB, true) : idesc_bf16_f32_ab(128, NB, true);
      constexpr int KSTEPS = D * C::ELEM / 32;       // 32-byte K steps over d
      constexpr int PSTEPS = C::KEYS * C::ELEM / 32; // 32-byte K steps over the keys
      auto issue_s = [&](int i) {
        const uint32_t kt = item_s(2 * i);
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((i & 1) * NB);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          // 128-byte chunk kk/4, 32 bytes into it
          const uint32_t a = kt + (kk >> 2) * (C::KEYS * 128) + (kk & 3) * 32;
          const uint32_t bq = base + C::Q_OFF + (kk >> 2) * (NB * 128) + (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(a, 16, 1024), bd = sdesc_sw128(bq, 16, 1024);
          if constexpr (KV8) mma_e4m3_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          else mma_bf16_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i) {
        const uint32_t vt = item_s(2 * i + 1);
        const uint32_t o_tmem = tmem + static_cast<uint32_t>(2 * NB);
        const uint32_t pbuf = base + C::P_OFF + (i & 1) * C::P_STRIDE;
#pragma unroll
        for (int kk = 0; kk < PSTEPS; ++kk) {
          // V^T, MN-major: 32 bytes of keys = 32 / ELEM keys per step, 128 bytes a key row;
          // the d direction crosses 128-byte chunks every KEYS * 128 bytes.
          const uint32_t a = vt + kk * (32 / C::ELEM) * 128;
          const uint32_t bp = pbuf + (kk >> 2) * (NB * 128) + (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(a, C::KEYS * 128, 1024), bd = sdesc_sw128(bp, 16, 1024);
          if constexpr (KV8) mma_e4m3_ss(o_tmem, ad, bd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
          else mma_bf16_ss(o_tmem, ad, bd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        }
      };
      // S_0, S_1, then per tile j: PV_j, S_{j+2}.  A K item is released
      // once its S MMAs complete, a V item once its PV MMAs complete.
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      for (int i = 0; ok && i < 2 && i < n_tiles; ++i) {
        if (!mbar_wait(bar_kv_full(2 * i), item_par(2 * i), abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        issue_s(i);
        tc_commit(bar_s_full(i & 1));
        tc_commit(bar_kv_empty(2 * i));
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (!mbar_wait(bar_p_full(j & 1), (j >> 1) & 1, abort_flag)) break;
        if (!mbar_wait(bar_kv_full(2 * j + 1), item_par(2 * j + 1), abort_flag)) break;
        tc_fence_after_sync();
        issue_pv(j);
        tc_commit(bar_o_done(j & 1));
        tc_commit(bar_kv_empty(2 * j + 1));
        const int n = j + 2;
        if (n < n_tiles) {
          if (!mbar_wait(bar_kv_full(2 * n), item_par(2 * n), abort_flag)) break;
          tc_fence_after_sync();
          issue_s(n);
          tc_commit(bar_s_full(n & 1));
          tc_commit(bar_kv_empty(2 * n));
        }
      }
      tc_commit(bar_final);
      volatile int never = 0;
      mbar_wait(bar_final, 0, &never);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;                // key of the tile / dimension of O^T
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + C::RED_OFF);    // [2][NPAD][4]
    float* scl = reinterpret_cast<float*>(smem + C::SCL_OFF);    // [NPAD]
    float* lred = reinterpret_cast<float*>(smem + C::LRED_OFF);  // [NPAD][4]
    auto softmax_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };

    if constexpr (KV8) {
      // Q^T operand: heads h = quad, quad + 4, ...; lane holds d = 4 lane .. 4 lane + 3.
      uint8_t* qs = smem + C::Q_OFF;
      for (int h = quad; h < NPAD; h += 4) {      // h = operand row t * G + head
        uint32_t hi = 0, lo = 0;
        float sq = 1.0f;
        const size_t qrow = (static_cast<size_t>(b) * QL + h / G) * p.num_q_heads + qh0 + h % G;
        if (h < R && FA_DBG_OK(qrow < static_cast<size_t>(p.batch) * QL * p.num_q_heads)) {
          const uint2 u = *reinterpret_cast<const uint2*>(p.q + qrow * D + 4 * lane);
          const float x[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                              __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
          float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
          for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
          // A power-of-two scale keeps q / sq an exact 8-bit (bf16) significand,
          // which hi (4 bits) + lo (4 bits) then hold exactly: amax / 448
          // rounded up to a power of two (exponent field bumped unless the
          // mantissa is zero).
          const uint32_t tb = __float_as_uint(amax * (1.0f / 448.0f));
          sq = amax > 0.0f ? __uint_as_float((tb + 0x007FFFFFu) & 0x7F800000u) : 1.0f;
          const float inv = 1.0f / sq;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float y = x[e] * inv;
            const uint32_t ch = to_e4m3(y);
            const uint32_t cl = to_e4m3(y - from_e4m3(ch));
            hi |= ch << (8 * e);
            lo |= cl << (8 * e);
          }
        }
        const int u = lane >> 2;                    // 16-byte unit of d = 4 lane
        *reinterpret_cast<uint32_t*>(qs + h * 128 + ((u ^ (h & 7)) << 4) + (lane & 3) * 4) = hi;
        const int hl = NPAD + h;
        *reinterpret_cast<uint32_t*>(qs + hl * 128 + ((u ^ (hl & 7)) << 4) + (lane & 3) * 4) = lo;
        if (lane == 0) scl[h] = sq * p.scale_log2;
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q);
    } else {
      if (quad == 0 && lane < NPAD) scl[lane] = p.scale_log2;
    }
    softmax_sync();
    float c[NPAD], m[NPAD], l[NPAD];
    int lim[NPAD];                 // last visible key of each row (token t of the chunk)
#pragma unroll
    for (int h = 0; h < NPAD; ++h) {
      c[h] = scl[h];
      m[h] = -INFINITY;
      l[h] = 0.0f;
      lim[h] = h < R ? seqlen - QL + h / G : -1;
    }

    // Every softmax warp passes the named barrier once per tile and once in
    // the epilogue, also after a failed wait (it then skips the work), so a
    // timeout in one warp cannot leave the others waiting on the barrier.
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_s_full(j & 1), (j >> 1) & 1, abort_flag));
      float s[NPAD];
      if (ok) {
        tc_fence_after_sync();
        uint32_t sr[NB];
        tmem_ld_n<NB>(tmem + lane_base + static_cast<uint32_t>((j & 1) * NB), sr);
        tmem_ld_n_wait<NB>(sr);
        const int key = t_begin + j * C::KEYS + r;
        const bool valid = key < t_end;
#pragma unroll
        for (int h = 0; h < NPAD; ++h) {
          const float raw = KV8 ? __uint_as_float(sr[h]) + __uint_as_float(sr[NPAD + h])
                                : __uint_as_float(sr[h]);
          s[h] = (valid && key <= lim[h]) ? raw * c[h] : -INFINITY;
        }
      } else {
#pragma unroll
        for (int h = 0; h < NPAD; ++h) s[h] = -INFINITY;
      }
      // tile maximum of every head over the 128 keys
      float t[NPAD];
#pragma unroll
      for (int h = 0; h < NPAD; ++h) t[h] = s[h];
      xpose32<NPAD, 16, true>(t, lane);
      float* rb = red + (j & 1) * NPAD * 4;
      if ((lane & (32 / NPAD - 1)) == 0) rb[xpose32_base<NPAD>(lane) * 4 + quad] = t[0];
      softmax_sync();
      bool grew = false;
      float alpha[NPAD], mu[NPAD];
#pragma unroll
      for (int h = 0; h < NPAD; ++h) {
        const float4 w = *reinterpret_cast<const float4*>(rb + h * 4);
        const float mt = fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w));
        const float mn = fmaxf(m[h], mt);
        grew |= (mn > m[h]) && j > 0;
        alpha[h] = (j > 0 && mn > m[h]) ? ex2_approx(m[h] - mn) : 1.0f;
        m[h] = mn;
        mu[h] = (mn == -INFINITY) ? 0.0f : mn;
      }
      // P^T buffer j&1 was last read by PV(j-2)
      if (j >= 2) ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done(j & 1), ((j - 2) >> 1) & 1, abort_flag));
      if (!ok) continue;
      uint8_t* pb = smem + C::P_OFF + (j & 1) * C::P_STRIDE;
#pragma unroll
      for (int h = 0; h < NPAD; ++h) {
        const float pr = ex2_approx(s[h] - mu[h]);
        l[h] = l[h] * alpha[h] + pr;
        if constexpr (KV8) {
          const float y = pr * 256.0f;
          const uint32_t ch = to_e4m3(y);
          const uint32_t cl = to_e4m3(y - from_e4m3(ch));
          const int u = r >> 4;
          pb[h * 128 + ((u ^ (h & 7)) << 4) + (r & 15)] = static_cast<uint8_t>(ch);
          const int hl = NPAD + h;
          pb[hl * 128 + ((u ^ (hl & 7)) << 4) + (r & 15)] = static_cast<uint8_t>(cl);
        } else {
          const int ck = r >> 6, byte = (r & 63) * 2, u = byte >> 4;
          *reinterpret_cast<__nv_bfloat16*>(pb + ck * (NPAD * 128) + h * 128 + ((u ^ (h & 7)) << 4) +
                                            (byte & 15)) = __float2bfloat16_rn(pr);
        }
      }
      fence_async_shared();
      if (grew) {
        // O^T still holds the sum over tiles < j against the old maxima: once
        // PV(j-1) has landed, scale column h (and its lo twin) by alpha[h].
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag));
        if (!ok) continue;
        tc_fence_after_sync();
        uint32_t o[NB];
        tmem_ld_n<NB>(tmem + lane_base + static_cast<uint32_t>(2 * NB), o);
        tmem_ld_n_wait<NB>(o);
#pragma unroll
        for (int h = 0; h < NPAD; ++h) {
          o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
          if constexpr (KV8) o[NPAD + h] = __float_as_uint(__uint_as_float(o[NPAD + h]) * alpha[h]);
        }
        tmem_st_n<NB>(tmem + lane_base + static_cast<uint32_t>(2 * NB), o);
        tmem_st_wait();
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full(j & 1));
    }

    // ---- epilogue: normalisers over the 128 keys, then O^T row r = dimension r
    xpose32<NPAD, 16, false>(l, lane);
    if ((lane & (32 / NPAD - 1)) == 0) lred[xpose32_base<NPAD>(lane) * 4 + quad] = l[0];
    softmax_sync();
    const int jl = n_tiles - 1;
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done(jl & 1), (jl >> 1) & 1, abort_flag))) {
      tc_fence_after_sync();
      uint32_t o[NB];
      tmem_ld_n<NB>(tmem + lane_base + static_cast<uint32_t>(2 * NB), o);
      tmem_ld_n_wait<NB>(o);
#pragma unroll
      for (int h = 0; h < NPAD; ++h) {
        if (h >= R) continue;
        const float4 w = *reinterpret_cast<const float4*>(lred + h * 4);
        const float lsum = (w.x + w.y) + (w.z + w.w);
        float ov = KV8 ? (__uint_as_float(o[h]) + __uint_as_float(o[NPAD + h])) * (p.v_scale * (1.0f / 256.0f))
                       : __uint_as_float(o[h]);
        ov = lsum > 0.0f ? ov / lsum : 0.0f;
        const float lse_v = (lsum > 0.0f) ? (m[h] + log2f(lsum)) * 0.69314718055994530942f : -INFINITY;
        const size_t row = (static_cast<size_t>(b) * QL + h / G) * p.num_q_heads + qh0 + h % G;
        const size_t rows = static_cast<size_t>(p.batch) * QL * p.num_q_heads;
        if (direct) {
          if (FA_DBG_OK(row < rows)) {
            p.out[row * D + r] = __float2bfloat16_rn(ov);
            if (r == 0 && p.lse != nullptr) p.lse[row] = lse_v;
          }
        } else {
          const size_t srow = static_cast<size_t>(split) * rows + row;
          if (FA_DBG_OK(srow < static_cast<size_t>(p.max_splits) * rows)) {
            p.ws_o[srow * D + r] = ov;
            if (r == 0) p.ws_lse[srow] = lse_v;
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
