// Ping-pong exact-attention prefill for sm_100a: two 128-row query tiles per
// CTA share every K/V tile, and two softmax warpgroups take turns with the
// tensor core.
//
// Roles (10 warps):
//   warps 0-3  softmax + epilogue of slot 0 (thread r owns TMEM lane r)
//   warps 4-7  softmax + epilogue of slot 1
//   warp  8    TMA producer: both Q tiles once, then K_0, V_0, K_1, V_1, ...
//              through one ring of NS shared-memory slots
//   warp  9    tcgen05 MMA issuer, order per key tile j:
//                PV_0(j), S_0(j+1), PV_1(j), S_1(j+1)
//              so the tensor core computes one slot's P V and next scores
//              while the other slot's softmax warpgroup exponentiates.
// A slot is two query heads of one kv head at the same rows when the GQA
// group is even, otherwise two consecutive 128-row tiles of one head; either
// way both slots read the same K/V tiles, which are loaded once per CTA.
//
// The per-tile math is the tiling + online softmax of cloud.baidu.com
// "FasterTransformer与FlashAttention的联系与区别", section 三 (load a K/V block, score
// it, update running max and normaliser, accumulate the output), on tcgen05
// tensor cores with accumulators in tensor memory; nothing of size N x N
// reaches HBM.  S lives in TMEM, P (bf16) is written over S and fed to the PV
// MMA straight from TMEM (TS form, V as the MN-major B operand in SMEM),
// base-2 exponentials with a reference maximum that is only raised when a tile
// exceeds it by more than 8 (a factor 256), which keeps O / l exact while
// skipping most O rescales.
//
// Exponentials go to the MUFU unit (ex2.approx), whose 16 results per clock
// per SM take as long for a 128 x 128 tile as its two MMAs.  (Moving a share
// of them to a polynomial on the FMA pipes, or deferring the row maximum,
// measured slower on B200 in every form tried.)

#pragma once

#include "ptx_sm100.cuh"

namespace fa {

constexpr int kPrefillMaxGroups = 2048;  // (sequence, kv head) groups per launch
constexpr float kRescaleThreshold = 8.0f;

// Work order.  CTAs are launched in groups, one group per (sequence, kv head):
// groups of longer sequences first; inside a group the q tiles go heaviest
// first and the Hq/Hkv query heads that share the kv head are adjacent.  So at
// any moment only a few heads' K/V are being read and re-reads hit L2, and the
// block scheduler's greedy fill ends on light tiles.
//
// Paged form (chunked prefill): K/V come from a page pool through block_table
// instead of being packed like Q.  Request b's cache holds cache_seqlens[b]
// keys, its q_len queries are the last q_len of them, and a causal query i
// sees keys up to position cache_seqlens[b] - q_len + i.
struct PrefillParams {
  CUtensorMap tm_q;   // 3-D {d, Hq, T}, box {64, 1, 128}, 128B swizzle
  CUtensorMap tm_k;   // packed: 3-D {d, Hkv, T}; paged: 4-D over the pool, box of
  CUtensorMap tm_v;   //   64 columns x one 64-token page, 128B swizzle
  __nv_bfloat16* out;        // [T, Hq, d]
  float* lse;                // [T, Hq] or null
  const int32_t* cu_seqlens; // [B+1] query offsets, or null: one sequence of uniform_q_len
  const int32_t* block_table;    // paged: [B, max_pages]
  const int32_t* cache_seqlens;  // paged: [B] keys per request, or null: uniform_k_len
  int uniform_q_len;
  int uniform_k_len;
  // Key-range splits (full attention only): the key tiles of every q tile are
  // cut into kv_splits ranges of kv_split_tiles; each range's normalised O and
  // LSE go to part_o [kv_splits, total_q, Hq, d] / part_lse [kv_splits, total_q, Hq]
  // (fp32) for an LSE merge.  part_o null: bf16 out / lse as usual (kv_splits 1).
  int kv_splits;
  int kv_split_tiles;
  int total_q;
  float* part_o;
  float* part_lse;
  float v_scale;             // E4M3 inputs: V dequantisation scale
  int max_pages;
  int num_pages;
  int head_coord;            // paged: tensor-map dimension (1..3) of the kv head
  int page_coord;            // paged: tensor-map dimension (1..3) of the page id
  int num_q_heads;
  int out_v8;                // out is 32-byte aligned: O rows go out in 32-byte stores
  int batch;                 // sequences (rows of cu_seqlens - 1, of block_table)
  int group;                 // Hq / Hkv
  int causal;
  float scale_log2;          // scale * log2(e)
  int num_groups;
  int group_start[kPrefillMaxGroups + 1];   // first CTA of each group (+ total)
  uint32_t group_id[kPrefillMaxGroups];     // (sequence << 16) | kv head
};

constexpr int kPrefillPPThreads = 320;

// F8: Q, K and V are E4M3 bytes (one scale per tensor).  S = Q K^T runs as a
// kind::f8f6f4 MMA on them as stored (exact products, half the tensor time of
// bf16); P is kept as f16 and V is widened to f16 in shared memory by two
// converter warps (E4M3 -> f16 is exact), so P V stays a kind::f16 MMA and
// the softmax does no more work than with bf16 inputs.
template <int D, bool F8 = false>
struct PrefillPPCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(!F8 || D == 128, "E4M3 inputs: head_dim 128");
  static constexpr int ELEM = F8 ? 1 : 2;
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int CHUNKS = D * ELEM / 128;            // 128-byte column chunks of a row
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;
  static constexpr int NS = F8 ? 8 : (D == 128) ? 5 : 8;   // K/V ring slots
  static constexpr int Q_OFF = 0;                          // two Q tiles
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int VH_OFF = KV_OFF + NS * TILE_BYTES;  // F8: two f16 V tiles (2 chunks each)
  static constexpr int VH_TILE = 2 * CHUNK_BYTES;
  static constexpr int BAR_OFF = VH_OFF + (F8 ? 2 * VH_TILE : 0);
  // q_full (slot 0), kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_done[2], final, v_tail,
  // q_full (slot 1), F8: vh_full[2], vh_empty[2]; then p_half[2]
  static constexpr int P_HALF_BAR = 10 + 2 * NS + (F8 ? 4 : 0);
  static constexpr int NUM_BARS = P_HALF_BAR + 2;
  static constexpr int THREADS = F8 ? 384 : 320;           // F8: + two converter warps
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
};

// Three-input maximum (sm_100 max.f32 with three sources).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__host__ __device__ constexpr uint32_t idesc_e4m3_k(int M, int N) {
  // F32 accumulate, A and B E4M3 (format 0), both K-major
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool b_mn_major) {
  // F32 accumulate, A and B f16 (format 0)
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four E4M3 bytes (low byte first) -> two f16x2 words (exact).
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(w));
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

constexpr int kPrefillPage = 64;

// Online softmax of one 128 x 128 score tile for a slot's 128 rows (thread =
// row = TMEM lane of its warpgroup): read S (fp32, columns sc .. sc+127),
// write P (bf16, or f16 with E4M3 inputs) over S's first 64 columns, and
// update the row's reference maximum m_ref (base 2, scale folded in) and
// normaliser l_sum.  masked (the same for the whole tile): some row of the
// tile has keys past its last visible one, lim: this row's last visible
// column.  first: the row's first tile.  The reference maximum is raised only
// when the tile's maximum exceeds it by more than kRescaleThreshold; then O
// (columns oc ..) is rescaled once the previous P V has landed (o_done,
// parity o_parity).  Returns false when a wait gave up.
// 32 bf16 columns of one O row (64 bytes): two 32-byte stores (whole L2
// sectors) when the output is 32-byte aligned, else four 16-byte stores.
__device__ __forceinline__ void store_o_chunk(__nv_bfloat16* dst, const uint32_t (&pk)[16], int v8) {
  if (v8) {
    st_global_v8(dst, pk);
    st_global_v8(dst + 16, pk + 8);
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v) d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
  }
}

template <int D, bool F8>
__device__ __forceinline__ bool prefill_softmax_tile(uint32_t sc, uint32_t oc, bool first, bool masked,
                                                     int lim, float scale_log2, float& m_ref,
                                                     float& l_sum, uint32_t bar_o_done,
                                                     uint32_t o_parity, uint32_t bar_p_half,
                                                     volatile int* abort_flag) {
  uint32_t s[4][32];
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_x32(sc + c * 32, s[c]);
  tmem_ld_wait(s[0]);
  reg_dep(s[1]);
  reg_dep(s[2]);
  reg_dep(s[3]);
  if (masked) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c * 32 + i > lim) s[c][i] = __float_as_uint(-INFINITY);
  }
  // row maximum: eight independent 3-input-max chains of 16 columns, then a tree
  float mx[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const uint32_t* v = &s[h >> 1][(h & 1) * 16];
    float m = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
    for (int i = 3; i < 15; i += 2) m = fmax3(m, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
    mx[h] = fmaxf(m, __uint_as_float(v[15]));
  }
  const float rmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
  const float m_tile = rmax * scale_log2;
  float alpha = 1.0f;
  bool rescale = false;
  if (first) {
    m_ref = (m_tile == -INFINITY) ? 0.0f : m_tile;
  } else {
    const bool need = m_tile > m_ref + kRescaleThreshold;
    rescale = __any_sync(0xffffffffu, need);
    if (need) {
      alpha = ex2_approx(m_ref - m_tile);
      m_ref = m_tile;
    }
  }
  // x = s * scale * log2(e) - m on the packed f32x2 FMA pipe; P chunk c (16
  // packed columns) lands on S columns already in registers.  After the first
  // two chunks (keys 0-63) the warp arrives on p_half, so the first half of
  // P V can start while the second half is exponentiated.
  const float2 scale2 = make_float2(scale_log2, scale_log2);
  const float2 neg_m2 = make_float2(-m_ref, -m_ref);
  float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                  make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 x = __ffma2_rn(
          make_float2(__uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1])), scale2, neg_m2);
      const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      ps[i & 3].x += e.x;   // (packed f32x2 adds here cost registers: spills)
      ps[i & 3].y += e.y;
      pk[i] = F8 ? pack_f16x2(e.x, e.y) : pack_bf16x2(e.x, e.y);
    }
    tmem_st_x16(sc + c * 16, pk);
    if (c == 1) {
      if (rescale) {
        // O holds the P V of earlier tiles against the old reference: scale
        // it by alpha (1 on rows that kept their maximum) before any of this
        // tile's P V.  S(j) completing implies the previous P V did (one
        // thread issues both, in order), so this wait ends at once.
        if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done, o_parity, abort_flag))) return false;
        tc_fence_after_sync();
#pragma unroll
        for (int oc32 = 0; oc32 < D / 32; ++oc32) {
          uint32_t o[32];
          tmem_ld_x32(oc + oc32 * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st_x32(oc + oc32 * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bar_p_half);
    }
  }
  l_sum = l_sum * alpha + (((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) +
                           ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y)));
  return true;
}

template <int D, bool PAGED, bool F8 = false>
__global__ void __launch_bounds__(PrefillPPCfg<D, F8>::THREADS, 1)
    fa_prefill_pp_kernel(const __grid_constant__ PrefillParams p) {
  static_assert(!(F8 && PAGED), "E4M3 inputs: packed K/V only");
  using C = PrefillPPCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- CTA -> (sequence, kv head, two query slots)
  const int bid = static_cast<int>(blockIdx.x);
  int lo = 0, hi = p.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.group_start[mid] <= bid) lo = mid; else hi = mid - 1;
  }
  const int seq = static_cast<int>(p.group_id[lo] >> 16);
  const int kv_head = static_cast<int>(p.group_id[lo] & 0xFFFFu);
  if (!FA_DBG_OK(seq < p.batch)) return;   // uniform in the CTA; nothing allocated yet
  int rank = bid - p.group_start[lo];
  const int s0 = p.cu_seqlens != nullptr ? p.cu_seqlens[seq] : 0;
  const int L = p.cu_seqlens != nullptr ? p.cu_seqlens[seq + 1] - s0 : p.uniform_q_len;   // queries
  const int n_qtiles = (L >= 1 && L <= p.total_q) ? (L + C::BM - 1) / C::BM : 0;
  int Lk = L;                                   // keys
  if constexpr (PAGED) {
    Lk = p.cache_seqlens != nullptr ? p.cache_seqlens[seq] : p.uniform_k_len;
    // A causal chunk's own tokens are among the keys (k_len >= q_len); full
    // attention (the shared prefix of a cascade) may have fewer keys than queries.
    const int cap = p.max_pages * kPrefillPage;
    if ((p.causal && Lk < L) || Lk > cap || Lk < 0) {
      if (rank == 0 && threadIdx.x == 0) record_status(FA_ERR_PLAN_MISMATCH);
      Lk = min(max(Lk, p.causal ? L : 0), cap);
    }
  }
  const int G = p.group;
  {
    // The device offsets must describe what the host planned: rows inside the
    // T packed ones, and this group's CTA count (cu_seqlens_dev must equal
    // cu_seqlens_host).  Otherwise record it and leave (uniform in the CTA).
    const bool in_rows = s0 >= 0 && L >= 1 && s0 <= p.total_q - L;
    const int nq = in_rows ? n_qtiles : 0;
    const int derived = (((G & 1) == 0) ? nq * (G >> 1) : ((nq + 1) >> 1) * G) * max(p.kv_splits, 1);
    if (!in_rows || derived != p.group_start[lo + 1] - p.group_start[lo]) {
      if (rank == 0 && threadIdx.x == 0) record_status(FA_ERR_PLAN_MISMATCH);
      return;
    }
  }
  const int off = p.causal ? Lk - L : 0;        // query i sits at key position i + off
  const int n_ktiles_all = (Lk + C::BN - 1) / C::BN;
  // Key-range split: a group holds kv_splits copies of its q-tile CTAs, one
  // per range of kv_split_tiles key tiles (tiles [kt0, n_ktiles)).
  int kt0 = 0, n_ktiles = n_ktiles_all, split = 0;
  if (p.kv_splits > 1) {
    const int base_ctas = ((G & 1) == 0) ? n_qtiles * (G >> 1) : ((n_qtiles + 1) >> 1) * G;
    split = rank / base_ctas;
    rank -= split * base_ctas;
    kt0 = split * p.kv_split_tiles;
    n_ktiles = min(n_ktiles_all, kt0 + p.kv_split_tiles);
  }
  int qtile[2], head[2];
  if ((G & 1) == 0) {            // two heads of the group, same rows
    const int half = G >> 1;
    const int t = n_qtiles - 1 - rank / half;
    const int hp = rank % half;
    qtile[0] = qtile[1] = t;
    head[0] = kv_head * G + 2 * hp;
    head[1] = head[0] + 1;
  } else {                        // one head, two consecutive row tiles
    const int npairs = (n_qtiles + 1) >> 1;
    const int pr = npairs - 1 - rank / G;
    qtile[0] = 2 * pr;
    qtile[1] = 2 * pr + 1;
    head[0] = head[1] = kv_head * G + rank % G;
  }
  int n_kv[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool active = qtile[k] >= 0 && qtile[k] < n_qtiles;
    n_kv[k] = !active ? 0
                      : (p.causal ? min(n_ktiles, (qtile[k] * C::BM + C::BM - 1 + off) / C::BN + 1)
                                  : n_ktiles) - kt0;
    if (n_kv[k] < 0) n_kv[k] = 0;
  }
  if (n_kv[0] == 0 && n_kv[1] == 0) return;   // uniform; nothing allocated yet
  const int n_max = max(n_kv[0], n_kv[1]);

  const uint32_t q_s = base + C::Q_OFF;
  auto kv_s = [&](int item) { return base + C::KV_OFF + (item % C::NS) * C::TILE_BYTES; };
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t bar_q = bars;
  auto bar_kv_full = [&](int item) { return bars + 8 * (1 + item % C::NS); };
  auto bar_kv_empty = [&](int item) { return bars + 8 * (1 + C::NS + item % C::NS); };
  auto bar_s_full = [&](int k) { return bars + 8 * (1 + 2 * C::NS + k); };
  auto bar_p_full = [&](int k) { return bars + 8 * (3 + 2 * C::NS + k); };
  auto bar_o_done = [&](int k) { return bars + 8 * (5 + 2 * C::NS + k); };
  const uint32_t bar_final = bars + 8 * (7 + 2 * C::NS);
  const uint32_t bar_vtail = bars + 8 * (8 + 2 * C::NS);
  const uint32_t bar_q1 = bars + 8 * (9 + 2 * C::NS);   // slot 1's Q tile
  auto bar_vh_full = [&](int sl) { return bars + 8 * (10 + 2 * C::NS + sl); };
  auto bar_vh_empty = [&](int sl) { return bars + 8 * (12 + 2 * C::NS + sl); };
  auto bar_p_half = [&](int k) { return bars + 8 * (C::P_HALF_BAR + k); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar_kv_full(i), 1);
      // F8: the V tiles (odd items, odd slots since NS is even) are released
      // by the two converter warps, the K tiles by the MMA issuer
      mbar_init(bar_kv_empty(i), (F8 && (i & 1)) ? 2 : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s_full(k), 1);
      mbar_init(bar_p_full(k), 4);
      mbar_init(bar_p_half(k), 4);
      mbar_init(bar_o_done(k), 1);
      if constexpr (F8) {
        mbar_init(bar_vh_full(k), 2);
        mbar_init(bar_vh_empty(k), 1);
      }
    }
    mbar_init(bar_final, 1);
    mbar_init(bar_vtail, 1);
    mbar_init(bar_q1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (PAGED && warp == 8) {
    // ------------------------------------------------- TMA producer, paged K/V
    // Key tile jt is logical pages 2jt and 2jt+1; their physical ids are read
    // 32 at a time by the whole warp.  A page past the cache end (or an id
    // outside the pool, which is also recorded) is loaded from page index
    // num_pages, i.e. out of the tensor map's bounds, which TMA fills with
    // zeros without touching memory.  The cache's last page may end inside
    // the page: its slots past the end hold whatever the pool had, so the V
    // tile holding it lands on its own barrier, the warp zeroes those rows
    // (0 * NaN would otherwise reach O through P V), and only then marks the
    // tile full.  That tile is always the last one loaded.
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      // slot 0's Q first (its first S needs only Q0 and K0); slot 1's Q
      // follows K0 in the loop below
      if (n_kv[0] > 0) {
        mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(q_s + c * C::CHUNK_BYTES, &p.tm_q, bar_q, c * 64, head[0], s0 + qtile[0] * C::BM);
      }
    }
    auto load_q1 = [&] {
      if (lane == 0 && n_kv[1] > 0) {
        mbar_arrive_expect_tx(bar_q1, C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(q_s + C::TILE_BYTES + c * C::CHUNK_BYTES, &p.tm_q, bar_q1, c * 64, head[1],
                      s0 + qtile[1] * C::BM);
      }
    };
    const int32_t* bt_row = p.block_table + static_cast<size_t>(seq) * p.max_pages;
    const int tail_tile = (Lk % kPrefillPage != 0) ? (Lk - 1) / C::BN - kt0 : -1;   // split-relative
    int pg_base = -1, pg_mine = 0, issued = 0, tail_item = -1;
    bool ok = true;
    for (int item = 0; item < 2 * n_max; ++item) {
      const int jt = item >> 1;                       // split-relative key tile
      const int lp0 = 2 * (kt0 + jt);
      if ((lp0 & ~31) != pg_base) {
        pg_base = lp0 & ~31;
        const int lp = pg_base + lane;
        int id = p.num_pages;
        if (lp * kPrefillPage < Lk && FA_DBG_OK(lp < p.max_pages)) {
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
        if (mbar_wait(bar_kv_empty(item), ((item / C::NS) & 1) ^ 1, abort_flag)) {
          const bool vtail = (item & 1) && jt == tail_tile;
          const uint32_t bar = vtail ? bar_vtail : bar_kv_full(item);
          mbar_arrive_expect_tx(bar, C::TILE_BYTES);
          const CUtensorMap* map = (item & 1) ? &p.tm_v : &p.tm_k;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int phys = h ? ph1 : ph0;
            const int c1 = (p.head_coord == 1) ? kv_head : (p.page_coord == 1 ? phys : 0);
            const int c2 = (p.head_coord == 2) ? kv_head : (p.page_coord == 2 ? phys : 0);
            const int c3 = (p.head_coord == 3) ? kv_head : (p.page_coord == 3 ? phys : 0);
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c)
              tma_load_4d(kv_s(item) + c * C::CHUNK_BYTES + h * (C::CHUNK_BYTES / 2), map, bar,
                          c * 64, c1, c2, c3);
          }
          ++issued;
          if (vtail) tail_item = item;
        } else {
          ok = false;
        }
      }
      if (item == 0) load_q1();
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    tail_item = __shfl_sync(0xffffffffu, tail_item, 0);
    bool tail_landed = true;
    if (tail_item >= 0) {
      tail_landed = __all_sync(0xffffffffu, mbar_wait(bar_vtail, 0, abort_flag));
      if (tail_landed) {
        // rows [Lk, end of its page) of the tile, in every 64-column chunk
        const int r0 = Lk - (kt0 + (tail_item >> 1)) * C::BN;
        const int r1 = ((Lk + kPrefillPage - 1) / kPrefillPage) * kPrefillPage - (kt0 + (tail_item >> 1)) * C::BN;
        uint4* tile = reinterpret_cast<uint4*>(smem + C::KV_OFF + (tail_item % C::NS) * C::TILE_BYTES);
        const int per_chunk = (r1 - r0) * 8;          // 16-byte stores per chunk
        for (int e = lane; e < C::CHUNKS * per_chunk; e += 32) {
          const int c = e / per_chunk, w = e % per_chunk;
          tile[(c * C::CHUNK_BYTES + r0 * 128) / 16 + w] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_kv_full(tail_item));
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int never = 0;
      for (int i = (issued > C::NS ? issued - C::NS : 0); i < issued; ++i) {
        if (i == tail_item) {
          if (!tail_landed) mbar_wait(bar_vtail, 0, &never);
        } else {
          mbar_wait(bar_kv_full(i), (i / C::NS) & 1, &never);
        }
      }
    }
  } else if (warp == 8) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      // slot 0's Q, then K0, then slot 1's Q: the first S needs only Q0 and K0
      auto load_q = [&](int k, int h, int t, uint32_t bar) {
        mbar_arrive_expect_tx(bar, C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(q_s + k * C::TILE_BYTES + c * C::CHUNK_BYTES, &p.tm_q, bar, c * 64, h,
                      s0 + t * C::BM);
      };
      if (n_kv[0] > 0) load_q(0, head[0], qtile[0], bar_q);
      int issued = 0;
      for (int item = 0; item < 2 * n_max; ++item) {
        if (!mbar_wait(bar_kv_empty(item), ((item / C::NS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_kv_full(item), C::TILE_BYTES);
        const CUtensorMap* map = (item & 1) ? &p.tm_v : &p.tm_k;
        const int row = s0 + (kt0 + (item >> 1)) * C::BN;
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(kv_s(item) + c * C::CHUNK_BYTES, map, bar_kv_full(item), c * 64, kv_head, row);
        ++issued;
        if (item == 0 && n_kv[1] > 0) load_q(1, head[1], qtile[1], bar_q1);
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int i = (issued > C::NS ? issued - C::NS : 0); i < issued; ++i)
          mbar_wait(bar_kv_full(i), (i / C::NS) & 1, &never);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_k(C::BM, C::BN) : idesc_bf16_f32(C::BM, C::BN, false);
      constexpr uint32_t idesc_pv = F8 ? idesc_f16_f32(C::BM, D, true) : idesc_bf16_f32(C::BM, D, true);
      // k is always a literal below, so per-slot values stay in registers.
      // This thread's issue rate is on the per-tile critical path (it shares
      // its SMSP with two softmax warps), so descriptors are built once and
      // each MMA only adds a compile-time offset (address field in 16-byte
      // units; no carry leaves the 14-bit field inside shared memory).
      const uint64_t q_desc = sdesc_sw128(q_s, 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(base + C::KV_OFF, 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(base + (F8 ? C::VH_OFF : C::KV_OFF), C::CHUNK_BYTES, 1024);
      auto ring_off = [&](int item) { return static_cast<uint64_t>((item % C::NS) * (C::TILE_BYTES >> 4)); };
      auto issue_qk = [&](int k, int item) {
        const uint64_t qd = q_desc + (k ? (C::TILE_BYTES >> 4) : 0);
        const uint64_t kd = k_desc0 + ring_off(item);
        const uint32_t d_tmem = tmem + (k ? 128u : 0u);
#pragma unroll
        for (int kk = 0; kk < D * C::ELEM / 32; ++kk) {   // 32-byte K steps
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4);
          if constexpr (F8) mma_f8_ss(d_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
          else mma_bf16_ss(d_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_k += P_k V over keys 64h .. 64h+63 (the P columns of half h)
      auto issue_pv_half = [&](int k, int item, bool accumulate, int h) {
        const uint32_t o_tmem = tmem + 256u + (k ? D : 0);
        const uint32_t p_tmem = tmem + (k ? 128u : 0u);
        // F8: the f16 copy of V_j in slot j & 1 (item = 2j + 1)
        const uint64_t vd = F8 ? v_desc0 + static_cast<uint64_t>((((item >> 1) & 1) * C::VH_TILE) >> 4)
                               : v_desc0 + ring_off(item);
#pragma unroll
        for (int kk = h * C::BN / 32; kk < (h + 1) * C::BN / 32; ++kk)
          mma_bf16_ts(o_tmem, p_tmem + kk * 8, vd + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                      (accumulate || kk > 0) ? 1u : 0u);
      };
      const int nkv0 = n_kv[0], nkv1 = n_kv[1];
      bool ok = mbar_wait(bar_q, 0, abort_flag) && mbar_wait(bar_kv_full(0), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        if (nkv0 > 0) {
          issue_qk(0, 0);
          tc_commit(bar_s_full(0));
        }
        if (nkv1 > 0) {
          ok = mbar_wait(bar_q1, 0, abort_flag);
          if (ok) {
            tc_fence_after_sync();
            issue_qk(1, 0);
            tc_commit(bar_s_full(1));
          }
        }
        if (ok) tc_commit(bar_kv_empty(0));
      }
      // One slot's step at key tile j: O_k += P_k V_j, then S_k(j+1).
      // S_k(j+1) overwrites the columns P_k(j) occupies; the PV MMA that reads
      // them was issued first and MMAs of one thread run in order.
      auto slot_step = [&](int k, int nk, int j, int v_item, int k_item) -> bool {
        if (j >= nk) return true;
        // the first half of P V starts while the softmax finishes the second half
        if (!mbar_wait(bar_p_half(k), j & 1, abort_flag)) return false;
        tc_fence_after_sync();
        issue_pv_half(k, v_item, j > 0, 0);
        if (!mbar_wait(bar_p_full(k), j & 1, abort_flag)) return false;
        tc_fence_after_sync();
        issue_pv_half(k, v_item, true, 1);
        tc_commit(bar_o_done(k));
        if (j + 1 < nk) {
          issue_qk(k, k_item);
          tc_commit(bar_s_full(k));
        }
        return true;
      };
      for (int j = 0; ok && j < n_max; ++j) {
        const int v_item = 2 * j + 1, k_item = 2 * j + 2;
        const bool need_k = (j + 1 < nkv0) || (j + 1 < nkv1);
        if (F8 ? !mbar_wait(bar_vh_full(j & 1), (j >> 1) & 1, abort_flag)
               : !mbar_wait(bar_kv_full(v_item), (v_item / C::NS) & 1, abort_flag))
          break;
        if (need_k && !mbar_wait(bar_kv_full(k_item), (k_item / C::NS) & 1, abort_flag)) break;
        ok = slot_step(0, nkv0, j, v_item, k_item) && slot_step(1, nkv1, j, v_item, k_item);
        if (!ok) break;
        if constexpr (F8) tc_commit(bar_vh_empty(j & 1));
        else tc_commit(bar_kv_empty(v_item));
        if (need_k) tc_commit(bar_kv_empty(k_item));
      }
      tc_commit(bar_final);
      volatile int never = 0;
      mbar_wait(bar_final, 0, &never);
    }
  } else if (F8 && warp >= 10) {
    // ---------------------------------------------------------------- V converters
    // Warp 10 widens keys 0-63 of V_j, warp 11 keys 64-127: each 16-byte
    // E4M3 unit (16 columns of one key) becomes two 16-byte f16 units of the
    // 128-byte-swizzled, two-chunk f16 tile the P V MMA reads.
    const int half = warp - 10;
    for (int j = 0; j < n_max; ++j) {
      const int v_item = 2 * j + 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_kv_full(v_item), (v_item / C::NS) & 1, abort_flag))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_vh_empty(j & 1), ((j >> 1) & 1) ^ 1, abort_flag))) break;
      const uint8_t* src = smem + C::KV_OFF + (v_item % C::NS) * C::TILE_BYTES;
      uint8_t* dst = smem + C::VH_OFF + (j & 1) * C::VH_TILE;
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
        const int c = u >> 2, w0 = 2 * (u & 3);   // f16 chunk and unit of columns 16u..16u+7
        uint8_t* row = dst + c * C::CHUNK_BYTES + key * 128;
        *reinterpret_cast<uint4*>(row + ((w0 ^ sw) << 4)) = lo4;
        *reinterpret_cast<uint4*>(row + (((w0 + 1) ^ sw) << 4)) = hi4;
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_vh_full(j & 1));
        mbar_arrive(bar_kv_empty(v_item));
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int k = warp >> 2;                       // slot
    const int r = threadIdx.x & 127;               // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sc = tmem + lane_base + (k ? 128u : 0u);
    const uint32_t oc = tmem + lane_base + 256u + (k ? D : 0);
    const int my_qtile = k ? qtile[1] : qtile[0];
    const int my_head = k ? head[1] : head[0];
    const int q_row = my_qtile * C::BM + r;
    const int nk = k ? n_kv[1] : n_kv[0];
    // Last visible key of this row, and the smallest such bound in the tile:
    // key tiles reaching past the latter need the mask.
    const int row_last = p.causal ? min(q_row + off, Lk - 1) : Lk - 1;
    const int tile_last = p.causal ? min(my_qtile * C::BM + off, Lk - 1) : Lk - 1;
    float m_ref = 0.0f, l_sum = 0.0f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(k), j & 1, abort_flag))) { ok = false; break; }
      tc_fence_after_sync();
      // key tiles reaching past tile_last need the mask
      const bool masked = (kt0 + j) * C::BN + C::BN - 1 > tile_last;
      if (!prefill_softmax_tile<D, F8>(sc, oc, j == 0, masked, row_last - (kt0 + j) * C::BN,
                                                     p.scale_log2, m_ref, l_sum, bar_o_done(k),
                                                     (j - 1) & 1, bar_p_half(k), abort_flag)) {
        ok = false;
        break;
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full(k));   // one arrival per warp
    }
    if (nk > 0 && ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done(k), (nk - 1) & 1, abort_flag))) {
      tc_fence_after_sync();
      const float inv_l = F8 ? p.v_scale / l_sum : 1.0f / l_sum;
      const bool valid = q_row < L && FA_DBG_OK(s0 + q_row < p.total_q && my_head < p.num_q_heads);
      __nv_bfloat16* orow =
          p.out + (static_cast<size_t>(s0 + q_row) * p.num_q_heads + my_head) * D;
      if (p.part_o != nullptr) {
        // key-range split: normalised fp32 O and LSE of this range
        const size_t prow = (static_cast<size_t>(split) * p.total_q + s0 + q_row) * p.num_q_heads + my_head;
        const bool pvalid = valid && FA_DBG_OK(split < max(p.kv_splits, 1));
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_x32(oc + c * 32, o);
          tmem_ld_wait(o);
          if (pvalid) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                   __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
          }
        }
        if (pvalid) p.part_lse[prow] = (m_ref + log2f(l_sum)) * 0.69314718055994530942f;
      } else {
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
        p.lse[static_cast<size_t>(s0 + q_row) * p.num_q_heads + my_head] =
            (m_ref + log2f(l_sum)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
