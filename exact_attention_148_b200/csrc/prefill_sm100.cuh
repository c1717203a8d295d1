// Causal / full exact-attention prefill for sm_100a.
//
// One CTA computes one 128-row query tile of one query head:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r);
//   warp  4    TMA producer: Q once, then K_j / V_j into 3-stage rings;
//   warp  5    MMA issuer: S_j = Q K_j^T into one of two TMEM score buffers,
//              O += P_j V_j with P_j (bf16) read straight from TMEM.
// The loop is the tiling + online-softmax scheme of cloud.baidu.com
// "FasterTransformer与FlashAttention的联系与区别", section 三 (load a K/V block,
// score it, update running max and normaliser, accumulate the output), on
// tcgen05 tensor cores with the accumulators in tensor memory.  Scores live
// only in TMEM; nothing of size N x N reaches HBM.
//
// TMEM columns: S/P buffer 0 [0,128), S/P buffer 1 [128,256), O [256,256+D).
// The score of key tile j+1 is computed while the softmax warps work on tile j.
//
// Online softmax in base 2: x = s * scale * log2(e).  The running maximum used
// for the exponentials is only raised when the tile maximum exceeds it by more
// than 8 (a factor of 256); otherwise the stale maximum is kept.  Every
// exponential, the normaliser l and the accumulator O use the same reference
// value, so O / l is unchanged; it only skips most O rescales (which are TMEM
// round trips).  P values stay <= 2^8, safely inside bf16 and fp32 ranges.
#pragma once

#include "ptx_sm100.cuh"

namespace fa {

constexpr int kPrefillMaxTiles = 2048;   // (sequence, q-tile) entries per launch
constexpr int kPrefillThreads = 192;
constexpr float kRescaleThreshold = 8.0f;

struct PrefillParams {
  CUtensorMap tm_q;   // 3-D {d, Hq, T}, box {64, 1, 128}, 128B swizzle
  CUtensorMap tm_k;   // 3-D {d, Hkv, T}
  CUtensorMap tm_v;
  __nv_bfloat16* out;        // [T, Hq, d]
  float* lse;                // [T, Hq] or null
  const int32_t* cu_seqlens; // [B+1]
  int num_q_heads;
  int group;                 // Hq / Hkv
  int causal;
  float scale_log2;          // scale * log2(e)
  int num_tiles;
  uint32_t tiles[kPrefillMaxTiles];   // (sequence << 16) | q_tile, heaviest first
};

template <int D>
struct PrefillCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int BM = 128;                 // query rows per tile
  static constexpr int BN = 128;                 // keys per tile
  static constexpr int STAGES = 3;               // K ring depth == V ring depth
  static constexpr int CHUNKS = D / 64;          // 128-byte swizzle atoms along d
  static constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STAGES * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STAGES * TILE_BYTES;
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2],
  // o_done, final
  static constexpr int NUM_BARS = 1 + 4 * STAGES + 2 + 2 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;   // tmem base, abort flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;   // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 128, O_COL = 256;
};

template <int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    fa_prefill_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.x;
  const uint32_t entry = p.tiles[blockIdx.y];
  const int seq = static_cast<int>(entry >> 16);
  const int qtile = static_cast<int>(entry & 0xFFFFu);
  const int s0 = p.cu_seqlens[seq];
  const int L = p.cu_seqlens[seq + 1] - s0;
  const int q_row0 = qtile * C::BM;
  if (q_row0 >= L) return;   // uniform over the CTA; nothing allocated yet
  const int kv_head = head / p.group;
  const int n_kv = p.causal ? qtile + 1 : (L + C::BN - 1) / C::BN;

  const uint32_t q_s = base + C::Q_OFF;
  auto k_s = [&](int st) { return base + C::K_OFF + st * C::TILE_BYTES; };
  auto v_s = [&](int st) { return base + C::V_OFF + st * C::TILE_BYTES; };
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t bar_q = bars;
  auto bar_k_full = [&](int st) { return bars + 8 * (1 + st); };
  auto bar_k_empty = [&](int st) { return bars + 8 * (1 + C::STAGES + st); };
  auto bar_v_full = [&](int st) { return bars + 8 * (1 + 2 * C::STAGES + st); };
  auto bar_v_empty = [&](int st) { return bars + 8 * (1 + 3 * C::STAGES + st); };
  auto bar_s_full = [&](int b) { return bars + 8 * (1 + 4 * C::STAGES + b); };
  // One P barrier per S/P buffer: the softmax warps may finish tile j+1
  // before the MMA warp has observed tile j, so a single barrier could
  // complete two phases unobserved.
  auto bar_p_full = [&](int b) { return bars + 8 * (3 + 4 * C::STAGES + b); };
  const uint32_t bar_o_done = bars + 8 * (5 + 4 * C::STAGES);
  const uint32_t bar_final = bars + 8 * (6 + 4 * C::STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int st = 0; st < C::STAGES; ++st) {
      mbar_init(bar_k_full(st), 1);
      mbar_init(bar_k_empty(st), 1);
      mbar_init(bar_v_full(st), 1);
      mbar_init(bar_v_empty(st), 1);
    }
    mbar_init(bar_s_full(0), 1);
    mbar_init(bar_s_full(1), 1);
    mbar_init(bar_p_full(0), 128);
    mbar_init(bar_p_full(1), 128);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_3d(q_s + c * C::CHUNK_BYTES, &p.tm_q, bar_q, c * 64, head, s0 + q_row0);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(bar_k_empty(st), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_k_full(st), C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(k_s(st) + c * C::CHUNK_BYTES, &p.tm_k, bar_k_full(st), c * 64, kv_head,
                      s0 + j * C::BN);
        ++k_issued;
        if (!mbar_wait(bar_v_empty(st), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_v_full(st), C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(v_s(st) + c * C::CHUNK_BYTES, &p.tm_v, bar_v_full(st), c * 64, kv_head,
                      s0 + j * C::BN);
        ++v_issued;
      }
      if (*abort_flag) {
        // Let the copies still in flight land before the CTA exits.  Only the
        // newest load of each stage can be outstanding.
        volatile int never = 0;
        for (int j = (k_issued > C::STAGES ? k_issued - C::STAGES : 0); j < k_issued; ++j)
          mbar_wait(bar_k_full(j % C::STAGES), (j / C::STAGES) & 1, &never);
        for (int j = (v_issued > C::STAGES ? v_issued - C::STAGES : 0); j < v_issued; ++j)
          mbar_wait(bar_v_full(j % C::STAGES), (j / C::STAGES) & 1, &never);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(C::BM, C::BN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(C::BM, D, true);
      auto issue_qk = [&](uint32_t d_tmem, uint32_t kbase) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, sdesc_sw128(q_s + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                      idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](uint32_t p_tmem, uint32_t vbase, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          mma_bf16_ts(tmem + C::O_COL, p_tmem + kk * 8,
                      sdesc_sw128(vbase + kk * 16 * 128, C::CHUNK_BYTES, 1024), idesc_pv,
                      (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar_q, 0, abort_flag) && mbar_wait(bar_k_full(0), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        issue_qk(tmem + C::S_COL0, k_s(0));
        tc_commit(bar_s_full(0));
        tc_commit(bar_k_empty(0));
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) {
          const int st = (j + 1) % C::STAGES;
          if (!mbar_wait(bar_k_full(st), ((j + 1) / C::STAGES) & 1, abort_flag)) break;
          tc_fence_after_sync();
          // Buffer (j+1)&1 last held P_{j-1}, whose PV was issued earlier;
          // tcgen05.mma from one thread execute in issue order.
          issue_qk(tmem + (((j + 1) & 1) ? C::S_COL1 : C::S_COL0), k_s(st));
          tc_commit(bar_s_full((j + 1) & 1));
          tc_commit(bar_k_empty(st));
        }
        if (!mbar_wait(bar_p_full(j & 1), (j >> 1) & 1, abort_flag)) break;
        const int vst = j % C::STAGES;
        if (!mbar_wait(bar_v_full(vst), (j / C::STAGES) & 1, abort_flag)) break;
        tc_fence_after_sync();
        issue_pv(tmem + ((j & 1) ? C::S_COL1 : C::S_COL0), v_s(vst), j > 0);
        tc_commit(bar_o_done);
        tc_commit(bar_v_empty(vst));
      }
      // Nothing of ours may still be in flight when TMEM is released.
      tc_commit(bar_final);
      volatile int never = 0;
      mbar_wait(bar_final, 0, &never);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int r = threadIdx.x;                 // query row within the tile
    const int q_row = q_row0 + r;              // in-sequence query index
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = 0.0f;                        // reference max (base-2 scaled units)
    float l_sum = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const uint32_t s_col = (j & 1) ? C::S_COL1 : C::S_COL0;
      // Waits are made warp-uniform so the warp-collective tcgen05.ld/st that
      // follow are never reached by part of a warp.
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(j & 1), (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_x32(tmem + lane_base + s_col + c * 32, s[c]);
      tmem_ld_wait(s[0]);
      reg_dep(s[1]);
      reg_dep(s[2]);
      reg_dep(s[3]);

      const bool diag = p.causal ? (j == qtile) : ((j + 1) * C::BN > L);
      float rmax = -INFINITY;
      if (diag) {
        const int lim = p.causal ? (q_row - j * C::BN) : (L - 1 - j * C::BN);   // last allowed col
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x = __uint_as_float(s[c][i]);
            x = (c * 32 + i <= lim) ? x : -INFINITY;
            s[c][i] = __float_as_uint(x);
            rmax = fmaxf(rmax, x);
          }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) rmax = fmaxf(rmax, __uint_as_float(s[c][i]));
      }
      const float m_tile = rmax * p.scale_log2;   // -inf stays -inf (scale > 0)
      if (j == 0) {
        m_ref = (m_tile == -INFINITY) ? 0.0f : m_tile;
      } else {
        const bool need = m_tile > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_ref - m_tile) : 1.0f;
          if (need) m_ref = m_tile;
          l_sum *= alpha;
          // O must hold P_{j-1} V_{j-1} before it is rescaled.
          if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done, (j - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_x32(tmem + lane_base + C::O_COL + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_x32(tmem + lane_base + C::O_COL + c * 32, o);
          }
          tmem_st_wait();
        }
      }
      const float neg_m = -m_ref;
      float psum = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c][2 * i]), p.scale_log2, neg_m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c][2 * i + 1]), p.scale_log2, neg_m));
          psum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        // P chunk c (32 scores -> 16 packed columns) goes over already-read S columns.
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c][i] = pk[i];
      }
      l_sum += psum;
      {
        uint32_t pa[32], pb[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pa[i] = s[0][i];
          pa[16 + i] = s[1][i];
          pb[i] = s[2][i];
          pb[16 + i] = s[3][i];
        }
        tmem_st_x32(tmem + lane_base + s_col, pa);
        tmem_st_x32(tmem + lane_base + s_col + 32, pb);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(bar_p_full(j & 1));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done, (n_kv - 1) & 1, abort_flag))) {
      tc_fence_after_sync();
      const float inv_l = 1.0f / l_sum;
      const bool valid = q_row < L;
      __nv_bfloat16* orow =
          p.out + (static_cast<size_t>(s0 + q_row) * p.num_q_heads + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld_x32(tmem + lane_base + C::O_COL + c * 32, o);
        tmem_ld_wait(o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (valid && p.lse != nullptr)
        p.lse[static_cast<size_t>(s0 + q_row) * p.num_q_heads + head] =
            (m_ref + log2f(l_sum)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
