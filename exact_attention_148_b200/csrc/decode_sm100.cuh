// Flash-Decoding split kernel over a paged KV cache, and the LSE merge kernel.
//
// Decode has one query row per request, so the work is split along the cached
// context instead ("Flash Attention & Paged Attention", section
// "FA对decode阶段的影响": split the KV sequence, let idle SMs each take a block,
// emit a local result plus its LogSumExp, then reduce with a light kernel).
// The cache is addressed through a logical-to-physical page table (same page,
// section 2).
//
// One CTA = one (request b, kv head g, sub-group of GC query heads, split s):
//   warp 4      TMA producer: for each logical page of the split, reads the
//               physical page id from block_table and loads that page's K and
//               V rows of kv head g (64 tokens x d, one 4-D tensor-map box each)
//               into a 3-stage shared-memory ring;
//   warps 0-3   consumers: warp w takes tokens [16w, 16w+16) of every page, half
//               warp h takes every other token, each lane owns d/16 columns.
//               q.k partial dot products are reduced across the 16 lanes with a
//               transpose-and-add butterfly (each lane ends holding whole scores
//               for different (token, head) pairs), the online softmax runs on
//               those scores, and P.V accumulates in fp32 registers (packed
//               f32x2 FMA).  All GC query heads that share kv head g are served
//               from one read of each K/V byte (GQA packing).
// At the end the four warps' states are combined in shared memory.  A request
// with a single split writes bf16 O and LSE directly; otherwise the split's
// normalised O and LSE go to the fp32 workspace for fa_merge_kernel.
//
// Accumulation order depends only on logical token positions, never on the
// physical page ids, so permuting the page pool gives bit-identical output.
//
// FP8 cache (KV8): K/V pages hold E4M3 bytes with one scale per tensor.  A byte
// s.eeee.mmm is widened with integer operations only: placed in a float's
// bits 31 and 26..20 it reads as its E4M3 value times 2^-120 exactly (the
// E4M3 exponent field lands in the float's biased exponent, so subnormals map
// to float subnormals with the same ratio).  Scores are multiplied back by
// 2^120 after the dot-product reduction (k_scale is folded into the query's
// pre-scale); probabilities are taken as p * 2^60 so the P V accumulation
// (~2^-60 p v) stays in the normal float range, and the final division
// removes both factors and applies v_scale.
#pragma once

#include "ptx_sm100.cuh"

namespace fa {

constexpr int kDecodePage = 64;
constexpr int kDecodeThreads = 160;

struct DecodeParams {
  CUtensorMap tm_k;   // 4-D over the page pool, dims sorted by stride: {d, ., ., .}
  CUtensorMap tm_v;
  CUtensorMap tm_q;   // tensor-core kernel, bf16: 4-D {d, Hq, q_len, B}, box {64, G, q_len, 1}
  const __nv_bfloat16* q;        // [B, q_len, Hq, d]
  const int32_t* block_table;    // [B, max_pages]
  const int32_t* cache_seqlens;  // [B]
  __nv_bfloat16* out;            // [B, q_len, Hq, d]
  float* lse;                    // [B, q_len, Hq] or null
  float* ws_o;                   // [max_splits, B, q_len, Hq, d]
  float* ws_lse;                 // [max_splits, B, q_len, Hq]
  int batch;
  int q_len;                     // query tokens per request (1, or more on tensor cores)
  int num_q_heads;
  int group;                     // Hq / Hkv
  int subgroups;                 // group / GC
  int max_pages;                 // block_table row length
  int num_pages;                 // physical pages in the pool
  int chunk_tokens;              // keys per split (multiple of 64)
  int max_splits;
  int head_coord;                // tensor-map dimension (1..3) indexed by kv head
  int page_coord;                // tensor-map dimension (1..3) indexed by page id
  float scale_log2;              // scale * log2(e) (* k_scale for an FP8 cache)
  float v_scale;                 // FP8 cache: V dequantisation scale
};

constexpr float kTwo60 = 1152921504606846976.0f;                           // 2^60
constexpr float kTwo120 = 1329227995784915872903807060280344576.0f;       // 2^120

template <int D, int GC, bool KV8>
struct DecodeCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(GC == 1 || GC == 2 || GC == 4 || GC == 8, "1, 2, 4 or 8 heads per CTA");
  static constexpr int ELEM = KV8 ? 1 : 2;             // bytes per cached element
  // An FP8 page is half the bytes: twice the stages keeps as many bytes in flight.
  static constexpr int STAGES = KV8 ? 6 : 3;
  static constexpr int COLS = D / 16;                  // columns per lane
  static constexpr int ROW_BYTES = D * ELEM;
  static constexpr int TILE_BYTES = kDecodePage * ROW_BYTES;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = STAGES * TILE_BYTES;
  static constexpr int SC_OFF = 2 * STAGES * TILE_BYTES;        // 4 warps x 16 x GC floats
  static constexpr int BAR_OFF = SC_OFF + 4 * 16 * GC * 4;
  static constexpr int MISC_OFF = BAR_OFF + 2 * STAGES * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  // combine scratch (aliases the K/V ring once every page is consumed)
  static constexpr int CMB_O = 0;                      // [4][GC][D] floats
  static constexpr int CMB_M = 4 * GC * D * 4;         // [4][GC]
  static constexpr int CMB_L = CMB_M + 4 * GC * 4;     // [4][GC]
  static_assert(CMB_L + 4 * GC * 4 <= SC_OFF, "combine scratch fits the ring");
};

// Reduce N partial sums per lane across the 16 lanes of a half warp.  Each
// round exchanges half of the remaining values with the partner lane and adds
// the received half to the kept half, so after four rounds every lane holds
// max(1, N/16) complete sums (the classic transpose-reduce butterfly).
template <int N, int MASK>
__device__ __forceinline__ void xpose_reduce16(float* v, int lane) {
  if constexpr (MASK > 0) {
    if constexpr (N >= 2) {
      const bool upper = (lane & MASK) != 0;
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        const float send = upper ? v[k] : v[k + N / 2];
        const float keep = upper ? v[k + N / 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
      }
      xpose_reduce16<N / 2, MASK / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], MASK);
      xpose_reduce16<1, MASK / 2>(v, lane);
    }
  }
}

// Index (into the original N values) of the first value a lane holds after
// xpose_reduce16<N, 8>.
template <int N>
__device__ __forceinline__ int xpose_base(int lane16) {
  int base = 0, n = N;
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    if (n >= 2) {
      if (lane16 & m) base += n / 2;
      n /= 2;
    }
  }
  return base;
}

template <int COLS>
__device__ __forceinline__ void load_bf16_row(const uint8_t* src, float2 (&f)[COLS / 2]) {
  if constexpr (COLS == 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(src);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i)
      f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
}

// E4M3 byte i (0..3, compile-time) of w as a float equal to its value times
// 2^-120: the byte goes to bits 31..24, an arithmetic shift by 4 puts
// s.eeee.mmm at bits 27..20 with the sign copied above, and the mask keeps the
// sign at bit 31 and eeee.mmm at bits 26..20.
template <int I>
__device__ __forceinline__ float e4m3_scaled(uint32_t w) {
  const int32_t t = static_cast<int32_t>(w << (24 - 8 * I));
  return __int_as_float((t >> 4) & static_cast<int32_t>(0x87F00000u));
}

template <int COLS>
__device__ __forceinline__ void load_e4m3_row(const uint8_t* src, float2 (&f)[COLS / 2]) {
  if constexpr (COLS == 8) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    f[0] = make_float2(e4m3_scaled<0>(u.x), e4m3_scaled<1>(u.x));
    f[1] = make_float2(e4m3_scaled<2>(u.x), e4m3_scaled<3>(u.x));
    f[2] = make_float2(e4m3_scaled<0>(u.y), e4m3_scaled<1>(u.y));
    f[3] = make_float2(e4m3_scaled<2>(u.y), e4m3_scaled<3>(u.y));
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
    f[0] = make_float2(e4m3_scaled<0>(u), e4m3_scaled<1>(u));
    f[1] = make_float2(e4m3_scaled<2>(u), e4m3_scaled<3>(u));
  }
}

template <bool KV8, int COLS>
__device__ __forceinline__ void load_kv_row(const uint8_t* src, float2 (&f)[COLS / 2]) {
  if constexpr (KV8) load_e4m3_row<COLS>(src, f);
  else load_bf16_row<COLS>(src, f);
}

// Two CTAs per SM (their rings overlap each other's pipeline fill), except
// with 8 packed heads, whose accumulators need the larger register budget.
template <int D, int GC, bool KV8>
__global__ void __launch_bounds__(kDecodeThreads, GC == 8 ? 1 : 2)
    fa_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<D, GC, KV8>;
  constexpr int COLS = C::COLS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int kv_head = blockIdx.y / p.subgroups;
  const int qh0 = kv_head * p.group + (blockIdx.y % p.subgroups) * GC;
  const int b = blockIdx.z;

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

  const uint32_t bars = base + C::BAR_OFF;
  auto bar_full = [&](int st) { return bars + 8 * st; };
  auto bar_empty = [&](int st) { return bars + 8 * (C::STAGES + st); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF);

  if (threadIdx.x == 0) {
    for (int st = 0; st < C::STAGES; ++st) {
      mbar_init(bar_full(st), 1);
      mbar_init(bar_empty(st), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    const int32_t* bt_row = p.block_table + static_cast<size_t>(b) * p.max_pages + page_begin;
    int issued = 0;
    bool ok = true;
    for (int i0 = 0; ok && i0 < num_pg; i0 += 32) {
      const int mine = (i0 + lane < num_pg && FA_DBG_OK(page_begin + i0 + lane < p.max_pages))
                           ? bt_row[i0 + lane] : 0;
      const int cnt = min(32, num_pg - i0);
      for (int ii = 0; ii < cnt; ++ii) {
        int phys = __shfl_sync(0xffffffffu, mine, ii);
        if (lane == 0) {
          const int i = i0 + ii;
          const int st = i % C::STAGES;
          if (mbar_wait(bar_empty(st), ((i / C::STAGES) & 1) ^ 1, abort_flag)) {
            // A page id outside the pool is recorded and replaced by num_pages,
            // one past the tensor map's last page, which TMA reads as zeros.
            if (phys < 0 || phys >= p.num_pages) {
              record_status(FA_ERR_BAD_PAGE);
              phys = p.num_pages;
            }
            int c1 = 0, c2 = 0, c3 = 0;
            c1 = (p.head_coord == 1) ? kv_head : (p.page_coord == 1 ? phys : 0);
            c2 = (p.head_coord == 2) ? kv_head : (p.page_coord == 2 ? phys : 0);
            c3 = (p.head_coord == 3) ? kv_head : (p.page_coord == 3 ? phys : 0);
            mbar_arrive_expect_tx(bar_full(st), 2 * C::TILE_BYTES);
            tma_load_4d(base + C::K_OFF + st * C::TILE_BYTES, &p.tm_k, bar_full(st), 0, c1, c2, c3);
            tma_load_4d(base + C::V_OFF + st * C::TILE_BYTES, &p.tm_v, bar_full(st), 0, c1, c2, c3);
            ++issued;
          } else {
            ok = false;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int never = 0;
      for (int i = (issued > C::STAGES ? issued - C::STAGES : 0); i < issued; ++i)
        mbar_wait(bar_full(i % C::STAGES), (i / C::STAGES) & 1, &never);
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int half = lane >> 4;
    const int l16 = lane & 15;
    const int c0 = l16 * COLS;
    float* sc = reinterpret_cast<float*>(smem + C::SC_OFF) + warp * 16 * GC;

    float2 qr[GC][COLS / 2];
#pragma unroll
    for (int gi = 0; gi < GC; ++gi) {
      const size_t qrow = static_cast<size_t>(b) * p.num_q_heads + qh0 + gi;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(
          p.q + (FA_DBG_OK(qrow < static_cast<size_t>(p.batch) * p.num_q_heads) ? qrow : 0) * D + c0);
      load_bf16_row<COLS>(src, qr[gi]);
#pragma unroll
      for (int c = 0; c < COLS / 2; ++c) {
        qr[gi][c].x *= p.scale_log2;
        qr[gi][c].y *= p.scale_log2;
      }
    }
    float2 acc[GC][COLS / 2];
#pragma unroll
    for (int gi = 0; gi < GC; ++gi)
#pragma unroll
      for (int c = 0; c < COLS / 2; ++c) acc[gi][c] = make_float2(0.f, 0.f);
    // Online-softmax state of query head (lane % GC), replicated across the
    // lanes of that residue class.
    float m_run = -INFINITY, l_run = 0.0f;

    constexpr int NV = 8 * GC;                  // partial sums per lane per page
    constexpr int R = NV >= 16 ? NV / 16 : 1;   // complete sums per lane after reduce
    const int xbase = xpose_base<NV>(l16);
    const bool writer = (NV >= 16) || ((l16 & 1) == 0);
    constexpr int E = 16 * GC;                  // scores per warp per page
    constexpr int PER = (E + 31) / 32;

    for (int i = 0; i < num_pg; ++i) {
      const int st = i % C::STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_full(st), (i / C::STAGES) & 1, abort_flag))) break;
      const uint8_t* Ks = smem + C::K_OFF + st * C::TILE_BYTES;
      const uint8_t* Vs = smem + C::V_OFF + st * C::TILE_BYTES;
      const int tok0 = (page_begin + i) * kDecodePage + warp * 16;   // logical index of token 0

      // ---- scores: q . k for this half's 8 tokens x GC heads
      float part[NV];
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        const int tt = warp * 16 + 2 * ii + half;
        float2 kf[COLS / 2];
        load_kv_row<KV8, COLS>(Ks + tt * C::ROW_BYTES + c0 * C::ELEM, kf);
#pragma unroll
        for (int gi = 0; gi < GC; ++gi) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < COLS / 2; ++c) a = __ffma2_rn(qr[gi][c], kf[c], a);
          part[ii * GC + gi] = a.x + a.y;
        }
      }
      xpose_reduce16<NV, 8>(part, lane);
#pragma unroll
      for (int k = 0; k < R; ++k) {
        const int idx = xbase + k;
        const int ii = idx / GC, gi = idx % GC;
        const int tok = 2 * ii + half;
        const float val = (tok0 + tok < t_end) ? (KV8 ? part[k] * kTwo120 : part[k]) : -INFINITY;
        if (writer) sc[tok * GC + gi] = val;
      }
      __syncwarp();

      // ---- online softmax over the warp's 16 tokens (entries idx = lane + 32k)
      float sv[PER];
      float mt = -INFINITY;
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int idx = lane + 32 * k;
        sv[k] = (idx < E) ? sc[idx] : -INFINITY;
        mt = fmaxf(mt, sv[k]);
      }
#pragma unroll
      for (int m = GC; m < 32; m <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, m));
      const float m_new = fmaxf(m_run, mt);
      const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
      const float alpha = ex2_approx(m_run - m_use);
      m_run = m_new;
      float ps = 0.0f;
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int idx = lane + 32 * k;
        // FP8: p * 2^60 keeps the P V products of E4M3 values (x 2^-120) normal
        const float pv = ex2_approx(KV8 ? (sv[k] - m_use) + 60.0f : sv[k] - m_use);
        if (idx < E) sc[idx] = pv;
        ps += pv;
      }
#pragma unroll
      for (int m = GC; m < 32; m <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
      l_run = l_run * alpha + ps;
      float alpha_g[GC];
#pragma unroll
      for (int gi = 0; gi < GC; ++gi) alpha_g[gi] = __shfl_sync(0xffffffffu, alpha, gi);
      __syncwarp();

      // ---- O = alpha * O + P V
#pragma unroll
      for (int gi = 0; gi < GC; ++gi)
#pragma unroll
        for (int c = 0; c < COLS / 2; ++c) {
          acc[gi][c].x *= alpha_g[gi];
          acc[gi][c].y *= alpha_g[gi];
        }
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        const int tok = 2 * ii + half;
        float2 vf[COLS / 2];
        load_kv_row<KV8, COLS>(Vs + (warp * 16 + tok) * C::ROW_BYTES + c0 * C::ELEM, vf);
        if (tok0 + tok >= t_end) {   // page tail past the cache end: never read its values
#pragma unroll
          for (int c = 0; c < COLS / 2; ++c) vf[c] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int gi = 0; gi < GC; ++gi) {
          const float pw = sc[tok * GC + gi];
          const float2 pp = make_float2(pw, pw);
#pragma unroll
          for (int c = 0; c < COLS / 2; ++c) acc[gi][c] = __ffma2_rn(pp, vf[c], acc[gi][c]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(st));
    }

    // ---- combine the two halves (same running max), then the four warps
#pragma unroll
    for (int gi = 0; gi < GC; ++gi)
#pragma unroll
      for (int c = 0; c < COLS / 2; ++c) {
        acc[gi][c].x += __shfl_xor_sync(0xffffffffu, acc[gi][c].x, 16);
        acc[gi][c].y += __shfl_xor_sync(0xffffffffu, acc[gi][c].y, 16);
      }
    asm volatile("bar.sync 1, 128;" ::: "memory");   // every consumer is done with the ring
    float* cmb_o = reinterpret_cast<float*>(smem + C::CMB_O);
    float* cmb_m = reinterpret_cast<float*>(smem + C::CMB_M);
    float* cmb_l = reinterpret_cast<float*>(smem + C::CMB_L);
    if (half == 0) {
#pragma unroll
      for (int gi = 0; gi < GC; ++gi)
#pragma unroll
        for (int c = 0; c < COLS / 2; ++c)
          *reinterpret_cast<float2*>(&cmb_o[(warp * GC + gi) * D + c0 + 2 * c]) = acc[gi][c];
    }
    if (lane < GC) {
      cmb_m[warp * GC + lane] = m_run;
      cmb_l[warp * GC + lane] = l_run;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");

    const int tid = threadIdx.x;   // 0..127
    const bool direct = (nsplit_eff == 1);
    for (int e = tid; e < GC * D; e += 128) {
      const int gi = e / D, c = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, cmb_m[w * GC + gi]);
      float o = 0.0f, lsum = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float f = ex2_approx(cmb_m[w * GC + gi] - M);
          lsum += cmb_l[w * GC + gi] * f;
          o += cmb_o[(w * GC + gi) * D + c] * f;
        }
        if constexpr (KV8)   // o ~ 2^-60 sum p v, lsum = 2^60 sum p
          o = (o * kTwo60) * (kTwo60 * p.v_scale / lsum);
        else
          o = o / lsum;
      }
      const float lse_v = (M == -INFINITY) ? -INFINITY
                                           : (M + log2f(lsum) - (KV8 ? 60.0f : 0.0f)) * 0.69314718055994530942f;
      const size_t row = static_cast<size_t>(b) * p.num_q_heads + qh0 + gi;
      const size_t rows = static_cast<size_t>(p.batch) * p.num_q_heads;
      if (direct) {
        if (FA_DBG_OK(row < rows)) {
          p.out[row * D + c] = __float2bfloat16_rn(o);
          if (c == 0 && p.lse != nullptr) p.lse[row] = lse_v;
        }
      } else {
        const size_t srow = static_cast<size_t>(split) * rows + row;
        if (FA_DBG_OK(srow < static_cast<size_t>(p.max_splits) * rows)) {
          p.ws_o[srow * D + c] = o;
          if (c == 0) p.ws_lse[srow] = lse_v;
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// LSE merge: out = sum_i w_i O_i / sum_i w_i, w_i = e^{LSE_i - max}, one warp
// per (row, head).  With `cache_seqlens` set (decode), row r has
// ceil(seqlen_r / chunk) states and rows with a single state are skipped (the
// split kernel wrote them directly); otherwise every row has num_states.
// ----------------------------------------------------------------------------
struct MergeParams {
  const float* o_parts;        // [S, rows, H, D]
  const float* lse_parts;      // [S, rows, H]
  __nv_bfloat16* out;          // [rows, H, D]
  float* lse;                  // [rows, H] or null
  const int32_t* cache_seqlens;// null for a plain merge
  int q_len;                   // rows per request (row r belongs to request r / q_len)
  int num_states;
  int rows;
  int num_heads;
  int chunk_tokens;
  int max_pages;
};

template <int D>
__global__ void __launch_bounds__(128) fa_merge_kernel(const MergeParams p) {
  constexpr int V = D / 32;   // columns per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rh = blockIdx.x * 4 + warp;
  if (rh >= p.rows * p.num_heads) return;
  const int r = rh / p.num_heads;
  int ns = p.num_states;
  if (p.cache_seqlens != nullptr) {
    if (!FA_DBG_OK(r / p.q_len < (p.rows + p.q_len - 1) / p.q_len)) return;
    int seqlen = p.cache_seqlens[r / p.q_len];
    seqlen = max(0, min(seqlen, p.max_pages * kDecodePage));
    ns = min(p.num_states, (seqlen + p.chunk_tokens - 1) / p.chunk_tokens);
    if (ns <= 1) return;
  }
  const size_t stride = static_cast<size_t>(p.rows) * p.num_heads;
  if (!FA_DBG_OK(ns <= p.num_states)) return;
  float M = -INFINITY;
  for (int i = lane; i < ns; i += 32) M = fmaxf(M, p.lse_parts[i * stride + rh]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
  float o[V];
#pragma unroll
  for (int v = 0; v < V; ++v) o[v] = 0.0f;
  float wsum = 0.0f;
  constexpr float kLog2e = 1.4426950408889634f;
  if (M != -INFINITY) {
    for (int i = 0; i < ns; ++i) {
      const float li = p.lse_parts[i * stride + rh];
      const float w = ex2_approx((li - M) * kLog2e);   // li = -inf -> 0
      wsum += w;
      const float* src = p.o_parts + (i * stride + rh) * D + lane * V;
      if constexpr (V == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        o[0] = fmaf(w, x.x, o[0]);
        o[1] = fmaf(w, x.y, o[1]);
        o[2] = fmaf(w, x.z, o[2]);
        o[3] = fmaf(w, x.w, o[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        o[0] = fmaf(w, x.x, o[0]);
        o[1] = fmaf(w, x.y, o[1]);
      }
    }
  }
  const float inv = (wsum > 0.0f) ? 1.0f / wsum : 0.0f;
  __nv_bfloat16* dst = p.out + static_cast<size_t>(rh) * D + lane * V;
#pragma unroll
  for (int v = 0; v < V; v += 2) {
    *reinterpret_cast<__nv_bfloat162*>(dst + v) = __floats2bfloat162_rn(o[v] * inv, o[v + 1] * inv);
  }
  if (lane == 0 && p.lse != nullptr)
    p.lse[rh] = (wsum > 0.0f) ? M + logf(wsum) : -INFINITY;
}

}  // namespace fa

namespace fa {

// ----------------------------------------------------------------------------
// Cascade merge: for every (row, head), the LSE merge of the shared prefix's
// key-range states (fp32) and the row's own suffix state (bf16 O + LSE), one
// warp per (row, head).  An empty suffix carries LSE = -inf and zero weight.
// ----------------------------------------------------------------------------
struct CascadeMergeParams {
  const float* prefix_o;          // [S, rows, H, D] normalised
  const float* prefix_lse;        // [S, rows, H]
  const __nv_bfloat16* suffix_o;  // [rows, H, D] normalised
  const float* suffix_lse;        // [rows, H]
  __nv_bfloat16* out;             // [rows, H, D]
  float* lse;                     // [rows, H] or null
  int num_prefix;
  int rows;
  int num_heads;
};

template <int D>
__global__ void __launch_bounds__(128) fa_cascade_merge_kernel(const CascadeMergeParams p) {
  constexpr int V = D / 32;   // columns per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rh = blockIdx.x * 4 + warp;
  if (rh >= p.rows * p.num_heads) return;
  const size_t stride = static_cast<size_t>(p.rows) * p.num_heads;
  if (!FA_DBG_OK(p.num_prefix >= 0)) return;
  const float ls = p.suffix_lse[rh];
  float M = ls;
  for (int i = lane; i < p.num_prefix; i += 32) M = fmaxf(M, p.prefix_lse[i * stride + rh]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
  float o[V];
#pragma unroll
  for (int v = 0; v < V; ++v) o[v] = 0.0f;
  float wsum = 0.0f;
  constexpr float kLog2e = 1.4426950408889634f;
  if (M != -INFINITY) {
    for (int i = 0; i < p.num_prefix; ++i) {
      const float w = ex2_approx((p.prefix_lse[i * stride + rh] - M) * kLog2e);
      wsum += w;
      const float* src = p.prefix_o + (i * stride + rh) * D + lane * V;
#pragma unroll
      for (int v = 0; v < V; ++v) o[v] = fmaf(w, src[v], o[v]);
    }
    const float w = ex2_approx((ls - M) * kLog2e);   // -inf -> 0
    wsum += w;
    const __nv_bfloat16* src = p.suffix_o + static_cast<size_t>(rh) * D + lane * V;
#pragma unroll
    for (int v = 0; v < V; ++v) o[v] = fmaf(w, __bfloat162float(src[v]), o[v]);
  }
  const float inv = (wsum > 0.0f) ? 1.0f / wsum : 0.0f;
  __nv_bfloat16* dst = p.out + static_cast<size_t>(rh) * D + lane * V;
#pragma unroll
  for (int v = 0; v < V; v += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + v) = __floats2bfloat162_rn(o[v] * inv, o[v + 1] * inv);
  if (lane == 0 && p.lse != nullptr) p.lse[rh] = (wsum > 0.0f) ? M + logf(wsum) : -INFINITY;
}

}  // namespace fa
