"""Seeded synthetic inputs for exact attention (prefill and paged decode).

This module is shared by the CPU oracle's tests, the GPU parity tests and
``bench.py``.  It only draws random numbers, rounds them to bfloat16 and lays
them out; it holds none of the attention arithmetic.

Workload shapes follow the pages' problem statements:

* prefill: packed ``[T, H, d]`` Q/K/V with ``cu_seqlens`` offsets (the FA
  varlen form named on "FIA / FlashAttention", section 二 and 三);
* decode: one query row per request over a KV cache stored in fixed-size pages
  (64 tokens per page, "FlashAttention突破性架构", section 分页存储系统) addressed
  through a logical-to-physical page table ("Flash Attention & Paged
  Attention", section 2).

Every tensor is produced as float32 draws from N(0, 1), rounded to bfloat16
with round-to-nearest-even.  The ``*_bits`` arrays are the uint16 bit patterns
that go to the device; ``as_f64`` gives the same values widened for the oracle.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

PAGE_SIZE = 64


# ---------------------------------------------------------------------------
# bfloat16 helpers (bit manipulation only)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 values (exact widening)."""
    return bf16_bits_to_f32(b).astype(np.float64)


def _normal_bf16_bits(seed_seq: np.random.SeedSequence, shape, chunk_elems=1 << 24) -> np.ndarray:
    """N(0,1) float32 draws rounded to bf16, filled in parallel chunks.

    Each chunk draws from its own child of ``seed_seq`` so the result does not
    depend on the number of worker threads.
    """
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = max(1, math.ceil(n / chunk_elems))
    children = seed_seq.spawn(nchunks)

    def fill(i):
        lo = i * chunk_elems
        hi = min(n, lo + chunk_elems)
        g = np.random.Generator(np.random.PCG64(children[i]))
        out[lo:hi] = f32_to_bf16_bits(g.standard_normal(hi - lo, dtype=np.float32))

    workers = min(nchunks, os.cpu_count() or 1)
    if workers <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


# ---------------------------------------------------------------------------
# Prefill workloads
# ---------------------------------------------------------------------------

@dataclass
class PrefillInputs:
    name: str
    q_bits: np.ndarray          # [T, Hq, d] uint16 (bf16)
    k_bits: np.ndarray          # [T, Hkv, d]
    v_bits: np.ndarray          # [T, Hkv, d]
    cu_seqlens: np.ndarray      # [B+1] int32
    causal: bool
    scale: float
    q_f32_unrounded: np.ndarray | None = None   # only kept for tiny cases

    @property
    def num_q_heads(self):
        return self.q_bits.shape[1]

    @property
    def num_kv_heads(self):
        return self.k_bits.shape[1]

    @property
    def head_dim(self):
        return self.q_bits.shape[2]

    @property
    def seqlens(self):
        return np.diff(self.cu_seqlens).astype(np.int64)

    def causal_flops(self) -> float:
        """Algorithmic FLOPs: 4*d*Hq per (query, allowed key) pair."""
        L = self.seqlens
        pairs = (L * (L + 1) // 2).sum() if self.causal else (L * L).sum()
        return 4.0 * self.head_dim * self.num_q_heads * float(pairs)


def make_prefill(seqlens, num_q_heads, num_kv_heads, head_dim, *, causal=True,
                 scale=None, seed=0, name="prefill") -> PrefillInputs:
    seqlens = np.asarray(seqlens, dtype=np.int64)
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    T = int(cu[-1])
    ss = np.random.SeedSequence(seed)
    sq, sk, sv = ss.spawn(3)
    q = _normal_bf16_bits(sq, (T, num_q_heads, head_dim))
    k = _normal_bf16_bits(sk, (T, num_kv_heads, head_dim))
    v = _normal_bf16_bits(sv, (T, num_kv_heads, head_dim))
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return PrefillInputs(name, q, k, v, cu, causal, float(scale))


def tiny_causal_prefill() -> PrefillInputs:
    """Batch 1, 2 heads, 128 tokens, d=64, fp32 N(0,1) inputs, scale 1/sqrt(64).

    The fp32 draws are rounded to bf16 before either side sees them; the
    unrounded query is kept so tests can report the rounding effect.
    """
    g = np.random.default_rng(0)
    T, H, d = 128, 2, 64
    qf = g.standard_normal((T, H, d), dtype=np.float32)
    kf = g.standard_normal((T, H, d), dtype=np.float32)
    vf = g.standard_normal((T, H, d), dtype=np.float32)
    cu = np.array([0, T], dtype=np.int32)
    inp = PrefillInputs("tiny_causal_prefill", f32_to_bf16_bits(qf), f32_to_bf16_bits(kf),
                        f32_to_bf16_bits(vf), cu, True, 1.0 / math.sqrt(64))
    inp.q_f32_unrounded = qf
    return inp


def varlen_lengths(seed=1, batch=8, lo=512, hi=4096) -> np.ndarray:
    return np.random.default_rng(seed).integers(lo, hi + 1, size=batch).astype(np.int64)


def varlen_causal_prefill() -> PrefillInputs:
    """8 sequences, lengths uniform in [512, 4096], 32 heads MHA, d=128, causal."""
    return make_prefill(varlen_lengths(1), 32, 32, 128, causal=True, seed=1,
                        name="varlen_causal_prefill")


def long_gqa_prefill() -> PrefillInputs:
    """One 32768-token sequence, 32 query heads sharing 8 KV heads, d=128, causal."""
    return make_prefill([32768], 32, 8, 128, causal=True, seed=2, name="long_gqa_prefill")


# ---------------------------------------------------------------------------
# Paged decode workloads
# ---------------------------------------------------------------------------

@dataclass
class DecodeInputs:
    name: str
    q_bits: np.ndarray            # [B, Hq, d], or [B, q_len, Hq, d] for multi-token decode
    k_pages_bits: np.ndarray      # NHD: [P, page, Hkv, d]; HND: [P, Hkv, page, d]
    v_pages_bits: np.ndarray
    block_table: np.ndarray       # [B, max_pages] int32 (unused slots = -1)
    cache_seqlens: np.ndarray     # [B] int32
    scale: float
    layout: str = "NHD"
    page_size: int = PAGE_SIZE
    extra: dict = field(default_factory=dict)

    @property
    def batch(self):
        return self.q_bits.shape[0]

    @property
    def q_len(self):
        return self.q_bits.shape[1] if self.q_bits.ndim == 4 else 1

    @property
    def num_q_heads(self):
        return self.q_bits.shape[-2]

    @property
    def head_dim(self):
        return self.q_bits.shape[-1]

    @property
    def num_kv_heads(self):
        return self.k_pages_bits.shape[2] if self.layout == "NHD" else self.k_pages_bits.shape[1]

    @property
    def num_pages(self):
        return self.k_pages_bits.shape[0]

    def strides(self):
        """(page_stride, token_stride, head_stride) in elements."""
        P, a, b, d = self.k_pages_bits.shape
        if self.layout == "NHD":
            return a * b * d, b * d, d
        return a * b * d, d, b * d

    @property
    def kv_elem_bytes(self):
        """2 for a bf16 cache, 1 for an FP8 (E4M3) cache."""
        return self.k_pages_bits.dtype.itemsize

    def kv_bytes(self) -> float:
        """Bytes of K and V the decode must read: every cached token once."""
        return (2.0 * float(self.cache_seqlens.astype(np.int64).sum()) * self.num_kv_heads *
                self.head_dim * self.kv_elem_bytes)

    def algorithmic_bytes(self) -> float:
        """KV read once + q read + out/lse written + block_table entries used."""
        B, Hq, d = self.batch, self.num_q_heads, self.head_dim
        rows = B * self.q_len * Hq
        pages_used = int(np.sum((self.cache_seqlens.astype(np.int64) + self.page_size - 1) // self.page_size))
        return self.kv_bytes() + rows * d * 2 * 2 + rows * 4 + pages_used * 4 + B * 4


def make_decode(cache_seqlens, num_q_heads, num_kv_heads, head_dim, *, seed=3,
                page_size=PAGE_SIZE, layout="NHD", scale=None, extra_pages=0,
                name="decode", q_len=1) -> DecodeInputs:
    """Paged KV cache whose physical pages are a seeded random permutation.

    Request b owns ceil(seqlen_b / page_size) logical pages; the physical page
    for each logical page comes from a random permutation of the pool.  The pool
    is drawn i.i.d. N(0,1), which is the same distribution as drawing each
    request's logical K/V and scattering it.  ``extra_pages`` adds pool pages
    that no request uses.
    """
    cache_seqlens = np.asarray(cache_seqlens, dtype=np.int64)
    B = len(cache_seqlens)
    npages = (cache_seqlens + page_size - 1) // page_size
    total = int(npages.sum()) + int(extra_pages)
    ss = np.random.SeedSequence(seed)
    s_perm, s_q, s_k, s_v = ss.spawn(4)
    perm = np.random.Generator(np.random.PCG64(s_perm)).permutation(total).astype(np.int32)
    max_pages = int(max(1, npages.max()))
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(npages[b])
        bt[b, :n] = perm[off:off + n]
        off += n
    if layout == "NHD":
        shape = (total, page_size, num_kv_heads, head_dim)
    elif layout == "HND":
        shape = (total, num_kv_heads, page_size, head_dim)
    else:
        raise ValueError(layout)
    q_shape = (B, num_q_heads, head_dim) if q_len == 1 else (B, q_len, num_q_heads, head_dim)
    q = _normal_bf16_bits(s_q, q_shape)
    kp = _normal_bf16_bits(s_k, shape)
    vp = _normal_bf16_bits(s_v, shape)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return DecodeInputs(name, q, kp, vp, bt, cache_seqlens.astype(np.int32), float(scale),
                        layout, page_size)


def paged_decode_batch() -> DecodeInputs:
    """64 requests, cache lengths uniform in [1024, 32768], 32 q / 8 kv heads, d=128."""
    lens = np.random.default_rng(3).integers(1024, 32768 + 1, size=64)
    return make_decode(lens, 32, 8, 128, seed=3, name="paged_decode_batch")


def paged_decode_gqa8() -> DecodeInputs:
    """paged_decode_batch's lengths with 64 query heads over 8 kv heads (group 8)."""
    lens = np.random.default_rng(3).integers(1024, 32768 + 1, size=64)
    return make_decode(lens, 64, 8, 128, seed=8, name="paged_decode_gqa8")


def paged_decode_gqa16() -> DecodeInputs:
    """paged_decode_batch's lengths with 32 query heads over 2 kv heads (group 16)."""
    lens = np.random.default_rng(3).integers(1024, 32768 + 1, size=64)
    return make_decode(lens, 32, 2, 128, seed=16, name="paged_decode_gqa16")


def speculative_decode_batch() -> DecodeInputs:
    """paged_decode_batch's 64 requests with 4 query tokens each (multi-token
    decode, e.g. speculative verification), 32 q / 8 kv heads, d=128."""
    lens = np.random.default_rng(3).integers(1024, 32768 + 1, size=64)
    return make_decode(lens, 32, 8, 128, seed=17, q_len=4, name="speculative_decode_batch")


def paged_decode_batch16_lengths() -> np.ndarray:
    return np.random.default_rng(3).integers(1024, 32768 + 1, size=16)


def paged_decode_batch16() -> DecodeInputs:
    """Profiling-sized variant of the paged batch (16 requests, ~1 GB of KV):
    same length distribution and heads, small enough for multi-pass ncu."""
    return make_decode(paged_decode_batch16_lengths(), 32, 8, 128, seed=13, name="paged_decode_batch16")


def long_split_decode() -> DecodeInputs:
    """4 requests of 131072 cached tokens, 32 heads MHA, d=128, shuffled pages."""
    return make_decode([131072] * 4, 32, 32, 128, seed=4, name="long_split_decode")


def ragged_split_decode() -> DecodeInputs:
    """1 request at 131072 plus 63 at 2048 tokens, 32 heads MHA, d=128."""
    return make_decode([131072] + [2048] * 63, 32, 32, 128, seed=5, name="ragged_split_decode")


E4M3_MAX = 448.0


def quantize_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """Quantise x / scale to FP8 E4M3 codes (uint8): round to nearest even,
    saturating at +-448 (PyTorch's float8_e4m3fn cast after clipping)."""
    import torch
    y = np.clip(np.asarray(x, dtype=np.float32) / np.float32(scale), -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def to_fp8_cache(inp: DecodeInputs, amax: float = 4.0) -> DecodeInputs:
    """The same cache quantised to E4M3 with one scale per tensor:
    scale = amax / 448, so +-amax (4 standard deviations of the N(0,1) draws)
    spans the format's range.  Scales go in ``extra['k_scale'/'v_scale']``."""
    k_scale = v_scale = amax / E4M3_MAX
    kp = quantize_e4m3(bf16_bits_to_f32(inp.k_pages_bits), k_scale)
    vp = quantize_e4m3(bf16_bits_to_f32(inp.v_pages_bits), v_scale)
    extra = dict(inp.extra, k_scale=float(k_scale), v_scale=float(v_scale))
    return DecodeInputs(inp.name + "_fp8", inp.q_bits, kp, vp, inp.block_table, inp.cache_seqlens,
                        inp.scale, inp.layout, inp.page_size, extra)


def paged_decode_batch_fp8() -> DecodeInputs:
    """paged_decode_batch (64 requests, U[1024, 32768], 32 q / 8 kv heads,
    d=128) with its KV cache in FP8 E4M3, per-tensor scales."""
    return to_fp8_cache(paged_decode_batch())


@dataclass
class Fp8PrefillInputs(PrefillInputs):
    """A prefill workload in FP8 E4M3: q_bits / k_bits / v_bits hold uint8
    codes; the tensors are q_scale * E4M3(q8) and likewise for k and v."""
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0


def to_fp8_prefill(inp: PrefillInputs, amax: float = 4.0) -> Fp8PrefillInputs:
    """The same prefill inputs quantised to E4M3, one scale per tensor
    (scale = amax / 448, as for the FP8 cache)."""
    s = amax / E4M3_MAX
    q8, k8, v8 = (quantize_e4m3(bf16_bits_to_f32(x), s) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    return Fp8PrefillInputs(inp.name + "_fp8", q8, k8, v8, inp.cu_seqlens, inp.causal, inp.scale,
                            None, float(s), float(s), float(s))


def varlen_causal_prefill_fp8() -> Fp8PrefillInputs:
    """varlen_causal_prefill (8 sequences in [512, 4096], 32 heads, d=128,
    causal) with Q, K and V in FP8 E4M3, per-tensor scales."""
    return to_fp8_prefill(varlen_causal_prefill())


def relayout(inp: DecodeInputs, layout: str) -> DecodeInputs:
    """Same cache contents in the other page layout (NHD <-> HND)."""
    if layout == inp.layout:
        return inp
    kp = np.ascontiguousarray(np.swapaxes(inp.k_pages_bits, 1, 2))
    vp = np.ascontiguousarray(np.swapaxes(inp.v_pages_bits, 1, 2))
    return DecodeInputs(inp.name + "_" + layout, inp.q_bits, kp, vp, inp.block_table,
                        inp.cache_seqlens, inp.scale, layout, inp.page_size, dict(inp.extra))


def permute_pages(inp: DecodeInputs, seed: int) -> DecodeInputs:
    """Move every physical page to a new random slot and rewrite the block table."""
    P = inp.num_pages
    perm = np.random.default_rng(seed).permutation(P).astype(np.int32)   # old -> new
    kp = np.empty_like(inp.k_pages_bits)
    vp = np.empty_like(inp.v_pages_bits)
    kp[perm] = inp.k_pages_bits
    vp[perm] = inp.v_pages_bits
    bt = inp.block_table.copy()
    used = bt >= 0
    bt[used] = perm[bt[used]]
    return DecodeInputs(inp.name + "_perm", inp.q_bits, kp, vp, bt, inp.cache_seqlens,
                        inp.scale, inp.layout, inp.page_size, dict(inp.extra))


BF16_NAN_BITS = 0x7FC0
E4M3_NAN_BITS = 0x7F


def poison_unused(inp: DecodeInputs) -> DecodeInputs:
    """Fill every cache slot no request reads (page tails, unused pages) with NaN."""
    kp = inp.k_pages_bits.copy()
    vp = inp.v_pages_bits.copy()
    P = inp.num_pages
    ps = inp.page_size
    valid = np.zeros((P, ps), dtype=bool)
    for b in range(inp.batch):
        L = int(inp.cache_seqlens[b])
        for p in range((L + ps - 1) // ps):
            phys = int(inp.block_table[b, p])
            n = min(ps, L - p * ps)
            valid[phys, :n] = True
    inv = ~valid
    nan = E4M3_NAN_BITS if kp.dtype == np.uint8 else BF16_NAN_BITS
    if inp.layout == "NHD":
        kp[inv] = nan
        vp[inv] = nan
    else:
        kp.transpose(0, 2, 1, 3)[inv] = nan
        vp.transpose(0, 2, 1, 3)[inv] = nan
    return DecodeInputs(inp.name + "_poison", inp.q_bits, kp, vp, inp.block_table,
                        inp.cache_seqlens, inp.scale, inp.layout, inp.page_size, dict(inp.extra))


# ---------------------------------------------------------------------------
# Chunked (paged) prefill workloads
# ---------------------------------------------------------------------------

@dataclass
class ChunkedPrefillInputs:
    """A batch of prefill chunks over paged caches that already hold a prefix.

    Request b has ``prefix_lens[b]`` cached tokens in its pages and a new chunk
    of ``chunk_lens[b]`` tokens: its queries (``q_bits``) and its K/V rows
    (``k_new_bits``/``v_new_bits``), all packed by ``cu_seqlens_q``.  The pages
    already reserve room for the chunk (``cache_seqlens`` = prefix + chunk, the
    length after the append); the chunk's slots hold stale values until the
    append writes them.
    """
    name: str
    q_bits: np.ndarray            # [Tq, Hq, d]
    k_new_bits: np.ndarray        # [Tq, Hkv, d]
    v_new_bits: np.ndarray
    cu_seqlens_q: np.ndarray      # [B+1] int32
    k_pages_bits: np.ndarray      # NHD [P, page, Hkv, d] or HND [P, Hkv, page, d]
    v_pages_bits: np.ndarray
    block_table: np.ndarray       # [B, max_pages] int32 (unused = -1)
    cache_seqlens: np.ndarray     # [B] int32, after the append
    causal: bool
    scale: float
    layout: str = "NHD"
    page_size: int = PAGE_SIZE

    @property
    def batch(self):
        return len(self.cache_seqlens)

    @property
    def num_q_heads(self):
        return self.q_bits.shape[1]

    @property
    def num_kv_heads(self):
        return self.k_new_bits.shape[1]

    @property
    def head_dim(self):
        return self.q_bits.shape[2]

    @property
    def num_pages(self):
        return self.k_pages_bits.shape[0]

    @property
    def chunk_lens(self):
        return np.diff(self.cu_seqlens_q).astype(np.int64)

    @property
    def prefix_lens(self):
        return self.cache_seqlens.astype(np.int64) - self.chunk_lens

    def strides(self):
        """(page_stride, token_stride, head_stride) in elements."""
        P, a, b, d = self.k_pages_bits.shape
        if self.layout == "NHD":
            return a * b * d, b * d, d
        return a * b * d, d, b * d

    def causal_flops(self) -> float:
        """Algorithmic FLOPs: 4*d*Hq per (query, visible key) pair."""
        n = self.chunk_lens
        k = self.cache_seqlens.astype(np.int64)
        pairs = (n * (k - n) + n * (n + 1) // 2).sum() if self.causal else (n * k).sum()
        return 4.0 * self.head_dim * self.num_q_heads * float(pairs)

    def append_bytes(self) -> float:
        """KV append traffic: the new K and V rows read once and written once."""
        return 4.0 * self.k_new_bits.size * 2

    def attention_bytes(self) -> float:
        """Minimum HBM bytes of the attention: Q read, O written, every cached
        K/V row of each kv head read once."""
        Tq, Hq, d = self.q_bits.shape
        kv = 2.0 * float(self.cache_seqlens.astype(np.int64).sum()) * self.num_kv_heads * d * 2
        return kv + 2.0 * Tq * Hq * d * 2 + Tq * Hq * 4


def make_chunked_prefill(prefix_lens, chunk_lens, num_q_heads, num_kv_heads, head_dim, *,
                         seed=6, causal=True, page_size=PAGE_SIZE, layout="NHD", scale=None,
                         extra_pages=0, name="chunked_prefill") -> ChunkedPrefillInputs:
    prefix_lens = np.asarray(prefix_lens, dtype=np.int64)
    chunk_lens = np.asarray(chunk_lens, dtype=np.int64)
    assert prefix_lens.shape == chunk_lens.shape and (chunk_lens >= 1).all()
    total = prefix_lens + chunk_lens
    B = len(total)
    npages = (total + page_size - 1) // page_size
    P = int(npages.sum()) + int(extra_pages)
    ss = np.random.SeedSequence(seed)
    s_perm, s_q, s_kn, s_vn, s_k, s_v = ss.spawn(6)
    perm = np.random.Generator(np.random.PCG64(s_perm)).permutation(P).astype(np.int32)
    bt = np.full((B, int(max(1, npages.max()))), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(npages[b])
        bt[b, :n] = perm[off:off + n]
        off += n
    if layout == "NHD":
        shape = (P, page_size, num_kv_heads, head_dim)
    elif layout == "HND":
        shape = (P, num_kv_heads, page_size, head_dim)
    else:
        raise ValueError(layout)
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(chunk_lens)
    Tq = int(cu[-1])
    q = _normal_bf16_bits(s_q, (Tq, num_q_heads, head_dim))
    kn = _normal_bf16_bits(s_kn, (Tq, num_kv_heads, head_dim))
    vn = _normal_bf16_bits(s_vn, (Tq, num_kv_heads, head_dim))
    kp = _normal_bf16_bits(s_k, shape)
    vp = _normal_bf16_bits(s_v, shape)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return ChunkedPrefillInputs(name, q, kn, vn, cu, kp, vp, bt, total.astype(np.int32), causal,
                                float(scale), layout, page_size)


def tiny_chunked_prefill(head_dim=128, layout="NHD", causal=True) -> ChunkedPrefillInputs:
    """Five requests whose (prefix, chunk) pairs cover an empty prefix, a
    one-token chunk, page-aligned ends and page tails in either half of a
    128-key tile; 4 q / 2 kv heads."""
    return make_chunked_prefill([0, 100, 700, 64, 1000], [130, 1, 257, 64, 300], 4, 2, head_dim,
                                seed=7, causal=causal, layout=layout, extra_pages=3,
                                name="tiny_chunked_prefill")


def chunked_prefill_lengths(seed=6, batch=8):
    g = np.random.default_rng(seed)
    prefix = g.integers(1024, 16384 + 1, size=batch)
    chunk = g.integers(256, 2048 + 1, size=batch)
    return prefix.astype(np.int64), chunk.astype(np.int64)


def chunked_prefill_batch() -> ChunkedPrefillInputs:
    """8 requests, cached prefix uniform in [1024, 16384], new chunk uniform in
    [256, 2048], 32 q / 8 kv heads, d=128, causal, shuffled 64-token pages."""
    prefix, chunk = chunked_prefill_lengths(6)
    return make_chunked_prefill(prefix, chunk, 32, 8, 128, seed=6, name="chunked_prefill_batch")


def poison_chunked(inp: ChunkedPrefillInputs) -> ChunkedPrefillInputs:
    """NaN in every pool slot outside the cached prefixes: the chunk's own
    slots (the append must overwrite them), page tails and unused pages."""
    kp = inp.k_pages_bits.copy()
    vp = inp.v_pages_bits.copy()
    ps = inp.page_size
    valid = np.zeros((inp.num_pages, ps), dtype=bool)
    for b in range(inp.batch):
        L = int(inp.prefix_lens[b])
        for p in range((L + ps - 1) // ps):
            valid[int(inp.block_table[b, p]), :min(ps, L - p * ps)] = True
    inv = ~valid
    if inp.layout == "NHD":
        kp[inv] = BF16_NAN_BITS
        vp[inv] = BF16_NAN_BITS
    else:
        kp.transpose(0, 2, 1, 3)[inv] = BF16_NAN_BITS
        vp.transpose(0, 2, 1, 3)[inv] = BF16_NAN_BITS
    out = ChunkedPrefillInputs(**{**inp.__dict__})
    out.name = inp.name + "_poison"
    out.k_pages_bits, out.v_pages_bits = kp, vp
    return out


# ---------------------------------------------------------------------------
# Cascade (shared-prefix) decode workloads
# ---------------------------------------------------------------------------

@dataclass
class CascadeInputs:
    """Decode where every request shares one prefix (its pages listed once in
    ``prefix_block_table``) and then has its own suffix (``block_table`` rows,
    ``suffix_lens``)."""
    name: str
    q_bits: np.ndarray            # [B, Hq, d]
    k_pages_bits: np.ndarray      # NHD [P, page, Hkv, d] or HND [P, Hkv, page, d]
    v_pages_bits: np.ndarray
    prefix_block_table: np.ndarray   # [ceil(prefix_len / page)] int32
    prefix_len: int
    block_table: np.ndarray       # [B, max_suffix_pages] int32 (unused = -1)
    suffix_lens: np.ndarray       # [B] int32
    scale: float
    layout: str = "NHD"
    page_size: int = PAGE_SIZE

    @property
    def batch(self):
        return self.q_bits.shape[0]

    @property
    def num_q_heads(self):
        return self.q_bits.shape[1]

    @property
    def head_dim(self):
        return self.q_bits.shape[2]

    @property
    def num_kv_heads(self):
        return self.k_pages_bits.shape[2] if self.layout == "NHD" else self.k_pages_bits.shape[1]

    def strides(self):
        P, a, b, d = self.k_pages_bits.shape
        if self.layout == "NHD":
            return a * b * d, b * d, d
        return a * b * d, d, b * d

    def algorithmic_bytes(self) -> float:
        """The shared prefix's K/V once, every suffix's K/V once, q and out."""
        B, Hq, d = self.q_bits.shape
        tokens = self.prefix_len + float(self.suffix_lens.astype(np.int64).sum())
        return 2.0 * tokens * self.num_kv_heads * d * 2 + B * Hq * d * 2 * 2 + B * Hq * 4

    def as_plain_decode(self) -> "DecodeInputs":
        """The same contexts as a plain paged decode (each request's table row =
        prefix pages then suffix pages); needs a page-aligned prefix."""
        assert self.prefix_len % self.page_size == 0
        n_pre = len(self.prefix_block_table)
        bt = np.full((self.batch, n_pre + self.block_table.shape[1]), -1, dtype=np.int32)
        bt[:, :n_pre] = self.prefix_block_table
        bt[:, n_pre:] = self.block_table
        return DecodeInputs(self.name + "_plain", self.q_bits, self.k_pages_bits, self.v_pages_bits,
                            bt, (self.suffix_lens + self.prefix_len).astype(np.int32), self.scale,
                            self.layout, self.page_size)


def make_cascade(prefix_len, suffix_lens, num_q_heads, num_kv_heads, head_dim, *, seed=21,
                 layout="NHD", extra_pages=0, name="cascade") -> CascadeInputs:
    suffix_lens = np.asarray(suffix_lens, dtype=np.int64)
    B = len(suffix_lens)
    ps = PAGE_SIZE
    n_pre = (int(prefix_len) + ps - 1) // ps
    n_suf = (suffix_lens + ps - 1) // ps
    P = n_pre + int(n_suf.sum()) + int(extra_pages)
    ss = np.random.SeedSequence(seed)
    s_perm, s_q, s_k, s_v = ss.spawn(4)
    perm = np.random.Generator(np.random.PCG64(s_perm)).permutation(P).astype(np.int32)
    pre_bt = perm[:n_pre].copy()
    bt = np.full((B, int(max(1, n_suf.max()))), -1, dtype=np.int32)
    off = n_pre
    for b in range(B):
        bt[b, :n_suf[b]] = perm[off:off + n_suf[b]]
        off += int(n_suf[b])
    shape = (P, ps, num_kv_heads, head_dim) if layout == "NHD" else (P, num_kv_heads, ps, head_dim)
    q = _normal_bf16_bits(s_q, (B, num_q_heads, head_dim))
    kp = _normal_bf16_bits(s_k, shape)
    vp = _normal_bf16_bits(s_v, shape)
    return CascadeInputs(name, q, kp, vp, pre_bt, int(prefix_len), bt, suffix_lens.astype(np.int32),
                         1.0 / math.sqrt(head_dim), layout, ps)


def cascade_decode_batch() -> CascadeInputs:
    """64 requests sharing an 8192-token prefix, own suffixes U[64, 2048],
    32 q / 8 kv heads, d=128, shuffled pages."""
    suf = np.random.default_rng(21).integers(64, 2048 + 1, size=64)
    return make_cascade(8192, suf, 32, 8, 128, seed=21, name="cascade_decode_batch")


CONFIGS = {
    "tiny_causal_prefill": tiny_causal_prefill,
    "varlen_causal_prefill": varlen_causal_prefill,
    "long_gqa_prefill": long_gqa_prefill,
    "paged_decode_batch": paged_decode_batch,
    "paged_decode_batch16": paged_decode_batch16,
    "long_split_decode": long_split_decode,
    "ragged_split_decode": ragged_split_decode,
    "paged_decode_batch_fp8": paged_decode_batch_fp8,
    "varlen_causal_prefill_fp8": varlen_causal_prefill_fp8,
    "paged_decode_gqa8": paged_decode_gqa8,
    "paged_decode_gqa16": paged_decode_gqa16,
    "speculative_decode_batch": speculative_decode_batch,
    "cascade_decode_batch": cascade_decode_batch,
    "tiny_chunked_prefill": tiny_chunked_prefill,
    "chunked_prefill_batch": chunked_prefill_batch,
}
