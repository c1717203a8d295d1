"""Helpers shared by the GPU parity tests: move seeded inputs to the device
and compare results with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np

import workloads as W

# Tolerances for bf16 inputs/outputs with fp32 accumulation against the fp64
# oracle (O max-abs, O mean-abs, LSE abs).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32))).cuda()


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Assert the bf16/fp32 GPU result matches the fp64 oracle; returns errors."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: O max-abs {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: O mean-abs {mean:.3e} > {O_MEAN_ABS}"
    lerr = 0.0
    if lse_ref is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        both_inf = np.isneginf(lse_gpu) & np.isneginf(lse_ref)
        with np.errstate(invalid="ignore"):
            d = np.where(both_inf, 0.0, np.abs(lse_gpu - lse_ref))
        lerr = float(np.nanmax(d)) if d.size else 0.0
        assert not np.isnan(d).any(), f"{what}: NaN LSE"
        assert lerr <= LSE_ABS, f"{what}: LSE abs {lerr:.3e} > {LSE_ABS}"
    return mx, mean, lerr


def prefill_on_gpu(inp: W.PrefillInputs, **kw):
    import exact_attention_148_b200 as fa
    q, k, v = (to_dev_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    cu = to_dev_i32(inp.cu_seqlens)
    return fa.prefill(q, k, v, cu, causal=inp.causal, scale=inp.scale,
                      cu_seqlens_host=inp.cu_seqlens, **kw)


def decode_on_gpu(inp: W.DecodeInputs, num_splits=0, plan=None, dev=None, kernel="auto", **kw):
    import exact_attention_148_b200 as fa
    if dev is None:
        dev = decode_device_inputs(inp)
    if plan is None:
        plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=inp.num_q_heads,
                              num_kv_heads=inp.num_kv_heads, head_dim=inp.head_dim,
                              page_size=inp.page_size, max_pages_per_seq=inp.block_table.shape[1],
                              num_splits=num_splits, kernel=kernel)
    out, lse = fa.decode_paged(dev["q"], dev["k"], dev["v"], dev["bt"], dev["lens"], plan,
                               layout=inp.layout, scale=inp.scale, **kw)
    return out, lse, plan


def decode_device_inputs(inp: W.DecodeInputs):
    return dict(q=to_dev_bf16(inp.q_bits), k=to_dev_bf16(inp.k_pages_bits),
                v=to_dev_bf16(inp.v_pages_bits), bt=to_dev_i32(inp.block_table),
                lens=to_dev_i32(inp.cache_seqlens))


def chunked_device_inputs(inp: W.ChunkedPrefillInputs):
    return dict(q=to_dev_bf16(inp.q_bits), k_new=to_dev_bf16(inp.k_new_bits),
                v_new=to_dev_bf16(inp.v_new_bits), cu=to_dev_i32(inp.cu_seqlens_q),
                k=to_dev_bf16(inp.k_pages_bits), v=to_dev_bf16(inp.v_pages_bits),
                bt=to_dev_i32(inp.block_table), lens=to_dev_i32(inp.cache_seqlens))


def chunked_on_gpu(inp: W.ChunkedPrefillInputs, dev=None, append=True, **kw):
    """KV append (optional) then chunked prefill over the paged cache."""
    import exact_attention_148_b200 as fa
    if dev is None:
        dev = chunked_device_inputs(inp)
    if append:
        fa.append_kv(dev["k_new"], dev["v_new"], dev["cu"], dev["k"], dev["v"], dev["bt"],
                     dev["lens"], layout=inp.layout)
    out, lse = fa.prefill_paged(dev["q"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"],
                                causal=inp.causal, scale=inp.scale, layout=inp.layout,
                                cu_seqlens_q_host=inp.cu_seqlens_q,
                                cache_seqlens_host=inp.cache_seqlens, **kw)
    return out, lse, dev


def oracle_pool_after_append(inp: W.ChunkedPrefillInputs):
    """Page pool bits after the oracle's append (bit patterns, no arithmetic)."""
    import oracle
    return oracle.append_kv_ref(inp.k_pages_bits, inp.v_pages_bits, inp.k_new_bits, inp.v_new_bits,
                                inp.cu_seqlens_q, inp.block_table, inp.cache_seqlens,
                                inp.page_size, inp.layout)


def jumping_keys(inp, factors, tile=128):
    """inp with the key rows of key tile t of every sequence multiplied by
    factors[t % len(factors)]: scores that jump far above (or below) the
    earlier tiles' from one key tile to the next."""
    import workloads as W
    k = W.bf16_bits_to_f32(inp.k_bits).copy()
    cu = inp.cu_seqlens
    for b in range(len(cu) - 1):
        for t0 in range(int(cu[b]), int(cu[b + 1]), tile):
            k[t0:min(t0 + tile, int(cu[b + 1]))] *= factors[((t0 - int(cu[b])) // tile) % len(factors)]
    inp.k_bits = W.f32_to_bf16_bits(k)
    return inp


# Per-tile key scales: x8 lifts a tile's scores ~30 (base 2) above the first
# tile's (past the rescale threshold, under the bf16 overflow guard of 64),
# x25 and x40 by 65-75 more (past the guard).  Scores stay near 120, where
# fp32 scores still meet the LSE bound.
JUMP_FACTORS = [1.0, 8.0, 1.0, 25.0, 3.0, 40.0, 0.5, 12.0]


def jumping_keys_paged(inp, factors, tile=128):
    """A ChunkedPrefillInputs with the key at logical position t of every
    request multiplied by factors[(t // tile) % len(factors)]: the cached
    prefix in the page pool and the chunk's own new rows alike (NHD or HND)."""
    import workloads as W
    kp = W.bf16_bits_to_f32(inp.k_pages_bits).copy()
    kn = W.bf16_bits_to_f32(inp.k_new_bits).copy()
    ps = inp.page_size
    prefix = inp.prefix_lens
    for b in range(inp.batch):
        for t in range(int(prefix[b])):
            f = factors[(t // tile) % len(factors)]
            page, slot = int(inp.block_table[b, t // ps]), t % ps
            if inp.layout == "NHD":
                kp[page, slot] *= f
            else:
                kp[page, :, slot] *= f
        for i in range(int(inp.chunk_lens[b])):
            t = int(prefix[b]) + i
            kn[int(inp.cu_seqlens_q[b]) + i] *= factors[(t // tile) % len(factors)]
    inp.k_pages_bits = W.f32_to_bf16_bits(kp)
    inp.k_new_bits = W.f32_to_bf16_bits(kn)
    return inp


def jumping_keys_decode(inp, factors, tile=128):
    """A DecodeInputs with the cached key at logical position t of every
    request multiplied by factors[(t // tile) % len(factors)] (NHD or HND pool)."""
    import workloads as W
    kp = W.bf16_bits_to_f32(inp.k_pages_bits).copy()
    ps = inp.page_size
    for b in range(inp.batch):
        L = int(inp.cache_seqlens[b])
        for t0 in range(0, L, ps):
            page = int(inp.block_table[b, t0 // ps])
            for t in range(t0, min(t0 + ps, L)):
                f = factors[(t // tile) % len(factors)]
                if inp.layout == "NHD":
                    kp[page, t - t0] *= f
                else:
                    kp[page, :, t - t0] *= f
    inp.k_pages_bits = W.f32_to_bf16_bits(kp)
    return inp
