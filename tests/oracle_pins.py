"""Checks that tie the CPU oracle to facts outside itself.

Each ``pin_*`` takes the oracle function(s) under test as arguments and raises
``AssertionError`` when the oracle disagrees with the fact.  ``test_oracle_pins``
runs them on the real oracle; ``test_oracle_mutants`` runs them on oracles with
a planted mistake and expects at least one pin to fire.
"""
from __future__ import annotations

import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    same_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    err = np.where(same_inf, 0.0, np.abs(a - b))
    m = float(np.max(err)) if err.size else 0.0
    assert m <= tol, f"{what}: max abs err {m:.3e} > {tol:.1e}"


# --- golden fixtures (hand-derived closed forms) ----------------------------

def pin_golden_two_keys(attention_ref):
    g = load_golden("two_keys_prefill.json")
    q, k, v = (np.array(g[x]) for x in ("q", "k", "v"))
    for mode in ("noncausal", "causal"):
        o, l = attention_ref(q, k, v, g["cu_seqlens"], mode == "causal", g["scale"])
        _close(o, g[mode]["o"], 1e-13, f"two_keys {mode} O")
        _close(l, g[mode]["lse"], 1e-13, f"two_keys {mode} LSE")


def pin_golden_causal_uniform(attention_ref):
    g = load_golden("causal_uniform.json")
    q, k, v = (np.array(g[x]) for x in ("q", "k", "v"))
    o, l = attention_ref(q, k, v, g["cu_seqlens"], True, g["scale"])
    _close(o, g["causal"]["o"], 1e-13, "causal_uniform O")
    _close(l, g["causal"]["lse"], 1e-13, "causal_uniform LSE")


def pin_golden_merge(merge_states_ref):
    g = load_golden("merge_two_states.json")
    o_parts = np.array(g["o_parts"])
    lse_parts = np.array(g["lse_parts"])
    o, l = merge_states_ref(o_parts, lse_parts)
    _close(o, g["o"], 1e-13, "merge O")
    _close(l, g["lse"], 1e-13, "merge LSE")
    # an empty state carries no weight
    o2, l2 = merge_states_ref(np.concatenate([o_parts, [[9.0, 9.0]]]),
                              np.concatenate([lse_parts, [-np.inf]]))
    _close(o2, g["o"], 1e-13, "merge+empty O")
    _close(l2, g["lse"], 1e-13, "merge+empty LSE")
    # a large common shift must not overflow
    o3, l3 = merge_states_ref(o_parts, lse_parts + 1000.0)
    _close(o3, g["o"], 1e-12, "merge shifted O")
    _close(l3, g["lse"] + 1000.0, 1e-9, "merge shifted LSE")
    # all states empty -> O = 0, LSE = -inf
    o4, l4 = merge_states_ref(o_parts, np.array([-np.inf, -np.inf]))
    _close(o4, [0.0, 0.0], 0.0, "merge all-empty O")
    assert np.isneginf(l4), "merge all-empty LSE must be -inf"


def pin_golden_paged(paged_decode_ref):
    g = load_golden("paged_walk.json")
    o, l = paged_decode_ref(np.array(g["q"]), np.array(g["k_pages"]), np.array(g["v_pages"]),
                            np.array(g["block_table"]), np.array(g["cache_seqlens"]), g["scale"],
                            page_size=g["page_size"], layout="NHD")
    _close(o, g["o"], 1e-13, "paged O")
    _close(l, g["lse"], 1e-13, "paged LSE")


# --- invariants and closed forms ----------------------------------------------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_rows_sum_to_one(attention_probs_ref, causal=True):
    q = _rand((23, 2, 8), 11)
    k = _rand((23, 2, 8), 12)
    cu = [0, 7, 23]
    for P in attention_probs_ref(q, k, cu, causal):
        _close(P.sum(axis=1), np.ones(P.shape[0]), 1e-12, "softmax row sums")
        assert np.all(P >= 0), "negative softmax weight"
        if causal:
            assert np.all(np.triu(P, 1) == 0), "weight on a masked (future) key"


def pin_identical_keys(attention_ref, causal):
    """All keys equal: every allowed key has the same score s = scale q.k, so
    O = mean(V over allowed keys) and LSE = s + ln(n_allowed)."""
    T, H, d = 13, 1, 6
    q = _rand((T, H, d), 21)
    kk = _rand((d,), 22)
    k = np.broadcast_to(kk, (T, H, d)).copy()
    v = _rand((T, H, d), 23)
    scale = 0.37
    o, l = attention_ref(q, k, v, [0, T], causal, scale)
    for i in range(T):
        n = i + 1 if causal else T
        _close(o[i, 0], v[:n, 0].mean(axis=0), 1e-12, f"identical keys O row {i}")
        _close(l[i, 0], scale * q[i, 0] @ kk + math.log(n), 1e-12, f"identical keys LSE row {i}")


def pin_dominant_key(attention_ref):
    """One key whose score exceeds all others by >= 50 returns its V row."""
    T, d = 9, 4
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((T, 1, d))
    k[:, 0, 0] = np.linspace(-3, 3, T)
    k[5, 0, 0] = 60.0
    v = _rand((T, 1, d), 31)
    qq = np.concatenate([np.zeros((T - 1, 1, d)), q], axis=0)   # query at the last row
    o, l = attention_ref(qq, k, v, [0, T], True, 1.0)
    _close(o[T - 1, 0], v[5, 0], 1e-15 * 10, "dominant key O")


def pin_causal_row0(attention_ref):
    """Causal row 0 of every sequence sees only key 0: O = V[0], LSE = scale q0.k0."""
    q = _rand((20, 3, 5), 41)
    k = _rand((20, 3, 5), 42)
    v = _rand((20, 3, 5), 43)
    cu = [0, 6, 20]
    o, l = attention_ref(q, k, v, cu, True, 0.8)
    for s0 in cu[:-1]:
        for h in range(3):
            _close(o[s0, h], v[s0, h], 1e-14, "causal row0 O")
            _close(l[s0, h], 0.8 * q[s0, h] @ k[s0, h], 1e-14, "causal row0 LSE")


def pin_partition_merge(partial_state_ref, merge_states_ref, attention_rows_ref, seed=51):
    """Any partition of the keys, each split reduced to (O_i, LSE_i) and merged
    by LSE, reproduces the unsplit result."""
    g = np.random.default_rng(seed)
    L, d = 37, 6
    q = g.standard_normal((1, 1, d))
    k = g.standard_normal((L, 1, d))
    v = g.standard_normal((L, 1, d))
    o_ref, l_ref = attention_rows_ref(np.concatenate([np.zeros((L - 1, 1, d)), q]), k, v,
                                      [0, L], False, 0.5, [(L - 1, 0)])
    for trial in range(5):
        labels = g.integers(0, 4, size=L)      # arbitrary, non-contiguous partition
        os_, ls_ = [], []
        for part in range(5):                  # part 4 is always empty
            idx = np.nonzero(labels == part)[0]
            o_i, l_i = partial_state_ref(q[0], k[idx, 0], v[idx, 0], 0.5)
            os_.append(o_i[0])
            ls_.append(l_i[0])
        o, l = merge_states_ref(np.array(os_), np.array(ls_))
        _close(o, o_ref[0], 1e-12, "partition merge O")
        _close(l, l_ref[0], 1e-12, "partition merge LSE")


def _decimal_attention(q, k, v, causal, scale, digits=40):
    """Brute force with 40-digit decimal arithmetic, written without max
    subtraction: O_i = sum_j e^{s_ij} v_j / sum_j e^{s_ij}, LSE_i = ln sum_j e^{s_ij}."""
    getcontext().prec = digits
    T, d = q.shape
    sc = Decimal(repr(scale))
    O = np.zeros((T, v.shape[1]))
    LSE = np.zeros(T)
    for i in range(T):
        num = [Decimal(0)] * v.shape[1]
        den = Decimal(0)
        for j in range(T):
            if causal and j > i:
                continue
            s = sum((Decimal(repr(float(q[i, c]))) * Decimal(repr(float(k[j, c])))
                     for c in range(d)), Decimal(0)) * sc
            e = s.exp()
            den += e
            for c in range(v.shape[1]):
                num[c] += e * Decimal(repr(float(v[j, c])))
        for c in range(v.shape[1]):
            O[i, c] = float(num[c] / den)
        LSE[i] = float(den.ln())
    return O, LSE


def pin_bruteforce(attention_ref, T=4, dk=4, dv=4, seed=61):
    g = np.random.default_rng(seed)
    q = g.standard_normal((T, dk))
    k = g.standard_normal((T, dk))
    v = g.standard_normal((T, dv))
    for causal in (False, True):
        o, l = attention_ref(q[:, None], k[:, None], v[:, None], [0, T], causal, 0.7)
        ob, lb = _decimal_attention(q, k, v, causal, 0.7)
        _close(o[:, 0], ob, 1e-13, f"brute force O causal={causal}")
        _close(l[:, 0], lb, 1e-13, f"brute force LSE causal={causal}")


def pin_sdpa(attention_ref, seqlens=(5, 17, 9), hq=4, hkv=2, d=8, seed=71):
    """PyTorch CPU scaled_dot_product_attention in float64, one sequence at a
    time (is_causal is top-left aligned for equal q/k lengths; enable_gqa maps
    query head h to kv head h // (Hq/Hkv))."""
    import torch
    import torch.nn.functional as F

    g = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    T = int(cu[-1])
    q = g.standard_normal((T, hq, d))
    k = g.standard_normal((T, hkv, d))
    v = g.standard_normal((T, hkv, d))
    for causal in (False, True):
        o, _ = attention_ref(q, k, v, cu, causal, 0.3)
        for b in range(len(seqlens)):
            s0, s1 = int(cu[b]), int(cu[b + 1])
            tq = torch.from_numpy(q[s0:s1]).permute(1, 0, 2)[None]
            tk = torch.from_numpy(k[s0:s1]).permute(1, 0, 2)[None]
            tv = torch.from_numpy(v[s0:s1]).permute(1, 0, 2)[None]
            ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.3,
                                                 enable_gqa=True)
            _close(o[s0:s1], ref[0].permute(1, 0, 2).numpy(), 1e-12, f"sdpa seq {b} causal={causal}")


def pin_gqa_replication(attention_ref):
    """GQA equals MHA with each kv head repeated for its group of query heads."""
    q = _rand((15, 8, 4), 81)
    k = _rand((15, 2, 4), 82)
    v = _rand((15, 2, 4), 83)
    o1, l1 = attention_ref(q, k, v, [0, 6, 15], True, 0.5)
    o2, l2 = attention_ref(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), [0, 6, 15], True, 0.5)
    _close(o1, o2, 1e-14, "gqa vs repeated-mha O")
    _close(l1, l2, 1e-14, "gqa vs repeated-mha LSE")


def pin_varlen_packing(attention_ref):
    """Packing several sequences equals running each one alone."""
    q = _rand((30, 2, 4), 91)
    k = _rand((30, 2, 4), 92)
    v = _rand((30, 2, 4), 93)
    cu = [0, 11, 12, 30]
    o, l = attention_ref(q, k, v, cu, True, 0.5)
    for b in range(3):
        s0, s1 = cu[b], cu[b + 1]
        ob, lb = attention_ref(q[s0:s1], k[s0:s1], v[s0:s1], [0, s1 - s0], True, 0.5)
        _close(o[s0:s1], ob, 1e-14, "varlen packing O")
        _close(l[s0:s1], lb, 1e-14, "varlen packing LSE")


def pin_decode_walk(paged_decode_ref, partial_state_ref, layout="NHD", seed=101):
    """Scatter contiguous K/V into shuffled pages by hand; the paged decode must
    equal attention of each query row over the contiguous keys."""
    g = np.random.default_rng(seed)
    B, hq, hkv, d, ps = 3, 4, 2, 5, 4
    lens = [9, 1, 16]
    npages = [(L + ps - 1) // ps for L in lens]
    P = sum(npages) + 2
    perm = g.permutation(P)
    shape = (P, ps, hkv, d) if layout == "NHD" else (P, hkv, ps, d)
    kp = g.standard_normal(shape)
    vp = g.standard_normal(shape)
    bt = np.full((B, max(npages)), -1)
    q = g.standard_normal((B, hq, d))
    contig = []
    off = 0
    for b, L in enumerate(lens):
        K = g.standard_normal((L, hkv, d))
        V = g.standard_normal((L, hkv, d))
        contig.append((K, V))
        for t in range(L):
            phys = perm[off + t // ps]
            bt[b, t // ps] = phys
            if layout == "NHD":
                kp[phys, t % ps] = K[t]
                vp[phys, t % ps] = V[t]
            else:
                kp[phys, :, t % ps] = K[t]
                vp[phys, :, t % ps] = V[t]
        off += npages[b]
    o, l = paged_decode_ref(q, kp, vp, bt, lens, 0.6, page_size=ps, layout=layout)
    for b in range(B):
        K, V = contig[b]
        for h in range(hq):
            gh = h // (hq // hkv)
            ob, lb = partial_state_ref(q[b, h][None], K[:, gh], V[:, gh], 0.6)
            _close(o[b, h], ob[0], 1e-13, f"decode walk O b={b} h={h}")
            _close(l[b, h], lb[0], 1e-13, f"decode walk LSE b={b} h={h}")


# --- chunked (paged) prefill and KV append ----------------------------------

def pin_golden_append(append_kv_ref):
    g = load_golden("chunked_prefill_append.json")
    kp, vp = append_kv_ref(np.array(g["k_pages_before"]), np.array(g["v_pages_before"]),
                           np.array(g["k_new"]), np.array(g["v_new"]), g["cu_seqlens_new"],
                           np.array(g["block_table"]), g["cache_seqlens"], page_size=g["page_size"])
    _close(kp, g["k_pages_after"], 0.0, "append K pages")
    _close(vp, g["v_pages_after"], 0.0, "append V pages")


def pin_golden_chunked(paged_prefill_ref):
    g = load_golden("chunked_prefill_append.json")
    for mode in ("causal", "noncausal"):
        o, l = paged_prefill_ref(np.array(g["q"]), g["cu_seqlens_q"], np.array(g["k_pages_after"]),
                                 np.array(g["v_pages_after"]), np.array(g["block_table"]),
                                 g["cache_seqlens"], mode == "causal", g["scale"],
                                 page_size=g["page_size"])
        _close(o, g[mode]["o"], 1e-13, f"chunked {mode} O")
        _close(l, g[mode]["lse"], 1e-13, f"chunked {mode} LSE")


def _scatter_to_pages(seqs, ps, layout, g, spare=2):
    """Place each request's contiguous K/V ([L, Hkv, d] pairs) into randomly
    chosen physical pages by hand; returns (k_pages, v_pages, block_table)."""
    hkv, d = seqs[0][0].shape[1:]
    npages = [(K.shape[0] + ps - 1) // ps for K, _ in seqs]
    P = sum(npages) + spare
    perm = g.permutation(P)
    shape = (P, ps, hkv, d) if layout == "NHD" else (P, hkv, ps, d)
    kp = g.standard_normal(shape) * 50.0      # slots nobody owns hold large junk
    vp = g.standard_normal(shape) * 50.0
    bt = np.full((len(seqs), max(1, max(npages))), -1)
    off = 0
    for b, (K, V) in enumerate(seqs):
        for t in range(K.shape[0]):
            phys = perm[off + t // ps]
            bt[b, t // ps] = phys
            if layout == "NHD":
                kp[phys, t % ps] = K[t]
                vp[phys, t % ps] = V[t]
            else:
                kp[phys, :, t % ps] = K[t]
                vp[phys, :, t % ps] = V[t]
        off += npages[b]
    return kp, vp, bt


def pin_chunk_matches_full(paged_prefill_ref, attention_ref, layout="NHD", seed=111):
    """A chunk of the last q_len queries of a sequence must reproduce the same
    rows of a causal prefill over the whole sequence (the prefix is cached)."""
    g = np.random.default_rng(seed)
    hq, hkv, d, ps = 4, 2, 6, 4
    cases = [(0, 7), (5, 1), (9, 4), (3, 13), (8, 8)]      # (cached prefix, chunk)
    seqs, qs, full = [], [], []
    for prefix, n in cases:
        L = prefix + n
        q = g.standard_normal((L, hq, d))
        K = g.standard_normal((L, hkv, d))
        V = g.standard_normal((L, hkv, d))
        seqs.append((K, V))
        qs.append(q[prefix:])
        full.append(attention_ref(q, K, V, [0, L], True, 0.45))
    kp, vp, bt = _scatter_to_pages(seqs, ps, layout, g)
    cu = np.concatenate([[0], np.cumsum([n for _, n in cases])])
    lens = [p + n for p, n in cases]
    o, l = paged_prefill_ref(np.concatenate(qs), cu, kp, vp, bt, lens, True, 0.45,
                             page_size=ps, layout=layout)
    for b, (prefix, n) in enumerate(cases):
        of, lf = full[b]
        _close(o[cu[b]:cu[b + 1]], of[prefix:], 1e-12, f"chunk vs full O case {b}")
        _close(l[cu[b]:cu[b + 1]], lf[prefix:], 1e-12, f"chunk vs full LSE case {b}")


def pin_sdpa_lower_right(paged_prefill_ref, seed=121):
    """PyTorch CPU scaled_dot_product_attention in float64 with its own
    lower-right causal bias (torch.nn.attention.bias.causal_lower_right) and
    enable_gqa, on the gathered contiguous K/V of each request."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention.bias import causal_lower_right

    g = np.random.default_rng(seed)
    hq, hkv, d, ps = 6, 2, 5, 4
    cases = [(3, 2), (0, 5), (11, 6), (2, 1)]
    seqs = [(g.standard_normal((p + n, hkv, d)), g.standard_normal((p + n, hkv, d))) for p, n in cases]
    kp, vp, bt = _scatter_to_pages(seqs, ps, "NHD", g)
    cu = np.concatenate([[0], np.cumsum([n for _, n in cases])])
    q = g.standard_normal((int(cu[-1]), hq, d))
    lens = [p + n for p, n in cases]
    for causal in (False, True):
        o, l = paged_prefill_ref(q, cu, kp, vp, bt, lens, causal, 0.35, page_size=ps)
        for b, (p, n) in enumerate(cases):
            K, V = seqs[b]
            tq = torch.from_numpy(q[cu[b]:cu[b + 1]]).permute(1, 0, 2)[None]
            tk = torch.from_numpy(K).permute(1, 0, 2)[None]
            tv = torch.from_numpy(V).permute(1, 0, 2)[None]
            mask = causal_lower_right(n, p + n) if causal else None
            ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.35,
                                                 enable_gqa=True)
            _close(o[cu[b]:cu[b + 1]], ref[0].permute(1, 0, 2).numpy(), 1e-12,
                   f"sdpa lower-right case {b} causal={causal}")


def pin_chunk_single_query_is_decode(paged_prefill_ref, paged_decode_ref, seed=131):
    """A one-token chunk under causal masking sees the whole cache: decode."""
    g = np.random.default_rng(seed)
    hq, hkv, d, ps = 4, 1, 3, 4
    lens = [1, 6, 9]
    seqs = [(g.standard_normal((L, hkv, d)), g.standard_normal((L, hkv, d))) for L in lens]
    kp, vp, bt = _scatter_to_pages(seqs, ps, "HND", g)
    q = g.standard_normal((len(lens), hq, d))
    o, l = paged_prefill_ref(q, np.arange(len(lens) + 1), kp, vp, bt, lens, True, 0.8,
                             page_size=ps, layout="HND")
    od, ld = paged_decode_ref(q, kp, vp, bt, lens, 0.8, page_size=ps, layout="HND")
    _close(o, od, 1e-13, "single-query chunk vs decode O")
    _close(l, ld, 1e-13, "single-query chunk vs decode LSE")


# --- FP8 (E4M3) KV cache ------------------------------------------------------

def pin_e4m3_codes(e4m3_to_f64):
    """Hand-decoded codes, then all 256 codes against PyTorch's float8_e4m3fn."""
    import torch
    g = load_golden("fp8_decode.json")
    for code, val in g["codes"].items():
        got = float(e4m3_to_f64(np.array([int(code, 16)], dtype=np.uint8))[0])
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), \
            f"E4M3 {code}: {got} != {val}"
    allb = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(allb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_to_f64(allb)
    assert np.array_equal(np.isnan(got), np.isnan(ref)), "E4M3 NaN codes"
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok]), "E4M3 values vs torch float8_e4m3fn"


def pin_golden_fp8_decode(paged_decode_ref, dequantize_e4m3):
    g = load_golden("fp8_decode.json")
    kp = np.array(g["k_pages"], dtype=np.uint8)
    vp = np.array(g["v_pages"], dtype=np.uint8)
    o, l = paged_decode_ref(np.array(g["q"]), kp, vp, np.array(g["block_table"]),
                            np.array(g["cache_seqlens"]), g["scale"], page_size=g["page_size"],
                            k_to_f64=lambda a: dequantize_e4m3(a, g["k_scale"]),
                            v_to_f64=lambda a: dequantize_e4m3(a, g["v_scale"]))
    _close(o, g["o"], 1e-13, "fp8 decode O")
    _close(l, g["lse"], 1e-13, "fp8 decode LSE")


# --- cascade (shared-prefix) decode -------------------------------------------

def pin_cascade_matches_concatenation(cascade_decode_ref, partial_state_ref, layout="NHD", seed=161):
    """Hand-built contiguous context = prefix rows then suffix rows; the cascade
    must equal plain attention of each query over it (prefix not a page multiple)."""
    g = np.random.default_rng(seed)
    hq, hkv, d, ps = 4, 2, 5, 4
    P, suf = 7, [0, 3, 9]
    pre_k, pre_v = g.standard_normal((P, hkv, d)), g.standard_normal((P, hkv, d))
    seqs = [(pre_k, pre_v)] + [(g.standard_normal((L, hkv, d)), g.standard_normal((L, hkv, d)))
                               for L in suf]
    kp, vp, bt = _scatter_to_pages(seqs, ps, layout, g)
    q = g.standard_normal((len(suf), hq, d))
    o, l = cascade_decode_ref(q, kp, vp, bt[0][:(P + ps - 1) // ps], P, bt[1:], suf, 0.7,
                              page_size=ps, layout=layout)
    for b, L in enumerate(suf):
        K = np.concatenate([pre_k, seqs[b + 1][0]])
        V = np.concatenate([pre_v, seqs[b + 1][1]])
        for h in range(hq):
            gh = h // (hq // hkv)
            ob, lb = partial_state_ref(q[b, h][None], K[:, gh], V[:, gh], 0.7)
            _close(o[b, h], ob[0], 1e-13, f"cascade O b={b} h={h}")
            _close(l[b, h], lb[0], 1e-13, f"cascade LSE b={b} h={h}")


def pin_cascade_aligned_is_decode(cascade_decode_ref, paged_decode_ref, seed=171):
    """With a page-aligned prefix the cascade equals the plain paged decode whose
    table rows list the prefix pages and then the suffix pages."""
    g = np.random.default_rng(seed)
    hq, hkv, d, ps = 6, 3, 4, 4
    P, suf = 8, [1, 0, 6]
    seqs = [(g.standard_normal((P, hkv, d)), g.standard_normal((P, hkv, d)))] + \
        [(g.standard_normal((L, hkv, d)), g.standard_normal((L, hkv, d))) for L in suf]
    kp, vp, bt = _scatter_to_pages(seqs, ps, "HND", g)
    q = g.standard_normal((len(suf), hq, d))
    pre = bt[0][:P // ps]
    o, l = cascade_decode_ref(q, kp, vp, pre, P, bt[1:], suf, 0.5, page_size=ps, layout="HND")
    full = np.full((len(suf), len(pre) + bt.shape[1]), -1)
    full[:, :len(pre)] = pre
    full[:, len(pre):] = bt[1:]
    od, ld = paged_decode_ref(q, kp, vp, full, [P + L for L in suf], 0.5, page_size=ps, layout="HND")
    _close(o, od, 1e-13, "cascade vs decode O")
    _close(l, ld, 1e-13, "cascade vs decode LSE")
