"""Exact attention, float64, on the CPU — the oracle (test infrastructure only).

Definition followed (wsisp.com "FIA / FlashAttention", section 一, the formula
Attention(Q,K,V) = softmax(Q K^T / sqrt(d)) V; the 5688vip course page, section
1.2, spells the same steps as scores = Q K^T / sqrt(head_dim), softmax, times V):

    s_ij  = scale * sum_c q[i, h, c] * k[j, g, c]          over allowed keys j
    LSE_i = ln sum_j exp(s_ij)                              (natural log)
    O_i   = sum_j exp(s_ij - LSE_i) * v[j, g, :]

with ``scale = 1/sqrt(d)`` unless given, and kv head ``g = h // (Hq/Hkv)``.
The full score block is materialised (the "standard attention" the pages
contrast with tiling: "Flash Attention & Paged Attention", section 1 pseudocode)
and the softmax is summed explicitly.  No tiling, no online softmax, no
reordering: this is the thing the tiled kernels must reproduce.

Readings taken where the pages are silent:

* causal: key j is allowed for query i iff j <= i, both counted from the start
  of their sequence (one ``cu_seqlens`` for q and k, so q and k lengths match);
* GQA: consecutive groups of Hq/Hkv query heads share one kv head;
* LSE: natural log of the sum of exp of the *scaled* scores;
* an empty key set gives O = 0 and LSE = -inf (only reachable in decode with a
  zero cache length or an empty split);
* paged decode attends to all ``cache_seqlens[b]`` cached tokens, no mask;
* chunked (paged) prefill: a request's cache holds ``cache_seqlens[b]`` tokens
  after the new chunk is written, and the chunk's q_len queries are the last
  q_len positions of that sequence, so under causal masking query i of the
  chunk (position cache_seqlens[b] - q_len + i) sees keys at positions up to
  its own (the KV cache of "Flash Attention & Paged Attention", section
  "FA对Prefill阶段的影响": prefill stores K/V that later steps reuse; the
  mask keeps the same rule as a full prefill of the whole sequence);
* KV append: the chunk's n new K/V rows take logical positions
  cache_seqlens[b] - n ... cache_seqlens[b] - 1 of their request and are
  written through the page table (same page, section 2);
* multi-token decode (several query tokens per request) is the chunked
  prefill rule applied to a decode step: the tokens are the last q_len
  positions of the cache;
* cascade (prefix sharing, wsisp.com "FIA / FlashAttention", section 三): a
  request's keys are the shared prefix followed by its own suffix, and the
  result is plain attention over that concatenation.

Split/merge (Flash-Decoding, "Flash Attention & Paged Attention", section
"FA对decode阶段的影响", steps 3-4): each split yields a partial (O_i, LSE_i)
over its keys; the merged result is O = sum_i w_i O_i / sum_i w_i with
w_i = exp(LSE_i - max LSE), and LSE = max LSE + ln sum_i w_i.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def kv_head_of(h: int, num_q_heads: int, num_kv_heads: int) -> int:
    """kv head read by query head h: consecutive groups of Hq/Hkv share one."""
    group = num_q_heads // num_kv_heads
    return h // group


def allowed_key_count(i: int, seqlen: int, causal: bool) -> int:
    """Number of leading keys query i (in-sequence index) may attend to."""
    return i + 1 if causal else seqlen


def visible_key_count(i: int, q_len: int, k_len: int, causal: bool) -> int:
    """Keys visible to query i of a chunk whose q_len queries are the last
    q_len of a k_len-token sequence (i counted from the chunk's start)."""
    return k_len - q_len + i + 1 if causal else k_len


def _scores(q_rows: np.ndarray, keys: np.ndarray, scale: float) -> np.ndarray:
    """scale * Q K^T for a block of query rows against a block of keys."""
    return scale * (q_rows @ keys.T)


def _softmax_with_lse(s: np.ndarray):
    """Row softmax of a (possibly -inf masked) score block, plus its LSE.

    Rows with no allowed key (all -inf, or no columns at all) get zero
    weights and LSE = -inf."""
    if s.shape[-1] == 0:
        return np.zeros(s.shape), np.full(s.shape[:-1], NEG_INF)
    m = np.max(s, axis=-1, keepdims=True)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe)
    denom = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(denom > 0, e / np.where(denom > 0, denom, 1.0), 0.0)
        lse = np.where(denom[:, 0] > 0, m_safe[:, 0] + np.log(np.where(denom[:, 0] > 0, denom[:, 0], 1.0)),
                       NEG_INF)
    return p, lse


def _causal_mask_block(row0: int, nrows: int, nkeys: int) -> np.ndarray:
    """True where key j is NOT allowed for query row0 + r (j > row0 + r)."""
    i = np.arange(row0, row0 + nrows)[:, None]
    j = np.arange(nkeys)[None, :]
    return j > i


def attention_ref(q, k, v, cu_seqlens, causal: bool, scale: float | None = None,
                  row_block: int = 1024):
    """Exact attention over packed variable-length sequences.

    q: [T, Hq, d]; k, v: [T, Hkv, d] (float64 values); cu_seqlens: [B+1].
    Returns (O [T, Hq, d] float64, LSE [T, Hq] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((T, Hq, v.shape[2]))
    lse = np.full((T, Hq), NEG_INF)
    cu = [int(x) for x in cu_seqlens]
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        L = s1 - s0
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            Q = q[s0:s1, h]
            K = k[s0:s1, g]
            V = v[s0:s1, g]
            for r0 in range(0, L, row_block):
                r1 = min(L, r0 + row_block)
                nk = allowed_key_count(r1 - 1, L, causal)
                S = _scores(Q[r0:r1], K[:nk], scale)
                if causal:
                    S = np.where(_causal_mask_block(r0, r1 - r0, nk), NEG_INF, S)
                P, l = _softmax_with_lse(S)
                out[s0 + r0:s0 + r1, h] = P @ V[:nk]
                lse[s0 + r0:s0 + r1, h] = l
    return out, lse


def attention_rows_ref(q, k, v, cu_seqlens, causal: bool, scale: float | None, rows):
    """Selected rows of ``attention_ref``: rows = iterable of (token, q_head).

    Returns (O [n, d], LSE [n]); each row is computed on its own, so this is
    usable at full problem sizes.
    """
    q = np.asarray(q)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = list(rows)
    out = np.zeros((len(rows), v.shape[2]))
    lse = np.zeros(len(rows))
    for n, (t, h) in enumerate(rows):
        b = int(np.searchsorted(cu, t, side="right") - 1)
        s0, s1 = int(cu[b]), int(cu[b + 1])
        i = t - s0
        nk = allowed_key_count(i, s1 - s0, causal)
        g = kv_head_of(h, Hq, Hkv)
        K = np.asarray(k[s0:s0 + nk, g], dtype=np.float64)
        V = np.asarray(v[s0:s0 + nk, g], dtype=np.float64)
        qi = np.asarray(q[t, h], dtype=np.float64)[None, :]
        P, l = _softmax_with_lse(_scores(qi, K, scale))
        out[n] = (P @ V)[0]
        lse[n] = l[0]
    return out, lse


def attention_probs_ref(q, k, cu_seqlens, causal: bool, scale: float | None = None):
    """Softmax weights of every (sequence, head) as a list of [L, L] arrays.

    Used by the oracle's own pins (rows sum to one, masked weights are zero).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    res = []
    cu = [int(x) for x in cu_seqlens]
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        L = s1 - s0
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            S = _scores(q[s0:s1, h], k[s0:s1, g], scale)
            if causal:
                S = np.where(_causal_mask_block(0, L, L), NEG_INF, S)
            P, _ = _softmax_with_lse(S)
            res.append(P)
    return res


def gather_paged_kv(k_pages, v_pages, block_table_row, seqlen: int, kv_head: int,
                    page_size: int, layout: str = "NHD"):
    """Logical K/V rows [seqlen, d] of one request and kv head, by walking its page table.

    Logical token t lives in physical page block_table_row[t // page_size] at
    slot t % page_size ("Flash Attention & Paged Attention", section 2: fixed
    pages, non-contiguous physical memory, logical-to-physical page table).
    """
    n_pages = (seqlen + page_size - 1) // page_size
    ks, vs = [], []
    for p in range(n_pages):
        phys = int(block_table_row[p])
        if layout == "NHD":
            ks.append(k_pages[phys, :, kv_head, :])
            vs.append(v_pages[phys, :, kv_head, :])
        else:
            ks.append(k_pages[phys, kv_head, :, :])
            vs.append(v_pages[phys, kv_head, :, :])
    if n_pages == 0:
        d = k_pages.shape[-1]
        return np.zeros((0, d)), np.zeros((0, d))
    K = np.concatenate(ks, axis=0)[:seqlen]
    V = np.concatenate(vs, axis=0)[:seqlen]
    return K, V


def paged_decode_rows_ref(q, k_pages, v_pages, block_table, cache_seqlens, scale,
                          rows, page_size: int = 64, layout: str = "NHD",
                          to_f64=lambda a: np.asarray(a, dtype=np.float64),
                          k_to_f64=None, v_to_f64=None):
    """Decode output for selected (request, q_head) rows.

    ``to_f64`` widens the query and gathered cache slices (e.g. bf16 bit
    patterns); ``k_to_f64`` / ``v_to_f64``, when given, replace it for the K
    and V slices (e.g. dequantising an FP8 cache).  By default everything is
    taken to already hold float values.
    Returns (O [n, d], LSE [n]).
    """
    k_conv = k_to_f64 if k_to_f64 is not None else to_f64
    v_conv = v_to_f64 if v_to_f64 is not None else to_f64
    B, Hq, d = q.shape
    Hkv = k_pages.shape[2] if layout == "NHD" else k_pages.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((len(rows), d))
    lse = np.zeros(len(rows))
    cache = {}
    for n, (b, h) in enumerate(rows):
        g = kv_head_of(h, Hq, Hkv)
        key = (b, g)
        if key not in cache:
            K, V = gather_paged_kv(k_pages, v_pages, block_table[b], int(cache_seqlens[b]), g,
                                   page_size, layout)
            cache = {key: (k_conv(K), v_conv(V))}
        K, V = cache[key]
        qi = to_f64(q[b, h])[None, :]
        P, l = _softmax_with_lse(_scores(qi, K, scale))
        out[n] = (P @ V)[0] if K.shape[0] else 0.0
        lse[n] = l[0]
    return out, lse


def paged_decode_ref(q, k_pages, v_pages, block_table, cache_seqlens, scale=None,
                     page_size: int = 64, layout: str = "NHD",
                     to_f64=lambda a: np.asarray(a, dtype=np.float64),
                     k_to_f64=None, v_to_f64=None):
    """One query row per request against its whole paged KV cache.

    q: [B, Hq, d]. Returns (O [B, Hq, d], LSE [B, Hq]).
    """
    B, Hq, d = q.shape
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o, l = paged_decode_rows_ref(q, k_pages, v_pages, block_table, cache_seqlens, scale, rows,
                                 page_size, layout, to_f64, k_to_f64, v_to_f64)
    return o.reshape(B, Hq, d), l.reshape(B, Hq)


def partial_state_ref(q_rows, keys, values, scale: float):
    """(O_i, LSE_i) of query rows over one subset of keys (one Flash-Decoding split).

    q_rows: [n, d]; keys, values: [m, d].  An empty subset gives O=0, LSE=-inf.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    n, d = q_rows.shape
    if keys.shape[0] == 0:
        return np.zeros((n, values.shape[1] if values.ndim == 2 else d)), np.full(n, NEG_INF)
    P, l = _softmax_with_lse(_scores(q_rows, keys, scale))
    return P @ values, l


def merge_states_ref(o_parts, lse_parts):
    """Merge partial states along axis 0 by their LSE.

    o_parts: [S, ..., d]; lse_parts: [S, ...].  States with LSE = -inf carry
    zero weight; if every state is empty the result is O = 0, LSE = -inf.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    M = np.max(lse_parts, axis=0)
    finite = np.isfinite(M)
    M_safe = np.where(finite, M, 0.0)
    w = np.exp(lse_parts - M_safe[None])          # [S, ...]
    wsum = np.sum(w, axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.sum(w[..., None] * o_parts, axis=0) / np.where(wsum > 0, wsum, 1.0)[..., None]
        lse = np.where(wsum > 0, M_safe + np.log(np.where(wsum > 0, wsum, 1.0)), NEG_INF)
    o = np.where((wsum > 0)[..., None], o, 0.0)
    return o, lse


def append_kv_ref(k_pages, v_pages, k_new, v_new, cu_seqlens_new, block_table, cache_seqlens,
                  page_size: int = 64, layout: str = "NHD"):
    """Write each request's new K/V rows into its pages (KV-cache append).

    k_new, v_new: [T_new, Hkv, d] packed by ``cu_seqlens_new``; request b's
    n_b rows go to logical positions cache_seqlens[b] - n_b + i, each at page
    block_table[b][pos // page_size], slot pos % page_size.  Returns new
    (k_pages, v_pages) arrays; every other slot keeps its contents.
    """
    kp = np.array(k_pages, copy=True)
    vp = np.array(v_pages, copy=True)
    cu = [int(x) for x in cu_seqlens_new]
    for b in range(len(cu) - 1):
        n = cu[b + 1] - cu[b]
        first = int(cache_seqlens[b]) - n
        if first < 0:
            raise ValueError("cache length shorter than the appended chunk")
        for i in range(n):
            pos = first + i
            phys = int(block_table[b][pos // page_size])
            slot = pos % page_size
            if layout == "NHD":
                kp[phys, slot] = k_new[cu[b] + i]
                vp[phys, slot] = v_new[cu[b] + i]
            else:
                kp[phys, :, slot] = k_new[cu[b] + i]
                vp[phys, :, slot] = v_new[cu[b] + i]
    return kp, vp


def _chunk_causal_mask(q_len: int, k_len: int) -> np.ndarray:
    """True where key j is NOT visible to query i of the chunk."""
    i = np.arange(q_len)[:, None]
    j = np.arange(k_len)[None, :]
    return j > (k_len - q_len + i)


def paged_prefill_ref(q, cu_seqlens_q, k_pages, v_pages, block_table, cache_seqlens,
                      causal: bool, scale=None, page_size: int = 64, layout: str = "NHD",
                      to_f64=lambda a: np.asarray(a, dtype=np.float64),
                      k_to_f64=None, v_to_f64=None):
    """Chunked prefill: each request's new queries against its whole paged cache.

    q: [Tq, Hq, d] packed by ``cu_seqlens_q``; request b's cache holds
    cache_seqlens[b] >= q_len_b tokens (the chunk's own K/V included).
    ``k_to_f64`` / ``v_to_f64`` replace ``to_f64`` for the gathered K and V
    (as in ``paged_decode_rows_ref``).
    Returns (O [Tq, Hq, d], LSE [Tq, Hq]).
    """
    k_conv = k_to_f64 if k_to_f64 is not None else to_f64
    v_conv = v_to_f64 if v_to_f64 is not None else to_f64
    q = np.asarray(q)
    Tq, Hq, d = q.shape
    Hkv = k_pages.shape[2] if layout == "NHD" else k_pages.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((Tq, Hq, d))
    lse = np.full((Tq, Hq), NEG_INF)
    cu = [int(x) for x in cu_seqlens_q]
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        Lq, Lk = s1 - s0, int(cache_seqlens[b])
        if Lk < Lq:
            raise ValueError("cache length shorter than the chunk")
        for g in range(Hkv):
            K, V = gather_paged_kv(k_pages, v_pages, block_table[b], Lk, g, page_size, layout)
            K, V = k_conv(K), v_conv(V)
            for h in range(Hq):
                if kv_head_of(h, Hq, Hkv) != g:
                    continue
                S = _scores(to_f64(q[s0:s1, h]), K, scale)
                if causal:
                    S = np.where(_chunk_causal_mask(Lq, Lk), NEG_INF, S)
                P, l = _softmax_with_lse(S)
                out[s0:s1, h] = P @ V
                lse[s0:s1, h] = l
    return out, lse


def paged_prefill_rows_ref(q, cu_seqlens_q, k_pages, v_pages, block_table, cache_seqlens,
                           causal: bool, scale, rows, page_size: int = 64, layout: str = "NHD",
                           to_f64=lambda a: np.asarray(a, dtype=np.float64),
                           k_to_f64=None, v_to_f64=None):
    """Selected rows (token, q_head) of ``paged_prefill_ref``, each on its own.

    Returns (O [n, d], LSE [n]).
    """
    k_conv = k_to_f64 if k_to_f64 is not None else to_f64
    v_conv = v_to_f64 if v_to_f64 is not None else to_f64
    q = np.asarray(q)
    Tq, Hq, d = q.shape
    Hkv = k_pages.shape[2] if layout == "NHD" else k_pages.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cu = np.asarray(cu_seqlens_q, dtype=np.int64)
    rows = list(rows)
    out = np.zeros((len(rows), d))
    lse = np.zeros(len(rows))
    cache = {}
    for n, (t, h) in enumerate(rows):
        b = int(np.searchsorted(cu, t, side="right") - 1)
        Lq, Lk = int(cu[b + 1] - cu[b]), int(cache_seqlens[b])
        i = t - int(cu[b])
        g = kv_head_of(h, Hq, Hkv)
        if (b, g) not in cache:
            K, V = gather_paged_kv(k_pages, v_pages, block_table[b], Lk, g, page_size, layout)
            cache = {(b, g): (k_conv(K), v_conv(V))}
        K, V = cache[(b, g)]
        nk = visible_key_count(i, Lq, Lk, causal)
        P, l = _softmax_with_lse(_scores(to_f64(q[t, h])[None, :], K[:nk], scale))
        out[n] = (P @ V[:nk])[0]
        lse[n] = l[0]
    return out, lse


def cascade_decode_ref(q, k_pages, v_pages, prefix_block_table, prefix_len: int, block_table,
                       suffix_lens, scale=None, page_size: int = 64, layout: str = "NHD",
                       to_f64=lambda a: np.asarray(a, dtype=np.float64)):
    """Decode over a shared prefix followed by each request's own suffix.

    Request b's keys are the prefix_len tokens of the shared pages, then the
    suffix_lens[b] tokens of its own pages (prefix sharing, wsisp.com
    "FIA / FlashAttention", section 三): plain attention of its query row over
    that concatenation.  Returns (O [B, Hq, d], LSE [B, Hq]).
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    Hkv = k_pages.shape[2] if layout == "NHD" else k_pages.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for g in range(Hkv):
        Kp, Vp = gather_paged_kv(k_pages, v_pages, prefix_block_table, int(prefix_len), g,
                                 page_size, layout)
        for b in range(B):
            Ks, Vs = gather_paged_kv(k_pages, v_pages, block_table[b], int(suffix_lens[b]), g,
                                     page_size, layout)
            K = to_f64(np.concatenate([Kp, Ks], axis=0))
            V = to_f64(np.concatenate([Vp, Vs], axis=0))
            for h in range(Hq):
                if kv_head_of(h, Hq, Hkv) != g:
                    continue
                P, l = _softmax_with_lse(_scores(to_f64(q[b, h])[None, :], K, scale))
                out[b, h] = (P @ V)[0] if K.shape[0] else 0.0
                lse[b, h] = l[0]
    return out, lse
