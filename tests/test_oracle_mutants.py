"""Plant one plausible mistake at a time in the oracle (on the CPU) and check
that the pins catch it.  This shows the pins are sensitive to dropped terms,
wrong signs/indices and transposed operands."""
import math

import numpy as np
import pytest

import oracle
from oracle import attention as A
from tests import oracle_pins as P

ALL_PREFILL_PINS = [
    lambda: P.pin_golden_two_keys(A.attention_ref),
    lambda: P.pin_golden_causal_uniform(A.attention_ref),
    lambda: P.pin_identical_keys(A.attention_ref, True),
    lambda: P.pin_identical_keys(A.attention_ref, False),
    lambda: P.pin_causal_row0(A.attention_ref),
    lambda: P.pin_bruteforce(A.attention_ref),
    lambda: P.pin_sdpa(A.attention_ref),
    lambda: P.pin_rows_sum_to_one(A.attention_probs_ref, True),
]


def _some_pin_fires(pins):
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


MUTANTS = {
    # causal mask in the wrong direction (future keys allowed, past masked)
    "mask_flipped": ("_causal_mask_block",
                     lambda row0, n, nk: (np.arange(nk)[None, :] < np.arange(row0, row0 + n)[:, None])),
    # off-by-one: diagonal key masked
    "mask_excludes_diag": ("_causal_mask_block",
                           lambda row0, n, nk: (np.arange(nk)[None, :] >= np.arange(row0, row0 + n)[:, None])),
    # scale dropped
    "no_scale": ("_scores", lambda q, k, scale: q @ k.T),
    # operands transposed (K Q^T instead of Q K^T) on square blocks
    "transposed": ("_scores", lambda q, k, scale: scale * (k @ q.T) if q.shape == k.shape else scale * (q @ k.T)),
    # GQA head mapping interleaved instead of grouped
    "gqa_modulo": ("kv_head_of", lambda h, hq, hkv: h % hkv),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_prefill_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(A, attr, fn)
    assert _some_pin_fires(ALL_PREFILL_PINS), f"no pin caught mutant {name}"


def test_lse_base2_is_caught(monkeypatch):
    orig = A._softmax_with_lse

    def bad(s):
        p, lse = orig(s)
        return p, lse / math.log(2.0)
    monkeypatch.setattr(A, "_softmax_with_lse", bad)
    assert _some_pin_fires(ALL_PREFILL_PINS)


def test_lse_missing_max_is_caught(monkeypatch):
    orig = A._softmax_with_lse

    def bad(s):
        p, lse = orig(s)
        m = np.max(s, axis=-1)
        return p, lse - np.where(np.isfinite(m), m, 0.0)
    monkeypatch.setattr(A, "_softmax_with_lse", bad)
    assert _some_pin_fires(ALL_PREFILL_PINS)


def _merge_uniform(o_parts, lse_parts):
    o_parts = np.asarray(o_parts)
    return o_parts.mean(axis=0), np.max(lse_parts, axis=0)


def _merge_no_shift(o_parts, lse_parts):
    w = np.exp(np.asarray(lse_parts))
    return (w[..., None] * o_parts).sum(0) / w.sum(0)[..., None], np.log(w.sum(0))


def _merge_wrong_lse(o_parts, lse_parts):
    o, l = oracle.merge_states_ref(o_parts, lse_parts)
    return o, np.max(lse_parts, axis=0)


@pytest.mark.parametrize("bad", [_merge_uniform, _merge_no_shift, _merge_wrong_lse])
def test_merge_mutant_is_caught(bad):
    pins = [lambda: P.pin_golden_merge(bad),
            lambda: P.pin_partition_merge(oracle.partial_state_ref, bad, oracle.attention_rows_ref)]
    with np.errstate(all="ignore"):
        assert _some_pin_fires(pins)


def test_paged_walk_mutant_is_caught(monkeypatch):
    """Reading slot t % page_size from page t // page_size of the *physical*
    pool (ignoring the page table) must be caught."""
    def bad_gather(k_pages, v_pages, row, seqlen, g, ps, layout="NHD"):
        n = (seqlen + ps - 1) // ps
        if layout == "NHD":
            K = np.concatenate([k_pages[p, :, g] for p in range(n)])[:seqlen]
            V = np.concatenate([v_pages[p, :, g] for p in range(n)])[:seqlen]
        else:
            K = np.concatenate([k_pages[p, g] for p in range(n)])[:seqlen]
            V = np.concatenate([v_pages[p, g] for p in range(n)])[:seqlen]
        return K, V
    monkeypatch.setattr(A, "gather_paged_kv", bad_gather)
    pins = [lambda: P.pin_golden_paged(A.paged_decode_ref),
            lambda: P.pin_decode_walk(A.paged_decode_ref, A.partial_state_ref)]
    assert _some_pin_fires(pins)


CHUNKED_PINS = [
    lambda: P.pin_golden_chunked(A.paged_prefill_ref),
    lambda: P.pin_chunk_matches_full(A.paged_prefill_ref, A.attention_ref),
    lambda: P.pin_sdpa_lower_right(A.paged_prefill_ref),
    lambda: P.pin_chunk_single_query_is_decode(A.paged_prefill_ref, A.paged_decode_ref),
]

CHUNK_MASK_MUTANTS = {
    # top-left alignment: query i of the chunk sees keys 0..i
    "top_left": lambda q_len, k_len: np.arange(k_len)[None, :] > np.arange(q_len)[:, None],
    # off by one: the query's own position masked
    "excludes_own": lambda q_len, k_len: (np.arange(k_len)[None, :]
                                          >= (k_len - q_len + np.arange(q_len))[:, None]),
    # offset in the wrong direction
    "offset_sign": lambda q_len, k_len: (np.arange(k_len)[None, :]
                                         > (q_len - k_len + np.arange(q_len))[:, None]),
}


@pytest.mark.parametrize("name", sorted(CHUNK_MASK_MUTANTS))
def test_chunk_mask_mutant_is_caught(name, monkeypatch):
    monkeypatch.setattr(A, "_chunk_causal_mask", CHUNK_MASK_MUTANTS[name])
    with np.errstate(all="ignore"):
        assert _some_pin_fires(CHUNKED_PINS), f"no pin caught mutant {name}"


def test_chunked_paged_walk_mutant_is_caught(monkeypatch):
    """The chunked prefill reading physical pages in order, ignoring the table."""
    def bad_gather(k_pages, v_pages, row, seqlen, g, ps, layout="NHD"):
        n = (seqlen + ps - 1) // ps
        if n == 0:
            return np.zeros((0, k_pages.shape[-1])), np.zeros((0, k_pages.shape[-1]))
        if layout == "NHD":
            return (np.concatenate([k_pages[p, :, g] for p in range(n)])[:seqlen],
                    np.concatenate([v_pages[p, :, g] for p in range(n)])[:seqlen])
        return (np.concatenate([k_pages[p, g] for p in range(n)])[:seqlen],
                np.concatenate([v_pages[p, g] for p in range(n)])[:seqlen])
    monkeypatch.setattr(A, "gather_paged_kv", bad_gather)
    assert _some_pin_fires(CHUNKED_PINS)


def _append_from_old_length(kp, vp, kn, vn, cu, bt, lens, page_size=64, layout="NHD"):
    """Mistake: treats cache_seqlens as the length before the append."""
    n = np.diff(np.asarray(cu))
    return A.append_kv_ref(kp, vp, kn, vn, cu, bt, np.asarray(lens) + n, page_size, layout)


def _append_slot_from_page_index(kp, vp, kn, vn, cu, bt, lens, page_size=64, layout="NHD"):
    """Mistake: page and slot swapped (pos % page_size picks the page)."""
    kp = np.array(kp, copy=True)
    vp = np.array(vp, copy=True)
    for b in range(len(cu) - 1):
        n = cu[b + 1] - cu[b]
        for i in range(n):
            pos = int(lens[b]) - n + i
            phys = int(bt[b][pos % page_size])
            kp[phys, pos // page_size] = kn[cu[b] + i]
            vp[phys, pos // page_size] = vn[cu[b] + i]
    return kp, vp


@pytest.mark.parametrize("bad", [_append_from_old_length, _append_slot_from_page_index])
def test_append_mutant_is_caught(bad):
    with np.errstate(all="ignore"):
        try:
            P.pin_golden_append(bad)
        except (AssertionError, IndexError):
            return
    raise AssertionError("append mutant not caught")


E4M3_MUTANTS = {
    # exponent bias 8 instead of 7
    "bias8": lambda b: np.where(((np.asarray(b, np.int64) >> 3) & 15) == 0,
                                np.ldexp((np.asarray(b, np.int64) & 7) / 8.0, -6),
                                np.ldexp(1.0 + (np.asarray(b, np.int64) & 7) / 8.0,
                                         ((np.asarray(b, np.int64) >> 3) & 15) - 8))
    * np.where(np.asarray(b, np.int64) >> 7, -1.0, 1.0),
    # subnormals decoded with an implicit leading one
    "no_subnormal": lambda b: np.ldexp(1.0 + (np.asarray(b, np.int64) & 7) / 8.0,
                                       ((np.asarray(b, np.int64) >> 3) & 15) - 7)
    * np.where(np.asarray(b, np.int64) >> 7, -1.0, 1.0),
}


@pytest.mark.parametrize("name", sorted(E4M3_MUTANTS))
def test_e4m3_mutant_is_caught(name):
    with np.errstate(all="ignore"):
        try:
            P.pin_e4m3_codes(E4M3_MUTANTS[name])
        except AssertionError:
            return
    raise AssertionError(f"E4M3 mutant {name} not caught")


def test_fp8_scales_swapped_is_caught():
    from oracle import fp8
    swapped = lambda bits, scale: fp8.dequantize_e4m3(bits, 0.5 if scale != 0.5 else math.log(3.0))
    try:
        P.pin_golden_fp8_decode(A.paged_decode_ref, swapped)
    except AssertionError:
        return
    raise AssertionError("swapped K/V scales not caught")


def test_cascade_mutants_are_caught(monkeypatch):
    """A cascade that drops the prefix, or counts it twice, must be caught."""
    real = A.cascade_decode_ref

    def no_prefix(q, kp, vp, pre, P, bt, suf, scale=None, page_size=64, layout="NHD", **kw):
        return real(q, kp, vp, pre[:0], 0, bt, suf, scale, page_size, layout, **kw)

    def double_prefix(q, kp, vp, pre, P, bt, suf, scale=None, page_size=64, layout="NHD", **kw):
        n = len(pre)
        bt2 = np.full((bt.shape[0], n + bt.shape[1]), -1)
        bt2[:, :n] = pre
        bt2[:, n:] = bt
        if P % page_size:     # only page-aligned prefixes can be doubled through the table
            return real(q, kp, vp, pre, P, bt, suf, scale * 1.01, page_size, layout, **kw)
        return real(q, kp, vp, pre, P, bt2, np.asarray(suf) + P, scale, page_size, layout, **kw)

    for bad in (no_prefix, double_prefix):
        pins = [lambda: P.pin_cascade_matches_concatenation(bad, A.partial_state_ref),
                lambda: P.pin_cascade_aligned_is_decode(bad, A.paged_decode_ref)]
        with np.errstate(all="ignore"):
            assert _some_pin_fires(pins), bad.__name__
