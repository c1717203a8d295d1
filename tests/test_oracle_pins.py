"""The CPU oracle against facts it does not define itself (no GPU needed)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests import oracle_pins as P


def test_golden_two_keys():
    P.pin_golden_two_keys(oracle.attention_ref)


def test_golden_causal_uniform():
    P.pin_golden_causal_uniform(oracle.attention_ref)


def test_golden_merge():
    P.pin_golden_merge(oracle.merge_states_ref)


def test_golden_paged():
    P.pin_golden_paged(oracle.paged_decode_ref)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    P.pin_rows_sum_to_one(oracle.attention_probs_ref, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys(causal):
    P.pin_identical_keys(oracle.attention_ref, causal)


def test_dominant_key():
    P.pin_dominant_key(oracle.attention_ref)


def test_causal_row0():
    P.pin_causal_row0(oracle.attention_ref)


@pytest.mark.parametrize("seed", [51, 52, 53])
def test_partition_merge(seed):
    P.pin_partition_merge(oracle.partial_state_ref, oracle.merge_states_ref,
                          oracle.attention_rows_ref, seed)


@pytest.mark.parametrize("T,dk,dv", [(4, 4, 4), (4, 8, 3)])
def test_bruteforce_decimal(T, dk, dv):
    P.pin_bruteforce(oracle.attention_ref, T, dk, dv)


def test_sdpa_crosscheck():
    P.pin_sdpa(oracle.attention_ref)


def test_sdpa_crosscheck_mha():
    P.pin_sdpa(oracle.attention_ref, seqlens=(33, 1, 64), hq=2, hkv=2, d=16, seed=72)


def test_gqa_replication():
    P.pin_gqa_replication(oracle.attention_ref)


def test_varlen_packing():
    P.pin_varlen_packing(oracle.attention_ref)


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_decode_walk(layout):
    P.pin_decode_walk(oracle.paged_decode_ref, oracle.partial_state_ref, layout)


def test_attention_rows_match_full():
    q = np.random.default_rng(5).standard_normal((40, 4, 8))
    k = np.random.default_rng(6).standard_normal((40, 2, 8))
    v = np.random.default_rng(7).standard_normal((40, 2, 8))
    cu = [0, 25, 40]
    o, l = oracle.attention_ref(q, k, v, cu, True, 0.4, row_block=7)
    rows = [(0, 0), (24, 3), (25, 1), (39, 2), (13, 0)]
    orow, lrow = oracle.attention_rows_ref(q, k, v, cu, True, 0.4, rows)
    for n, (t, h) in enumerate(rows):
        assert np.max(np.abs(orow[n] - o[t, h])) < 1e-13
        assert abs(lrow[n] - l[t, h]) < 1e-13


def test_row_block_invariance():
    q = np.random.default_rng(8).standard_normal((50, 2, 4))
    k = np.random.default_rng(9).standard_normal((50, 2, 4))
    v = np.random.default_rng(10).standard_normal((50, 2, 4))
    o1, l1 = oracle.attention_ref(q, k, v, [0, 50], True, 0.5, row_block=1024)
    o2, l2 = oracle.attention_ref(q, k, v, [0, 50], True, 0.5, row_block=3)
    assert np.max(np.abs(o1 - o2)) < 1e-14 and np.max(np.abs(l1 - l2)) < 1e-14


def test_page_permutation_invariance_oracle():
    inp = W.make_decode([70, 5, 128], 4, 2, 16, seed=9, page_size=64, extra_pages=3)
    a = oracle.paged_decode_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits, inp.block_table,
                                inp.cache_seqlens, inp.scale, 64, inp.layout, to_f64=W.as_f64)
    p = W.permute_pages(inp, 17)
    b = oracle.paged_decode_ref(p.q_bits, p.k_pages_bits, p.v_pages_bits, p.block_table,
                                p.cache_seqlens, p.scale, 64, p.layout, to_f64=W.as_f64)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e38, 1e-40], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    back = W.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> rounds to even (1.0)
    assert back[0] == 1.0 and back[1] == 1.0
    # 1 + 1.5*2^-8 rounds up to 1 + 2^-7
    assert back[2] == np.float32(1.0078125)
    assert back[3] == -2.5
    import torch
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(t, bits)


def test_tiny_config_rounding_effect_reported():
    """fp32 inputs are rounded to bf16 before the oracle sees them; the oracle
    on the unrounded query differs by more than the LSE tolerance on some rows,
    which is why both sides consume the rounded values."""
    inp = W.tiny_causal_prefill()
    q = W.as_f64(inp.q_bits)
    k = W.as_f64(inp.k_bits)
    v = W.as_f64(inp.v_bits)
    o1, l1 = oracle.attention_ref(q, k, v, inp.cu_seqlens, True, inp.scale)
    o2, l2 = oracle.attention_ref(inp.q_f32_unrounded.astype(np.float64), k, v, inp.cu_seqlens,
                                  True, inp.scale)
    assert np.isfinite(o1).all() and np.isfinite(l1).all()
    assert np.max(np.abs(l1 - l2)) > 0.0


def test_golden_append():
    P.pin_golden_append(oracle.append_kv_ref)


def test_golden_chunked():
    P.pin_golden_chunked(oracle.paged_prefill_ref)


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_chunk_matches_full(layout):
    P.pin_chunk_matches_full(oracle.paged_prefill_ref, oracle.attention_ref, layout)


def test_sdpa_lower_right():
    P.pin_sdpa_lower_right(oracle.paged_prefill_ref)


def test_chunk_single_query_is_decode():
    P.pin_chunk_single_query_is_decode(oracle.paged_prefill_ref, oracle.paged_decode_ref)


def test_paged_prefill_rows_match_full():
    g = np.random.default_rng(141)
    hq, hkv, d, ps = 4, 2, 4, 4
    cases = [(5, 3), (0, 6)]
    seqs = [(g.standard_normal((p + n, hkv, d)), g.standard_normal((p + n, hkv, d))) for p, n in cases]
    kp, vp, bt = P._scatter_to_pages(seqs, ps, "NHD", g)
    cu = np.array([0, 3, 9])
    q = g.standard_normal((9, hq, d))
    lens = [8, 6]
    for causal in (False, True):
        o, l = oracle.paged_prefill_ref(q, cu, kp, vp, bt, lens, causal, 0.5, page_size=ps)
        rows = [(t, h) for t in range(9) for h in range(hq)]
        orr, lr = oracle.paged_prefill_rows_ref(q, cu, kp, vp, bt, lens, causal, 0.5, rows, page_size=ps)
        np.testing.assert_allclose(orr, o.reshape(-1, d), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lr, l.reshape(-1), rtol=0, atol=1e-14)


def test_visible_key_count_reduces_to_square_causal():
    for L in (1, 5):
        for i in range(L):
            assert oracle.visible_key_count(i, L, L, True) == i + 1
            assert oracle.visible_key_count(i, L, L, False) == L


def test_e4m3_codes():
    P.pin_e4m3_codes(oracle.e4m3_to_f64)


def test_golden_fp8_decode():
    P.pin_golden_fp8_decode(oracle.paged_decode_ref, oracle.dequantize_e4m3)


def test_empty_cache_decodes_to_zero():
    """A request with no cached token: O = 0 and LSE = -inf (the empty-key
    reading), next to a normal request that must be unaffected."""
    g = np.random.default_rng(151)
    kp = g.standard_normal((3, 4, 1, 2))
    vp = g.standard_normal((3, 4, 1, 2))
    bt = np.array([[0, 1], [-1, -1]])
    q = g.standard_normal((2, 1, 2))
    o, l = oracle.paged_decode_ref(q, kp, vp, bt, [5, 0], 0.5, page_size=4)
    assert np.array_equal(o[1], np.zeros((1, 2))) and np.isneginf(l[1, 0])
    K = np.concatenate([kp[0, :, 0], kp[1, :1, 0]])
    V = np.concatenate([vp[0, :, 0], vp[1, :1, 0]])
    ob, lb = oracle.partial_state_ref(q[0], K, V, 0.5)
    np.testing.assert_allclose(o[0], ob, atol=1e-14)
    np.testing.assert_allclose(l[0], lb, atol=1e-14)


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_cascade_matches_concatenation(layout):
    P.pin_cascade_matches_concatenation(oracle.cascade_decode_ref, oracle.partial_state_ref, layout)


def test_cascade_aligned_is_decode():
    P.pin_cascade_aligned_is_decode(oracle.cascade_decode_ref, oracle.paged_decode_ref)
