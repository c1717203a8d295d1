"""The seeded input generators (workloads/) that feed both the oracle and the
kernels: page tables are a permutation of the pool (no page shared unless the
recipe shares it), unused table slots are -1, shapes follow the layout, the
draws are bf16-rounded N(0,1) and reproducible from the seed, and the E4M3
quantiser never writes the NaN code."""
import numpy as np
import pytest

import workloads as W


def _used_pages(block_table, lens, page_size=64):
    return [block_table[b, :(int(L) + page_size - 1) // page_size] for b, L in enumerate(lens)]


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_decode_pages_are_a_permutation(layout):
    lens = [1, 63, 64, 65, 0, 700, 4097]
    inp = W.make_decode(lens, 8, 2, 64, seed=11, layout=layout, extra_pages=3)
    used = _used_pages(inp.block_table, lens)
    ids = np.concatenate(used)
    assert len(np.unique(ids)) == len(ids)                   # no page read by two requests
    assert inp.num_pages == len(ids) + 3                     # plus the spare pages
    assert ids.min() >= 0 and ids.max() < inp.num_pages
    for b, L in enumerate(lens):                             # slots past a request's pages are -1
        assert (inp.block_table[b, (L + 63) // 64:] == -1).all()
    P, a, b_, d = inp.k_pages_bits.shape
    assert (a, b_) == ((64, 2) if layout == "NHD" else (2, 64)) and d == 64
    assert inp.q_bits.shape == (len(lens), 8, 64)
    assert list(inp.cache_seqlens) == lens


def test_multi_token_query_shape():
    inp = W.make_decode([100, 200], 8, 2, 128, seed=1, q_len=3)
    assert inp.q_bits.shape == (2, 3, 8, 128) and inp.q_len == 3


def test_draws_are_seeded_bf16_normals():
    a = W.make_decode([3000, 2000], 16, 4, 128, seed=5)
    b = W.make_decode([3000, 2000], 16, 4, 128, seed=5)
    c = W.make_decode([3000, 2000], 16, 4, 128, seed=6)
    assert np.array_equal(a.k_pages_bits, b.k_pages_bits) and np.array_equal(a.block_table, b.block_table)
    assert not np.array_equal(a.k_pages_bits, c.k_pages_bits)
    x = W.as_f64(a.k_pages_bits).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # bf16 bit patterns: the low 16 bits of the float32 are zero after widening
    f = W.bf16_bits_to_f32(a.v_pages_bits[:4])
    assert (f.view(np.uint32) & 0xFFFF == 0).all()


def test_chunked_prefill_recipe():
    prefix, chunk = [0, 130, 64, 1000], [5, 64, 1, 300]
    inp = W.make_chunked_prefill(prefix, chunk, 8, 2, 128, seed=3, extra_pages=2)
    assert list(inp.cu_seqlens_q) == [0, 5, 69, 70, 370]
    assert list(inp.cache_seqlens) == [p + c for p, c in zip(prefix, chunk)]
    ids = np.concatenate(_used_pages(inp.block_table, inp.cache_seqlens))
    assert len(np.unique(ids)) == len(ids) and inp.k_pages_bits.shape[0] == len(ids) + 2
    assert inp.k_new_bits.shape == (370, 2, 128) and inp.q_bits.shape == (370, 8, 128)


def test_cascade_prefix_and_suffix_pages_are_disjoint():
    casc = W.make_cascade(200, [0, 64, 65, 3], 8, 2, 128, seed=4)
    pre = set(casc.prefix_block_table.tolist())
    suf = np.concatenate(_used_pages(casc.block_table, casc.suffix_lens))
    assert len(pre) == 4 and len(np.unique(suf)) == len(suf) and not (pre & set(suf.tolist()))
    aligned = W.make_cascade(192, [0, 64, 65, 3], 8, 2, 128, seed=4)
    plain = aligned.as_plain_decode()                # prefix pages first in every row
    for b in range(aligned.batch):
        assert list(plain.block_table[b, :3]) == aligned.prefix_block_table.tolist()
    assert list(plain.cache_seqlens) == [192 + s for s in aligned.suffix_lens]


def test_prefill_recipe():
    inp = W.make_prefill([1, 127, 128, 129], 8, 2, 64, causal=False, seed=2)
    assert list(inp.cu_seqlens) == [0, 1, 128, 256, 385]
    assert inp.q_bits.shape == (385, 8, 64) and inp.k_bits.shape == (385, 2, 64)
    assert inp.causal is False and abs(inp.scale - 1 / 8) < 1e-12


def test_e4m3_quantiser_never_writes_nan():
    inp = W.to_fp8_cache(W.make_decode([5000], 4, 4, 128, seed=9))
    codes = np.concatenate([inp.k_pages_bits.ravel(), inp.v_pages_bits.ravel()])
    assert not np.isin(codes, [0x7F, 0xFF]).any()
    assert inp.extra["k_scale"] == pytest.approx(4.0 / 448.0)
    # saturation: values beyond +-448 * scale map to the largest finite code
    big = W.quantize_e4m3(np.array([1e6, -1e6], dtype=np.float32), 1.0)
    assert list(big) == [0x7E, 0xFE]
