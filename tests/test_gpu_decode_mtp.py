"""GPU parity of multi-token decode (several query tokens per request, e.g.
speculative verification) on the tensor-core split kernel, against the fp64
oracle's chunked prefill (a chunk of q_len tokens that are the last q_len
entries of the cache)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import bf16_to_f64, compare, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


def _dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def run(inp, num_splits=0):
    import exact_attention_148_b200 as fa
    fp8 = inp.kv_elem_bytes == 1
    q = to_dev_bf16(inp.q_bits)
    kp = _dev_u8(inp.k_pages_bits) if fp8 else to_dev_bf16(inp.k_pages_bits)
    vp = _dev_u8(inp.v_pages_bits) if fp8 else to_dev_bf16(inp.v_pages_bits)
    bt, lens = to_dev_i32(inp.block_table), to_dev_i32(inp.cache_seqlens)
    plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=inp.num_q_heads,
                          num_kv_heads=inp.num_kv_heads, head_dim=inp.head_dim,
                          page_size=inp.page_size, max_pages_per_seq=inp.block_table.shape[1],
                          num_splits=num_splits, kv_dtype="e4m3" if fp8 else "bf16",
                          q_len=inp.q_len)
    assert plan.info.tensor_cores == 1 and plan.info.q_len == inp.q_len
    if fp8:
        return fa.decode_paged_fp8(q, kp, vp, bt, lens, plan, k_scale=inp.extra["k_scale"],
                                   v_scale=inp.extra["v_scale"], layout=inp.layout, scale=inp.scale)
    return fa.decode_paged(q, kp, vp, bt, lens, plan, layout=inp.layout, scale=inp.scale)


def oracle_all(inp):
    B, QL, Hq, d = inp.q_bits.shape
    qp = inp.q_bits.reshape(B * QL, Hq, d)
    cu = np.arange(B + 1) * QL
    conv = {}
    if inp.kv_elem_bytes == 1:
        ks, vs = inp.extra["k_scale"], inp.extra["v_scale"]
        conv = dict(k_to_f64=lambda a: oracle.dequantize_e4m3(a, ks),
                    v_to_f64=lambda a: oracle.dequantize_e4m3(a, vs))
    o, l = oracle.paged_prefill_ref(qp, cu, inp.k_pages_bits, inp.v_pages_bits, inp.block_table,
                                    inp.cache_seqlens, True, inp.scale, inp.page_size, inp.layout,
                                    to_f64=W.as_f64, **conv)
    return o.reshape(B, QL, Hq, d), l.reshape(B, QL, Hq)


def check(inp, num_splits=0, what=""):
    import exact_attention_148_b200 as fa
    assert fa.device_status(clear=True) == 0
    out, lse = run(inp, num_splits)
    o_ref, l_ref = oracle_all(inp)
    compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1),
            o_ref.reshape(-1, inp.head_dim), l_ref.reshape(-1), what)
    assert fa.device_status(clear=True) == 0
    return out, lse


LENS = [2, 63, 64, 65, 1000, 4097, 129]


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("q_len,hq,hkv", [(2, 8, 2), (3, 8, 2), (4, 8, 2), (2, 16, 2), (16, 2, 2),
                                          (5, 3, 1), (8, 4, 2)])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_multi_token_all_rows(q_len, hq, hkv, fp8, num_splits):
    inp = W.make_decode([max(L, q_len) for L in LENS], hq, hkv, 128, seed=1000 + q_len * 31 + hq,
                        q_len=q_len, extra_pages=2)
    if fp8:
        inp = W.to_fp8_cache(inp)
    check(inp, num_splits, f"multi-token q_len={q_len} hq={hq} hkv={hkv} fp8={fp8} s={num_splits}")


def test_single_token_plan_equals_plain_decode():
    """q_len = 1 through the 4-D path gives the plain decode's bits."""
    import torch
    import exact_attention_148_b200 as fa
    inp = W.make_decode(LENS, 8, 2, 128, seed=1100)
    q = to_dev_bf16(inp.q_bits)
    kp, vp = to_dev_bf16(inp.k_pages_bits), to_dev_bf16(inp.v_pages_bits)
    bt, lens = to_dev_i32(inp.block_table), to_dev_i32(inp.cache_seqlens)
    kw = dict(num_q_heads=8, num_kv_heads=2, head_dim=128, max_pages_per_seq=inp.block_table.shape[1],
              num_splits=3, kernel="tensor_cores")
    a = fa.decode_paged(q, kp, vp, bt, lens, fa.decode_plan(inp.cache_seqlens, **kw))
    b = fa.decode_paged(q[:, None], kp, vp, bt, lens, fa.decode_plan(inp.cache_seqlens, q_len=1, **kw))
    assert torch.equal(a[0], b[0].view_as(a[0])) and torch.equal(a[1], b[1].view_as(a[1]))


def test_poisoned_and_permuted():
    import torch
    inp = W.poison_unused(W.make_decode([max(L, 4) for L in LENS], 8, 2, 128, seed=1200, q_len=4,
                                        extra_pages=3))
    check(inp, 2, "multi-token poisoned")
    a = run(inp, 2)
    b = run(W.permute_pages(inp, 4), 2)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_full_size_sampled_rows():
    inp = W.speculative_decode_batch()
    out, lse = run(inp)
    g = np.random.default_rng(19)
    B, QL, Hq, d = inp.q_bits.shape
    rows = [(int(b) * QL + int(t), int(h)) for b, t, h in zip(g.integers(0, B, 40), g.integers(0, QL, 40),
                                                           g.integers(0, Hq, 40))]
    qp = inp.q_bits.reshape(B * QL, Hq, d)
    o_ref, l_ref = oracle.paged_prefill_rows_ref(qp, np.arange(B + 1) * QL, inp.k_pages_bits,
                                                 inp.v_pages_bits, inp.block_table, inp.cache_seqlens,
                                                 True, inp.scale, rows, inp.page_size, inp.layout,
                                                 to_f64=W.as_f64)
    ti = np.array([r[0] for r in rows])
    hi = np.array([r[1] for r in rows])
    o = out.float().cpu().numpy().reshape(B * QL, Hq, d)[ti, hi].astype(np.float64)
    compare(o, lse.cpu().numpy().reshape(B * QL, Hq)[ti, hi], o_ref, l_ref, "multi-token full size")
