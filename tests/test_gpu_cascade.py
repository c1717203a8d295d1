"""GPU parity of the cascade (shared-prefix) decode against the fp64 oracle:
plain attention of every request's query over the shared prefix followed by
its own suffix."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import bf16_to_f64, compare, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


def run(inp, num_splits=0, kernel="auto"):
    import exact_attention_148_b200 as fa
    q = to_dev_bf16(inp.q_bits)
    kp, vp = to_dev_bf16(inp.k_pages_bits), to_dev_bf16(inp.v_pages_bits)
    pre = to_dev_i32(inp.prefix_block_table if len(inp.prefix_block_table) else np.zeros(1, np.int32))
    bt, lens = to_dev_i32(inp.block_table), to_dev_i32(inp.suffix_lens)
    plan = fa.decode_plan(inp.suffix_lens, num_q_heads=inp.num_q_heads, num_kv_heads=inp.num_kv_heads,
                          head_dim=inp.head_dim, max_pages_per_seq=inp.block_table.shape[1],
                          num_splits=num_splits, kernel=kernel)
    return fa.cascade_decode(q, kp, vp, pre, inp.prefix_len, bt, lens, plan, layout=inp.layout,
                             scale=inp.scale)


def oracle_rows(inp, reqs=None):
    reqs = np.arange(inp.batch) if reqs is None else np.asarray(reqs)
    return oracle.cascade_decode_ref(inp.q_bits[reqs], inp.k_pages_bits, inp.v_pages_bits,
                                     inp.prefix_block_table, inp.prefix_len, inp.block_table[reqs],
                                     inp.suffix_lens[reqs], inp.scale, inp.page_size, inp.layout,
                                     to_f64=W.as_f64)


def check(inp, what, num_splits=0, kernel="auto"):
    import exact_attention_148_b200 as fa
    assert fa.device_status(clear=True) == 0
    out, lse = run(inp, num_splits, kernel)
    o_ref, l_ref = oracle_rows(inp)
    compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1),
            o_ref.reshape(-1, inp.head_dim), l_ref.reshape(-1), what)
    assert fa.device_status(clear=True) == 0
    return out, lse


SUFFIX = [0, 1, 63, 64, 65, 700, 2000, 5]


@pytest.mark.parametrize("prefix_len", [0, 1, 63, 64, 200, 1000, 3000])
def test_prefix_lengths(prefix_len):
    inp = W.make_cascade(prefix_len, SUFFIX, 8, 2, 128, seed=1300 + prefix_len, extra_pages=2)
    check(inp, f"cascade prefix={prefix_len}")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (6, 2), (16, 2), (8, 1), (32, 8)])
@pytest.mark.parametrize("kernel", ["tensor_cores", "cuda_cores"])
def test_group_sizes(hq, hkv, kernel):
    if kernel == "tensor_cores" and hq // hkv > 16:
        pytest.skip("group above the tensor-core limit")
    inp = W.make_cascade(777, SUFFIX, hq, hkv, 128, seed=1400 + hq + hkv)
    check(inp, f"cascade hq={hq} hkv={hkv} {kernel}", 3, kernel)


def test_more_than_one_query_tile():
    """150 requests: two 128-row query tiles over the prefix."""
    suf = np.random.default_rng(3).integers(0, 300, size=150)
    inp = W.make_cascade(1500, suf, 8, 2, 128, seed=1500, layout="HND")
    check(inp, "cascade 150 requests")


def test_d64():
    inp = W.make_cascade(500, SUFFIX, 8, 2, 64, seed=1600)
    check(inp, "cascade d=64")


def test_poisoned_unused_slots():
    """NaN in every pool slot outside the prefix and the suffixes."""
    inp = W.make_cascade(333, SUFFIX, 8, 2, 128, seed=1700, extra_pages=3)
    valid = np.zeros((inp.k_pages_bits.shape[0], inp.page_size), dtype=bool)
    for p in range((inp.prefix_len + 63) // 64):
        valid[inp.prefix_block_table[p], :min(64, inp.prefix_len - 64 * p)] = True
    for b in range(inp.batch):
        L = int(inp.suffix_lens[b])
        for p in range((L + 63) // 64):
            valid[inp.block_table[b, p], :min(64, L - 64 * p)] = True
    inp.k_pages_bits[~valid] = W.BF16_NAN_BITS
    inp.v_pages_bits[~valid] = W.BF16_NAN_BITS
    check(inp, "cascade poisoned")


def test_full_size_sampled_requests():
    inp = W.cascade_decode_batch()
    out, lse = run(inp)
    reqs = [0, 17, 40, 63]
    o_ref, l_ref = oracle_rows(inp, reqs)
    o = bf16_to_f64(out)[reqs]
    compare(o.reshape(-1, inp.head_dim), lse.cpu().numpy()[reqs].reshape(-1),
            o_ref.reshape(-1, inp.head_dim), l_ref.reshape(-1), "cascade full size")
