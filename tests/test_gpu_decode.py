"""GPU parity of the paged Flash-Decoding path against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import (JUMP_FACTORS, bf16_to_f64, compare, decode_device_inputs, decode_on_gpu,
                            jumping_keys_decode, to_dev_i32)

pytestmark = pytest.mark.gpu


def oracle_rows(inp, rows):
    return oracle.paged_decode_rows_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits,
                                        inp.block_table, inp.cache_seqlens, inp.scale, rows,
                                        inp.page_size, inp.layout, to_f64=W.as_f64)


def check_all_rows(inp, num_splits=0, what="", kernel="auto"):
    import exact_attention_148_b200 as fa
    assert fa.device_status(clear=True) == 0
    out, lse, plan = decode_on_gpu(inp, num_splits, kernel=kernel)
    assert fa.device_status(clear=True) == 0, what
    rows = [(b, h) for b in range(inp.batch) for h in range(inp.num_q_heads)]
    o_ref, l_ref = oracle_rows(inp, rows)
    compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1), o_ref, l_ref,
            what)
    return out, lse, plan


SMALL_LENS = [1, 63, 64, 65, 1000, 4097]


@pytest.mark.parametrize("num_splits", [0, 1, 2, 3, 16])
def test_small_batch_all_rows(num_splits):
    inp = W.make_decode(SMALL_LENS, 8, 2, 128, seed=200)
    check_all_rows(inp, num_splits, f"small decode splits={num_splits}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (32, 2), (6, 2), (12, 2), (8, 1)])
def test_group_sizes(d, hq, hkv):
    inp = W.make_decode([70, 1500, 129], hq, hkv, d, seed=300 + d + hq * 7 + hkv)
    check_all_rows(inp, 0, f"decode d={d} hq={hq} hkv={hkv}")
    check_all_rows(inp, 5, f"decode d={d} hq={hq} hkv={hkv} 5 splits")


@pytest.mark.parametrize("s", [1, 2, 4, 7, 8, 16, 32, 64])
def test_num_splits_sweep(s):
    inp = W.make_decode([8192 + 777, 4096], 4, 4, 128, seed=400)
    check_all_rows(inp, s, f"splits={s}")


def test_layouts_are_bit_identical():
    import torch
    inp = W.make_decode(SMALL_LENS, 8, 2, 128, seed=500)
    a = decode_on_gpu(inp, 3)
    b = decode_on_gpu(W.relayout(inp, "HND"), 3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_page_permutation_is_bit_identical(num_splits):
    import torch
    inp = W.make_decode(SMALL_LENS, 8, 2, 128, seed=600, extra_pages=5)
    a = decode_on_gpu(inp, num_splits)
    for seed in (1, 2):
        b = decode_on_gpu(W.permute_pages(inp, seed), num_splits)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_unused_slots_poisoned_with_nan():
    import torch
    inp = W.make_decode(SMALL_LENS, 8, 2, 128, seed=700, extra_pages=3)
    a = decode_on_gpu(inp, 2)
    b = decode_on_gpu(W.poison_unused(inp), 2)
    assert torch.isfinite(b[0].float()).all()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_zero_length_request():
    import torch
    inp = W.make_decode([0, 100, 0], 4, 2, 128, seed=800)
    out, lse, _ = decode_on_gpu(inp, 0)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isneginf(lse[2]))
    rows = [(1, h) for h in range(4)]
    o_ref, l_ref = oracle_rows(inp, rows)
    compare(bf16_to_f64(out[1]), lse[1].cpu().numpy(), o_ref, l_ref, "zero-length batch")


def test_isolation_between_requests():
    import torch
    inp = W.make_decode([300, 700], 4, 4, 128, seed=900)
    dev = decode_device_inputs(inp)
    a = decode_on_gpu(inp, 2, dev=dev)
    # overwrite request 0's pages
    for p in inp.block_table[0][:5]:
        dev["k"][int(p)] = 1.0
        dev["v"][int(p)] = -1.0
    b = decode_on_gpu(inp, 2, dev=dev)
    assert torch.equal(a[0][1], b[0][1]) and torch.equal(a[1][1], b[1][1])
    assert not torch.equal(a[0][0], b[0][0])


def test_deterministic():
    import torch
    inp = W.make_decode(SMALL_LENS, 8, 2, 128, seed=1000)
    dev = decode_device_inputs(inp)
    a = decode_on_gpu(inp, 3, dev=dev)
    b = decode_on_gpu(inp, 3, dev=dev)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("bad_id", ["past_end", "negative"])
def test_bad_page_id_is_reported_not_faulted(kernel, bad_id):
    """A block_table entry outside the pool is recorded and read as a page of
    zeros (the kernels replace it by one past the last page, which the tensor
    map's bounds turn into a zero fill); the other pages are unaffected."""
    import exact_attention_148_b200 as fa
    inp = W.make_decode([200], 4, 4, 128, seed=1100)
    fa.device_status(clear=True)
    bt = inp.block_table.copy()
    bt[0, 1] = inp.num_pages + 3 if bad_id == "past_end" else -5
    bad = W.DecodeInputs(inp.name, inp.q_bits, inp.k_pages_bits, inp.v_pages_bits, bt,
                         inp.cache_seqlens, inp.scale, inp.layout, inp.page_size)
    out, lse, _ = decode_on_gpu(bad, 1, kernel=kernel)
    assert fa.device_status(clear=True) == fa.FA_ERR_BAD_PAGE
    assert np.isfinite(out.float().cpu().numpy()).all()
    # the oracle on the same cache with that page's keys and values set to zero
    k = inp.k_pages_bits.copy()
    v = inp.v_pages_bits.copy()
    zero_page = inp.num_pages                # an extra all-zero page for the oracle only
    k = np.concatenate([k, np.zeros_like(k[:1])], axis=0)
    v = np.concatenate([v, np.zeros_like(v[:1])], axis=0)
    bt_ref = inp.block_table.copy()
    bt_ref[0, 1] = zero_page
    rows = [(0, h) for h in range(4)]
    o_ref, l_ref = oracle.paged_decode_rows_ref(inp.q_bits, k, v, bt_ref, inp.cache_seqlens, inp.scale,
                                                rows, inp.page_size, inp.layout, to_f64=W.as_f64)
    compare(bf16_to_f64(out[0]), lse[0].cpu().numpy(), o_ref, l_ref, f"bad page ({kernel}, {bad_id})")
    decode_on_gpu(inp, 1, kernel=kernel)
    assert fa.device_status(clear=True) == 0


def test_longer_cache_than_planned_is_reported():
    import exact_attention_148_b200 as fa
    inp = W.make_decode([640, 64], 4, 4, 128, seed=1200)
    plan = fa.decode_plan([128, 64], num_q_heads=4, num_kv_heads=4, head_dim=128,
                          max_pages_per_seq=inp.block_table.shape[1], num_splits=1)
    fa.device_status(clear=True)
    decode_on_gpu(inp, plan=plan)
    assert fa.device_status(clear=True) == fa.FA_ERR_PLAN_MISMATCH


_FULL_ORACLE = {}


def oracle_every_row(inp):
    """The oracle on every (request, head) row of a workload, kept for the
    workload last asked for (its inputs are seeded, so one result serves every
    split count and kernel)."""
    if inp.name not in _FULL_ORACLE:
        _FULL_ORACLE.clear()
        rows = [(b, h) for b in range(inp.batch) for h in range(inp.num_q_heads)]
        _FULL_ORACLE[inp.name] = oracle_rows(inp, rows)
    return _FULL_ORACLE[inp.name]


def check_every_row(inp, settings, what):
    """Every output row of the full-size workload against the oracle, for each
    (num_splits, kernel) in settings, in the launch configuration bench.py times."""
    import exact_attention_148_b200 as fa
    o_ref, l_ref = oracle_every_row(inp)
    dev = decode_device_inputs(inp)
    fa.device_status(clear=True)
    for s, kernel in settings:
        out, lse, plan = decode_on_gpu(inp, s, dev=dev, kernel=kernel)
        compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1), o_ref, l_ref,
                f"{what} splits={s or 'auto'} ({plan.info.max_splits}) kernel={kernel}")
        assert fa.device_status(clear=True) == 0, what


def test_paged_decode_batch_config_every_row():
    inp = W.paged_decode_batch()
    check_every_row(inp, [(0, "auto"), (0, "cuda_cores"), (16, "auto")],
                    "paged decode batch (64 req, 32q/8kv)")


def test_long_split_decode_config_every_row():
    inp = W.long_split_decode()
    check_every_row(inp, [(0, "auto"), (1, "auto"), (8, "auto"), (64, "auto"), (0, "tensor_cores")],
                    "long split decode (4 x 131072)")


def test_ragged_split_decode_config_every_row():
    inp = W.ragged_split_decode()
    check_every_row(inp, [(0, "auto"), (64, "auto"), (0, "tensor_cores")],
                    "ragged split decode (1 x 131072 + 63 x 2048)")


@pytest.mark.parametrize("kernel", ["tensor_cores", "cuda_cores"])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (6, 2), (12, 1), (8, 1)])
def test_group_sizes_both_kernels(hq, hkv, kernel):
    inp = W.make_decode([70, 1500, 129, 0, 4097], hq, hkv, 128, seed=900 + hq * 7 + hkv)
    check_all_rows(inp, 0, f"decode {kernel} hq={hq} hkv={hkv}", kernel)
    check_all_rows(inp, 5, f"decode {kernel} hq={hq} hkv={hkv} 5 splits", kernel)


def test_tensor_core_poisoned_and_permuted():
    import torch
    inp = W.poison_unused(W.make_decode(SMALL_LENS, 16, 2, 128, seed=950, extra_pages=4))
    check_all_rows(inp, 3, "tc poisoned", "tensor_cores")
    a = decode_on_gpu(inp, 3, kernel="tensor_cores")
    b = decode_on_gpu(W.permute_pages(inp, 7), 3, kernel="tensor_cores")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    c = decode_on_gpu(W.relayout(inp, "HND"), 3, kernel="tensor_cores")
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])


@pytest.mark.parametrize("kernel", ["tensor_cores", "cuda_cores"])
@pytest.mark.parametrize("num_splits", [0, 1, 5])
def test_score_jumps_between_key_blocks(kernel, num_splits):
    """Cached keys whose scores jump by tens to hundreds (base 2) from one
    128-key block to the next: every split's online softmax and the log-sum-exp
    merge across splits, against the oracle."""
    inp = jumping_keys_decode(W.make_decode([1000, 129, 2500, 64, 700], 8, 2, 128, seed=750), JUMP_FACTORS)
    check_all_rows(inp, num_splits, f"decode score jumps {kernel} splits={num_splits}", kernel=kernel)
