"""GPU parity of the KV append and the chunked (paged) prefill against the
fp64 oracle."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import (JUMP_FACTORS, bf16_to_f64, chunked_device_inputs, chunked_on_gpu, compare,
                            jumping_keys_paged, oracle_pool_after_append, prefill_on_gpu, to_dev_bf16,
                            to_dev_i32)

pytestmark = pytest.mark.gpu


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _device_status():
    import exact_attention_148_b200 as fa
    return fa.device_status(clear=True)


def check_full(inp, what=""):
    assert _device_status() == 0
    out, lse, dev = chunked_on_gpu(inp)
    kp, vp = oracle_pool_after_append(inp)
    assert np.array_equal(_bits(dev["k"]), kp), f"{what}: K pool after append"
    assert np.array_equal(_bits(dev["v"]), vp), f"{what}: V pool after append"
    o_ref, l_ref = oracle.paged_prefill_ref(inp.q_bits, inp.cu_seqlens_q, kp, vp, inp.block_table,
                                            inp.cache_seqlens, inp.causal, inp.scale,
                                            inp.page_size, inp.layout, to_f64=W.as_f64)
    res = compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, what)
    assert _device_status() == 0
    return out, lse, res


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("layout", ["NHD", "HND"])
@pytest.mark.parametrize("causal", [True, False])
def test_tiny_all_rows(d, layout, causal):
    check_full(W.tiny_chunked_prefill(d, layout, causal), f"chunked d={d} {layout} causal={causal}")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (6, 2), (8, 2), (8, 1), (16, 2)])
def test_group_sizes(hq, hkv):
    inp = W.make_chunked_prefill([0, 333, 129, 1024], [200, 77, 300, 128], hq, hkv, 128,
                                 seed=700 + hq + hkv, extra_pages=2)
    check_full(inp, f"chunked hq={hq} hkv={hkv}")


def test_unused_slots_poisoned_with_nan():
    inp = W.poison_chunked(W.tiny_chunked_prefill())
    check_full(inp, "chunked poisoned")


def _schedule_cases():
    return {
        "tiny causal": W.tiny_chunked_prefill(),
        "tiny full d=64 HND": W.tiny_chunked_prefill(64, "HND", False),
        "odd group, page tails": W.make_chunked_prefill([0, 333, 129, 1024, 5], [200, 77, 300, 128, 1], 6, 2,
                                                        128, seed=730, extra_pages=2),
        "poisoned": W.poison_chunked(W.tiny_chunked_prefill()),
    }


@pytest.mark.parametrize("case", list(_schedule_cases()))
def test_persistent_and_grid_schedules_bit_identical(case, monkeypatch):
    """The persistent paged prefill (the default) and the grid form read the
    same tiles in the same order: bit-identical O and LSE, including NaN-filled
    page tails, which both zero before P V."""
    import torch
    import exact_attention_148_b200 as fa
    inp = _schedule_cases()[case]
    dev = chunked_device_inputs(inp)
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", "grid")
    a = chunked_on_gpu(inp, dev=dev)
    assert fa.prefill_last_schedule() == "grid"
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    b = chunked_on_gpu(inp, dev=dev, append=False)
    assert fa.prefill_last_schedule() == "persistent"
    assert torch.equal(a[0], b[0]), f"{case}: O differs between the schedules"
    assert torch.equal(a[1], b[1]), f"{case}: LSE differs between the schedules"
    assert _device_status() == 0


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_score_jumps_between_key_tiles(schedule, monkeypatch):
    """Cached and new keys whose scores jump by tens to hundreds (base 2) from
    one 128-key tile to the next, through the block table: the reference
    maximum raised late or at once, against the oracle."""
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", schedule)
    inp = jumping_keys_paged(W.make_chunked_prefill([0, 333, 700, 1024], [200, 77, 300, 129], 8, 2, 128,
                                                    seed=740, extra_pages=2), JUMP_FACTORS)
    check_full(inp, f"chunked score jumps ({schedule})")


def test_empty_prefix_is_bit_identical_to_prefill():
    """With nothing cached the chunked kernel sees the same tiles and masks as
    the packed prefill: the results must agree bit for bit."""
    import torch
    pre = W.make_prefill([300, 128, 1000, 1], 8, 2, 128, causal=True, seed=710)
    o1, l1 = prefill_on_gpu(pre)
    ch = W.make_chunked_prefill([0, 0, 0, 0], [300, 128, 1000, 1], 8, 2, 128, seed=711)
    ch.q_bits, ch.k_new_bits, ch.v_new_bits = pre.q_bits, pre.k_bits, pre.v_bits
    o2, l2, _ = chunked_on_gpu(ch)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_page_permutation_is_bit_identical():
    import torch
    inp = W.tiny_chunked_prefill()
    a = chunked_on_gpu(inp)
    P = inp.num_pages
    perm = np.random.default_rng(5).permutation(P).astype(np.int32)
    moved = W.ChunkedPrefillInputs(**{**inp.__dict__})
    moved.k_pages_bits = np.empty_like(inp.k_pages_bits)
    moved.v_pages_bits = np.empty_like(inp.v_pages_bits)
    moved.k_pages_bits[perm] = inp.k_pages_bits
    moved.v_pages_bits[perm] = inp.v_pages_bits
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    moved.block_table = bt
    b = chunked_on_gpu(moved)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_append_only_touches_new_slots():
    inp = W.make_chunked_prefill([5, 64, 0], [60, 1, 129], 4, 2, 64, seed=720, extra_pages=4)
    dev = chunked_device_inputs(inp)
    import exact_attention_148_b200 as fa
    fa.append_kv(dev["k_new"], dev["v_new"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"])
    kp, vp = oracle_pool_after_append(inp)
    assert np.array_equal(_bits(dev["k"]), kp) and np.array_equal(_bits(dev["v"]), vp)
    assert _device_status() == 0


def test_bad_page_id_is_reported_not_faulted():
    import exact_attention_148_b200 as fa
    inp = W.tiny_chunked_prefill()
    dev = chunked_device_inputs(inp)
    fa.append_kv(dev["k_new"], dev["v_new"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"])
    assert _device_status() == 0
    bt = inp.block_table.copy()
    bt[2, 3] = inp.num_pages + 1000            # outside the pool (request 2 uses 15 pages)
    dev["bt"] = to_dev_i32(bt)
    out, lse, _ = chunked_on_gpu(inp, dev=dev, append=False)
    assert _device_status() == fa.FA_ERR_BAD_PAGE
    fa.append_kv(dev["k_new"], dev["v_new"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"])
    assert _device_status() in (0, fa.FA_ERR_BAD_PAGE)   # only if a new row maps to that page
    # the other requests are untouched by the bad entry
    kp, vp = oracle_pool_after_append(inp)
    o_ref, l_ref = oracle.paged_prefill_ref(inp.q_bits, inp.cu_seqlens_q, kp, vp, inp.block_table,
                                            inp.cache_seqlens, True, inp.scale, to_f64=W.as_f64)
    rows = np.r_[0:inp.cu_seqlens_q[2], inp.cu_seqlens_q[3]:inp.cu_seqlens_q[-1]]
    compare(bf16_to_f64(out)[rows], lse.cpu().numpy()[rows], o_ref[rows], l_ref[rows], "bad page")


def test_device_lengths_shorter_than_chunk_are_reported():
    import exact_attention_148_b200 as fa
    inp = W.tiny_chunked_prefill()
    dev = chunked_device_inputs(inp)
    bad = inp.cache_seqlens.copy()
    bad[0] = 3                                   # request 0 has a 130-token chunk
    dev["lens"] = to_dev_i32(bad)
    fa.prefill_paged(dev["q"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"],
                     cu_seqlens_q_host=inp.cu_seqlens_q, cache_seqlens_host=inp.cache_seqlens)
    assert _device_status() == fa.FA_ERR_PLAN_MISMATCH


def test_full_size_sampled_rows():
    """The bench workload (8 requests, 32 q / 8 kv heads) on sampled rows:
    every request's first and last query, plus random ones."""
    inp = W.chunked_prefill_batch()
    out, lse, dev = chunked_on_gpu(inp)
    g = np.random.default_rng(9)
    cu = inp.cu_seqlens_q
    rows = []
    for b in range(inp.batch):
        for t in (int(cu[b]), int(cu[b + 1]) - 1, int(g.integers(cu[b], cu[b + 1]))):
            for h in (0, int(g.integers(0, inp.num_q_heads)), inp.num_q_heads - 1):
                rows.append((t, h))
    kp, vp = oracle_pool_after_append(inp)
    o_ref, l_ref = oracle.paged_prefill_rows_ref(inp.q_bits, cu, kp, vp, inp.block_table,
                                                 inp.cache_seqlens, True, inp.scale, rows,
                                                 inp.page_size, inp.layout, to_f64=W.as_f64)
    ti = np.array([r[0] for r in rows])
    hi = np.array([r[1] for r in rows])
    o = out.float().cpu().numpy()[ti, hi].astype(np.float64)
    compare(o, lse.cpu().numpy()[ti, hi], o_ref, l_ref, "chunked full size")
    assert _device_status() == 0
