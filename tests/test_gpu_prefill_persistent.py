"""GPU parity of the prefill's two schedules: the persistent form (the default:
one CTA per SM taking work items from a counter, pipelines running across
items) and the grid form (FA_PREFILL_SCHEDULE=grid: one CTA per item).

Their per-tile arithmetic is the same, tile for tile, so the two forms must
agree bit for bit; the oracle comparisons and the counter checks (reset
between launches, one counter per stream, the grid form while a stream is
being captured) come on top.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import bf16_to_f64, compare, prefill_on_gpu, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


def both_forms(inp, monkeypatch, fp8=False):
    import exact_attention_148_b200 as fa
    from tests.test_gpu_prefill_fp8 import run_fp8
    run = run_fp8 if fp8 else prefill_on_gpu
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", "grid")
    grid = run(inp)
    assert fa.prefill_last_schedule() == "grid"
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    pers = run(inp)
    assert fa.prefill_last_schedule() == "persistent"
    return grid, pers


def assert_same(a, b):
    import torch
    assert torch.equal(a[0], b[0]), "O differs between the grid and persistent forms"
    assert torch.equal(a[1], b[1]), "LSE differs between the grid and persistent forms"


RAGGED = [1, 127, 128, 129, 300, 513]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 1), (8, 2), (3, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_small_varlen_bit_identical(d, hq, hkv, causal, monkeypatch):
    import exact_attention_148_b200 as fa
    inp = W.make_prefill(RAGGED, hq, hkv, d, causal=causal, seed=300 + d + hq + hkv)
    grid, pers = both_forms(inp, monkeypatch)
    assert_same(grid, pers)
    o_ref, l_ref = oracle.attention_ref(W.as_f64(inp.q_bits), W.as_f64(inp.k_bits), W.as_f64(inp.v_bits),
                                        inp.cu_seqlens, inp.causal, inp.scale)
    compare(bf16_to_f64(pers[0]), pers[1].cpu().numpy(), o_ref, l_ref, f"persistent d={d} {hq}/{hkv}")
    assert fa.device_status(clear=True) == 0


@pytest.mark.parametrize("hq,hkv,causal", [(4, 2, True), (3, 1, False)])
def test_fp8_bit_identical(hq, hkv, causal, monkeypatch):
    import exact_attention_148_b200 as fa
    inp = W.to_fp8_prefill(W.make_prefill(RAGGED, hq, hkv, 128, causal=causal, seed=310 + hq))
    grid, pers = both_forms(inp, monkeypatch, fp8=True)
    assert_same(grid, pers)
    assert fa.device_status(clear=True) == 0


def test_more_items_than_sms(monkeypatch):
    """Many items per CTA: a 2125-token GQA sequence and 40 short ones."""
    import exact_attention_148_b200 as fa
    inp = W.make_prefill([2048 + 77] + [130] * 40, 8, 2, 128, causal=True, seed=320)
    grid, pers = both_forms(inp, monkeypatch)
    assert_same(grid, pers)
    assert fa.device_status(clear=True) == 0


def test_counter_reset_between_launches(monkeypatch):
    """Back-to-back launches on one stream with different item counts."""
    import torch
    import exact_attention_148_b200 as fa
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    cases = [W.make_prefill(lens, 4, 2, 128, causal=True, seed=330 + i)
             for i, lens in enumerate(([700, 3], [129], [1000, 1000, 17], [1]))]
    first = [prefill_on_gpu(c) for c in cases]
    again = [prefill_on_gpu(c) for c in reversed(cases)][::-1]
    torch.cuda.synchronize()
    for a, b in zip(first, again):
        assert_same(a, b)
    assert fa.device_status(clear=True) == 0


def test_two_streams(monkeypatch):
    """Launches on two streams at once use separate counters."""
    import torch
    import exact_attention_148_b200 as fa
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    a_inp = W.make_prefill([3000, 513], 8, 2, 128, causal=True, seed=340)
    b_inp = W.make_prefill([2500, 700, 9], 4, 4, 128, causal=True, seed=341)
    want_a, want_b = prefill_on_gpu(a_inp), prefill_on_gpu(b_inp)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        got_a = prefill_on_gpu(a_inp, stream=s1)
    with torch.cuda.stream(s2):
        got_b = prefill_on_gpu(b_inp, stream=s2)
    torch.cuda.synchronize()
    assert_same(want_a, got_a)
    assert_same(want_b, got_b)
    assert fa.device_status(clear=True) == 0


def test_varlen_config_sampled(monkeypatch):
    from tests.test_gpu_prefill import check_sampled
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    check_sampled(W.varlen_causal_prefill(), 1024, 1, "persistent varlen causal prefill")


def test_long_gqa_config_sampled(monkeypatch):
    from tests.test_gpu_prefill import check_sampled
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    check_sampled(W.long_gqa_prefill(), 512, 2, "persistent 32K GQA causal prefill")


def test_capture_uses_the_grid_form(monkeypatch):
    """While a stream is being captured the library launches the grid form (a
    graph's replays could overlap other launches on one counter); replays give
    the eager persistent result bit for bit."""
    import torch
    import exact_attention_148_b200 as fa
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    inp = W.make_prefill([900, 130, 2000], 8, 2, 128, causal=True, seed=350)
    q, k, v = (to_dev_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    cu = to_dev_i32(inp.cu_seqlens)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)

    def step():
        fa.prefill(q, k, v, cu, causal=True, scale=inp.scale, out=out, lse=lse,
                   cu_seqlens_host=inp.cu_seqlens, stream=torch.cuda.current_stream())

    step()
    torch.cuda.synchronize()
    assert fa.prefill_last_schedule() == "persistent"
    want = (out.clone(), lse.clone())
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    assert fa.prefill_last_schedule() == "grid"
    out.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, want[0]) and torch.equal(lse, want[1])
    del g
    assert fa.device_status(clear=True) == 0
