"""GPU parity of fa_prefill against the fp64 oracle (run on a B200)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import (JUMP_FACTORS, bf16_to_f64, compare, jumping_keys, prefill_on_gpu, to_dev_bf16,
                            to_dev_i32)

pytestmark = pytest.mark.gpu


def oracle_full(inp):
    return oracle.attention_ref(W.as_f64(inp.q_bits), W.as_f64(inp.k_bits), W.as_f64(inp.v_bits),
                                inp.cu_seqlens, inp.causal, inp.scale)


def check_full(inp, what):
    out, lse = prefill_on_gpu(inp)
    o_ref, l_ref = oracle_full(inp)
    return compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, what)


def sample_rows(inp, n, seed):
    """Random (token, head) rows plus every sequence's first and last rows."""
    g = np.random.default_rng(seed)
    T = int(inp.cu_seqlens[-1])
    H = inp.num_q_heads
    rows = set()
    for b in range(len(inp.cu_seqlens) - 1):
        for t in (int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1]) - 1):
            rows.add((t, int(g.integers(H))))
    while len(rows) < n:
        rows.add((int(g.integers(T)), int(g.integers(H))))
    return sorted(rows)


def check_sampled(inp, n, seed, what):
    out, lse = prefill_on_gpu(inp)
    rows = sample_rows(inp, n, seed)
    q = W.bf16_bits_to_f32(inp.q_bits)
    k = W.bf16_bits_to_f32(inp.k_bits)
    v = W.bf16_bits_to_f32(inp.v_bits)
    o_ref, l_ref = oracle.attention_rows_ref(q, k, v, inp.cu_seqlens, inp.causal, inp.scale, rows)
    idx_t = np.array([r[0] for r in rows])
    idx_h = np.array([r[1] for r in rows])
    o = out.float().cpu().numpy()[idx_t, idx_h].astype(np.float64)
    l = lse.cpu().numpy()[idx_t, idx_h]
    return compare(o, l, o_ref, l_ref, what)


def test_tiny_causal_prefill():
    check_full(W.tiny_causal_prefill(), "tiny causal prefill")


RAGGED = [1, 127, 128, 129, 300, 513]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 1), (8, 2), (16, 2), (8, 1), (6, 2), (3, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_small_varlen(d, hq, hkv, causal):
    inp = W.make_prefill(RAGGED, hq, hkv, d, causal=causal, seed=100 + d + hq + hkv)
    check_full(inp, f"varlen d={d} hq={hq} hkv={hkv} causal={causal}")


def test_explicit_scale_and_single_token():
    inp = W.make_prefill([1], 2, 2, 128, causal=True, scale=0.3, seed=7)
    check_full(inp, "single token")
    inp = W.make_prefill([700, 1], 2, 2, 64, causal=False, scale=0.05, seed=8)
    check_full(inp, "non-causal explicit scale")


def test_multi_tile_long_sequence():
    inp = W.make_prefill([2048 + 77], 4, 2, 128, causal=True, seed=11)
    check_full(inp, "2125-token causal GQA")


def test_varlen_config_sampled():
    inp = W.varlen_causal_prefill()
    check_sampled(inp, 1024, 1, "varlen causal prefill (8 seqs, 32 heads)")


def test_long_gqa_config_sampled():
    inp = W.long_gqa_prefill()
    check_sampled(inp, 512, 2, "32K GQA causal prefill")


def check_whole_heads(inp, heads, what):
    """Every row of the chosen query heads of a full-size workload against the
    oracle run on those heads and their kv heads alone (heads are independent,
    and head h reads kv head h // (Hq / Hkv))."""
    out, lse = prefill_on_gpu(inp)
    G = inp.num_q_heads // inp.num_kv_heads
    # one chosen q head per kv head, ordered by kv head, so that q head j of the
    # sub-problem maps onto its kv head j
    heads = sorted(heads)
    kv = [h // G for h in heads]
    assert len(set(kv)) == len(kv), "one q head per kv head"
    o_ref, l_ref = oracle.attention_ref(W.as_f64(inp.q_bits[:, heads]), W.as_f64(inp.k_bits[:, kv]),
                                        W.as_f64(inp.v_bits[:, kv]), inp.cu_seqlens, inp.causal,
                                        inp.scale)
    o = bf16_to_f64(out[:, heads])
    l = lse.cpu().numpy()[:, heads]
    return compare(o, l, o_ref, l_ref, what)


def test_varlen_config_whole_heads():
    """Four whole heads (every one of the 20,730 packed rows) of the varlen config."""
    inp = W.varlen_causal_prefill()
    check_whole_heads(inp, [0, 9, 22, 31], "varlen causal prefill, heads 0/9/22/31")


def test_long_gqa_config_dense_rows():
    """The 32K GQA config: every 32nd row of two heads on different kv heads,
    plus every row of the first and last 128-row q tiles of both."""
    inp = W.long_gqa_prefill()
    out, lse = prefill_on_gpu(inp)
    T = int(inp.cu_seqlens[-1])
    heads = (0, 31)
    tok = sorted(set(range(0, T, 32)) | set(range(128)) | set(range(T - 128, T)))
    G = inp.num_q_heads // inp.num_kv_heads
    q = W.bf16_bits_to_f32(inp.q_bits[:, list(heads)])
    k = W.bf16_bits_to_f32(inp.k_bits[:, [h // G for h in heads]]).astype(np.float64)
    v = W.bf16_bits_to_f32(inp.v_bits[:, [h // G for h in heads]]).astype(np.float64)
    rows = [(t, j) for j in range(len(heads)) for t in tok]
    o_ref, l_ref = oracle.attention_rows_ref(q, k, v, inp.cu_seqlens, inp.causal, inp.scale, rows)
    ti = np.array([r[0] for r in rows])
    hi = np.array([heads[r[1]] for r in rows])
    o = out.float().cpu().numpy()[ti, hi].astype(np.float64)
    l = lse.cpu().numpy()[ti, hi]
    compare(o, l, o_ref, l_ref, "32K GQA causal prefill, dense rows of heads 0 and 31")


def test_sequences_are_isolated():
    """Changing one sequence's tokens leaves every other sequence bit-identical."""
    import torch
    inp = W.make_prefill([300, 200, 129], 4, 2, 128, causal=True, seed=21)
    out1, lse1 = prefill_on_gpu(inp)
    inp2 = W.make_prefill([300, 200, 129], 4, 2, 128, causal=True, seed=21)
    s0, s1 = int(inp.cu_seqlens[1]), int(inp.cu_seqlens[2])
    g = np.random.default_rng(5)
    for arr in (inp2.q_bits, inp2.k_bits, inp2.v_bits):
        arr[s0:s1] = W.f32_to_bf16_bits(g.standard_normal(arr[s0:s1].shape).astype(np.float32))
    out2, lse2 = prefill_on_gpu(inp2)
    keep = np.r_[0:s0, s1:int(inp.cu_seqlens[-1])]
    assert torch.equal(out1[keep], out2[keep])
    assert torch.equal(lse1[keep], lse2[keep])
    assert not torch.equal(out1[s0:s1], out2[s0:s1])


def test_deterministic():
    import torch
    inp = W.make_prefill([1000, 333], 8, 2, 128, causal=True, seed=31)
    a = prefill_on_gpu(inp)
    b = prefill_on_gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_output_only_16_byte_aligned(schedule, monkeypatch):
    """An `out` that is 16- but not 32-byte aligned takes the 16-byte stores;
    its bytes equal those of a 32-byte aligned `out`."""
    import torch
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", schedule)
    inp = W.make_prefill([300, 129], 4, 2, 128, causal=True, seed=43)
    a, la = prefill_on_gpu(inp)
    T, H, d = a.shape
    buf = torch.empty(T * H * d + 8, dtype=torch.bfloat16, device=a.device)
    out = buf[8:].view(T, H, d)   # 16 bytes past a 256-byte aligned allocation
    assert out.data_ptr() % 32 == 16
    b, lb = prefill_on_gpu(inp, out=out)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_score_jumps_between_key_tiles(schedule, monkeypatch):
    """Scores that jump by tens to hundreds (base 2) from one key tile to the
    next: the reference maximum raised a tile late, and re-referenced at once
    where a tile's P would otherwise overflow, against the oracle."""
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", schedule)
    inp = jumping_keys(W.make_prefill([700, 300, 1000, 129], 4, 2, 128, causal=True, seed=47), JUMP_FACTORS)
    check_full(inp, f"score jumps ({schedule})")
    inp = jumping_keys(W.make_prefill([1000, 257], 2, 2, 64, causal=False, seed=48), [1.0, 6.0, 1.0, 16.0, 2.0])
    check_full(inp, f"score jumps, d=64, full attention ({schedule})")


def test_without_lse_matches():
    import torch
    inp = W.make_prefill([257], 2, 2, 128, causal=True, seed=41)
    a, _ = prefill_on_gpu(inp)
    b, none = prefill_on_gpu(inp, return_lse=False)
    assert none is None and torch.equal(a, b)


def test_device_status_clean_after_prefill():
    import exact_attention_148_b200 as fa
    inp = W.make_prefill([129], 2, 2, 64, causal=True, seed=51)
    prefill_on_gpu(inp)
    assert fa.device_status() == 0


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_device_offsets_disagreeing_with_host_are_reported(schedule, monkeypatch):
    """cu_seqlens_dev must equal cu_seqlens_host.  A device sequence that
    leaves the T packed rows, or whose tile count differs from the host's, is
    recorded as FA_ERR_PLAN_MISMATCH by the kernel and skipped; the other
    sequences are computed as usual."""
    import torch
    import exact_attention_148_b200 as fa
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", schedule)
    inp = W.make_prefill([200, 400, 300], 4, 2, 128, causal=True, seed=61)
    q, k, v = (to_dev_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    want, want_lse = prefill_on_gpu(inp)
    fa.device_status(clear=True)
    # sequence 1 runs past T on the device (the host says it ends at 600)
    bad = inp.cu_seqlens.copy()
    bad[2] = bad[3] + 100
    out = torch.zeros_like(want)
    lse = torch.zeros_like(want_lse)
    fa.prefill(q, k, v, to_dev_i32(bad), causal=True, scale=inp.scale, out=out, lse=lse,
               cu_seqlens_host=inp.cu_seqlens)
    assert fa.device_status(clear=True) == fa.FA_ERR_PLAN_MISMATCH
    s0, s1 = int(inp.cu_seqlens[0]), int(inp.cu_seqlens[1])
    assert torch.equal(out[s0:s1], want[s0:s1]) and torch.equal(lse[s0:s1], want_lse[s0:s1])
    # sequence 0 one tile longer on the device than on the host
    bad = inp.cu_seqlens.copy()
    bad[1] = 260
    fa.prefill(q, k, v, to_dev_i32(bad), causal=True, scale=inp.scale, out=out, lse=lse,
               cu_seqlens_host=inp.cu_seqlens)
    assert fa.device_status(clear=True) == fa.FA_ERR_PLAN_MISMATCH
    # the consistent call afterwards is clean and unchanged
    again, again_lse = prefill_on_gpu(inp)
    assert fa.device_status(clear=True) == 0
    assert torch.equal(again, want) and torch.equal(again_lse, want_lse)
