"""GPU parity of the FP8 (E4M3) KV-cache decode against the fp64 oracle run
on the dequantised cache."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import (JUMP_FACTORS, bf16_to_f64, compare, decode_device_inputs, jumping_keys_decode,
                            to_dev_bf16, to_dev_i32)

pytestmark = pytest.mark.gpu


def _dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def fp8_device_inputs(inp):
    return dict(q=to_dev_bf16(inp.q_bits), k=_dev_u8(inp.k_pages_bits), v=_dev_u8(inp.v_pages_bits),
                bt=to_dev_i32(inp.block_table), lens=to_dev_i32(inp.cache_seqlens))


def run_fp8(inp, num_splits=0, dev=None, kernel="auto"):
    import exact_attention_148_b200 as fa
    dev = dev or fp8_device_inputs(inp)
    plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=inp.num_q_heads,
                          num_kv_heads=inp.num_kv_heads, head_dim=inp.head_dim,
                          page_size=inp.page_size, max_pages_per_seq=inp.block_table.shape[1],
                          num_splits=num_splits, kv_dtype="e4m3", kernel=kernel)
    out, lse = fa.decode_paged_fp8(dev["q"], dev["k"], dev["v"], dev["bt"], dev["lens"], plan,
                                   k_scale=inp.extra["k_scale"], v_scale=inp.extra["v_scale"],
                                   layout=inp.layout, scale=inp.scale)
    return out, lse


def oracle_rows(inp, rows):
    ks, vs = inp.extra["k_scale"], inp.extra["v_scale"]
    return oracle.paged_decode_rows_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits,
                                        inp.block_table, inp.cache_seqlens, inp.scale, rows,
                                        inp.page_size, inp.layout, to_f64=W.as_f64,
                                        k_to_f64=lambda a: oracle.dequantize_e4m3(a, ks),
                                        v_to_f64=lambda a: oracle.dequantize_e4m3(a, vs))


def check_all_rows(inp, num_splits=0, what="", kernel="auto"):
    import exact_attention_148_b200 as fa
    assert fa.device_status(clear=True) == 0
    out, lse = run_fp8(inp, num_splits, kernel=kernel)
    rows = [(b, h) for b in range(inp.batch) for h in range(inp.num_q_heads)]
    o_ref, l_ref = oracle_rows(inp, rows)
    compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1), o_ref, l_ref,
            what)
    assert fa.device_status(clear=True) == 0
    return out, lse


SMALL_LENS = [1, 63, 64, 65, 1000, 4097, 0]


KERNELS = ["tensor_cores", "cuda_cores"]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("num_splits", [0, 1, 3, 16])
def test_small_batch_all_rows(num_splits, kernel):
    inp = W.to_fp8_cache(W.make_decode(SMALL_LENS, 8, 2, 128, seed=800))
    check_all_rows(inp, num_splits, f"fp8 decode splits={num_splits} {kernel}", kernel)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2), (6, 2), (8, 1), (32, 2), (12, 1)])
def test_group_sizes(d, hq, hkv):
    """Automatic kernel choice: tensor cores at d = 128 for groups up to 16."""
    inp = W.to_fp8_cache(W.make_decode([70, 1500, 129], hq, hkv, d, seed=810 + d + hq + hkv))
    check_all_rows(inp, 0, f"fp8 d={d} hq={hq} hkv={hkv}")
    check_all_rows(inp, 4, f"fp8 d={d} hq={hq} hkv={hkv} 4 splits")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2), (6, 2)])
def test_group_sizes_cuda_cores(hq, hkv):
    inp = W.to_fp8_cache(W.make_decode([70, 1500, 129], hq, hkv, 128, seed=815 + hq + hkv))
    check_all_rows(inp, 3, f"fp8 cuda cores hq={hq} hkv={hkv}", "cuda_cores")


def test_hnd_layout_is_bit_identical():
    import torch
    inp = W.to_fp8_cache(W.make_decode(SMALL_LENS, 8, 2, 128, seed=820))
    a = run_fp8(inp, 3)
    b = run_fp8(W.relayout(inp, "HND"), 3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_page_permutation_is_bit_identical():
    import torch
    inp = W.to_fp8_cache(W.make_decode(SMALL_LENS, 8, 2, 128, seed=830, extra_pages=4))
    a = run_fp8(inp, 2)
    b = run_fp8(W.permute_pages(inp, 3), 2)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kernel", KERNELS)
def test_unused_slots_hold_nan_codes(kernel):
    inp = W.poison_unused(W.to_fp8_cache(W.make_decode(SMALL_LENS, 8, 2, 128, seed=840,
                                                       extra_pages=3)))
    check_all_rows(inp, 2, f"fp8 poisoned {kernel}", kernel)


@pytest.mark.parametrize("kernel", KERNELS)
def test_subnormal_heavy_cache(kernel):
    """Scales 1024x too large: many codes land in the E4M3 subnormal range."""
    inp = W.to_fp8_cache(W.make_decode([500, 2000], 8, 2, 128, seed=850), amax=4.0 * 1024)
    codes = inp.k_pages_bits & 0x7F
    assert np.mean((codes >> 3) == 0) > 0.05
    check_all_rows(inp, 0, f"fp8 subnormal-heavy {kernel}", kernel)


@pytest.mark.parametrize("kernel", KERNELS)
def test_every_code_decodes_exactly(kernel):
    """One cached token per request: O is that token's V row and LSE its score,
    so every E4M3 code (NaN codes excepted) is checked on its own, through
    both the V and the K path.  (On tensor cores P = 1 is exact in E4M3 and
    the one-hot query splits exactly, so this stays exact there too.)"""
    import exact_attention_148_b200 as fa
    B, Hq, Hkv, d = 32, 8, 1, 128
    base = W.make_decode([1] * B, Hq, Hkv, d, seed=860)
    codes = np.arange(256, dtype=np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    kp = np.zeros(base.k_pages_bits.shape, dtype=np.uint8)
    vp = np.zeros(base.v_pages_bits.shape, dtype=np.uint8)
    q = np.zeros((B, Hq, d), dtype=np.float32)
    for b in range(B):
        phys = int(base.block_table[b, 0])
        vp[phys, 0, 0, :] = codes[(b * d + np.arange(d)) % 256]
        for h in range(Hq):
            c = (b * Hq + h) % d
            kp[phys, 0, 0, c] = codes[b * Hq + h]
            q[b, h, c] = 1.0
    inp = W.DecodeInputs("every_code", W.f32_to_bf16_bits(q), kp, vp, base.block_table,
                         base.cache_seqlens, 1.0, extra={"k_scale": 1.0 / 64, "v_scale": 1.0})
    out, lse = run_fp8(inp, kernel=kernel)
    assert fa.device_status(clear=True) == 0
    want_v = oracle.e4m3_to_f64(vp[base.block_table[:, 0], 0, 0, :])        # [B, d]
    got = bf16_to_f64(out)                                                   # [B, Hq, d]
    for h in range(Hq):
        assert np.array_equal(got[:, h, :], want_v), "V codes decode exactly"
    want_s = np.array([[oracle.e4m3_to_f64(codes[b * Hq + h:b * Hq + h + 1])[0] / 64
                        for h in range(Hq)] for b in range(B)])
    np.testing.assert_allclose(lse.cpu().numpy(), want_s, rtol=2e-6, atol=2e-6)


@pytest.mark.parametrize("kernel", KERNELS)
def test_full_size_sampled_rows(kernel):
    inp = W.paged_decode_batch_fp8()
    out, lse = run_fp8(inp, kernel=kernel)
    g = np.random.default_rng(11)
    rows = [(int(b), int(h)) for b, h in zip(g.integers(0, inp.batch, 48),
                                             g.integers(0, inp.num_q_heads, 48))]
    o_ref, l_ref = oracle_rows(inp, rows)
    bi = np.array([r[0] for r in rows])
    hi = np.array([r[1] for r in rows])
    compare(out.float().cpu().numpy()[bi, hi].astype(np.float64), lse.cpu().numpy()[bi, hi],
            o_ref, l_ref, "fp8 full size")


@pytest.mark.parametrize("kernel", ["tensor_cores", "cuda_cores"])
@pytest.mark.parametrize("num_splits", [0, 1, 5])
def test_score_jumps_between_key_blocks_fp8(kernel, num_splits):
    """The bf16 decode's score-jump case on an E4M3 cache; K gets its own
    scale so the large keys do not saturate."""
    base = jumping_keys_decode(W.make_decode([1000, 129, 2500, 64, 700], 8, 2, 128, seed=751), JUMP_FACTORS)
    inp = W.to_fp8_cache(base)
    kf = W.bf16_bits_to_f32(base.k_pages_bits)
    k_scale = float(np.abs(kf).max()) / W.E4M3_MAX
    inp.k_pages_bits = W.quantize_e4m3(kf, k_scale)
    inp.extra = dict(inp.extra, k_scale=k_scale)
    check_all_rows(inp, num_splits, f"fp8 decode score jumps {kernel} splits={num_splits}", kernel=kernel)
