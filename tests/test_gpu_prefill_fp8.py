"""GPU parity of fa_prefill_fp8 (E4M3 Q, K and V) against the fp64 oracle run
on the dequantised tensors."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import JUMP_FACTORS, bf16_to_f64, compare, jumping_keys, to_dev_i32

pytestmark = pytest.mark.gpu


def _dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def run_fp8(inp: W.Fp8PrefillInputs, **kw):
    import exact_attention_148_b200 as fa
    q, k, v = (_dev_u8(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    return fa.prefill_fp8(q, k, v, to_dev_i32(inp.cu_seqlens), q_scale=inp.q_scale,
                          k_scale=inp.k_scale, v_scale=inp.v_scale, causal=inp.causal,
                          scale=inp.scale, cu_seqlens_host=inp.cu_seqlens, **kw)


def dequantised(inp):
    return (oracle.dequantize_e4m3(inp.q_bits, inp.q_scale),
            oracle.dequantize_e4m3(inp.k_bits, inp.k_scale),
            oracle.dequantize_e4m3(inp.v_bits, inp.v_scale))


def check_full(inp, what):
    import exact_attention_148_b200 as fa
    assert fa.device_status(clear=True) == 0
    out, lse = run_fp8(inp)
    q, k, v = dequantised(inp)
    o_ref, l_ref = oracle.attention_ref(q, k, v, inp.cu_seqlens, inp.causal, inp.scale)
    errs = compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, what)
    assert fa.device_status(clear=True) == 0
    return errs


RAGGED = [1, 127, 128, 129, 300, 513]


def test_tiny_causal_prefill_fp8():
    check_full(W.to_fp8_prefill(W.make_prefill([128], 2, 2, 128, seed=40)), "tiny fp8")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 1), (8, 2), (3, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_small_varlen_fp8(hq, hkv, causal):
    inp = W.to_fp8_prefill(W.make_prefill(RAGGED, hq, hkv, 128, causal=causal, seed=200 + hq + hkv))
    check_full(inp, f"fp8 varlen hq={hq} hkv={hkv} causal={causal}")


def test_multi_tile_long_sequence_fp8():
    inp = W.to_fp8_prefill(W.make_prefill([2048 + 77], 4, 2, 128, causal=True, seed=41))
    check_full(inp, "fp8 2125-token causal GQA")


def test_single_token_and_explicit_scale_fp8():
    check_full(W.to_fp8_prefill(W.make_prefill([1], 2, 2, 128, scale=0.3, seed=42)), "fp8 single token")
    check_full(W.to_fp8_prefill(W.make_prefill([700, 1], 2, 2, 128, causal=False, scale=0.05, seed=43)),
               "fp8 non-causal explicit scale")


def test_saturated_codes_and_unequal_scales():
    """amax 1.5: a seventh of the N(0,1) draws clip to +-448; the three tensors
    then get different scales (V's output scale must be applied, Q's and K's
    folded into the score scale)."""
    base = W.make_prefill([300, 129], 4, 2, 128, causal=True, seed=44)
    inp = W.to_fp8_prefill(base, amax=1.5)
    assert (inp.v_bits & 0x7F == 0x7E).mean() > 0.05          # many +-448 codes
    inp.q_scale, inp.k_scale, inp.v_scale = inp.q_scale * 2.0, inp.k_scale * 0.5, inp.v_scale * 3.0
    check_full(inp, "fp8 saturated, unequal scales")


def test_score_jumps_between_key_tiles_fp8():
    """Key tiles scaled by up to 200: with f16 P the overflow guard (2^15)
    re-references most jumping tiles at once; K gets its own scale so the
    large keys do not saturate."""
    base = jumping_keys(W.make_prefill([700, 300, 1000], 4, 2, 128, causal=True, seed=49), JUMP_FACTORS)
    inp = W.to_fp8_prefill(base)
    kf = W.bf16_bits_to_f32(base.k_bits)
    inp.k_scale = float(np.abs(kf).max()) / W.E4M3_MAX
    inp.k_bits = W.quantize_e4m3(kf, inp.k_scale)
    check_full(inp, "fp8 score jumps")


def test_matches_bf16_kernel_on_exact_inputs():
    """E4M3 codes are exact in bf16: the bf16 kernel on the dequantised
    tensors (power-of-two scales) and the FP8 kernel agree to the output rounding."""
    import torch
    import exact_attention_148_b200 as fa
    inp = W.to_fp8_prefill(W.make_prefill([513, 128], 4, 2, 128, causal=True, seed=45))
    inp.q_scale = inp.k_scale = inp.v_scale = 2.0 ** -7   # code * 2^-7: exact in bf16
    o8, l8 = run_fp8(inp)
    q, k, v = (torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda() for x in dequantised(inp))
    o16, l16 = fa.prefill(q, k, v, to_dev_i32(inp.cu_seqlens), causal=True, scale=inp.scale,
                          cu_seqlens_host=inp.cu_seqlens)
    o8, o16 = bf16_to_f64(o8), bf16_to_f64(o16)
    scale = np.abs(o16).max()
    assert np.abs(o8 - o16).max() <= 2e-2 * max(scale, 1.0)
    assert np.abs(l8.cpu().numpy() - l16.cpu().numpy()).max() <= 1e-3 * max(1.0, float(l16.abs().max()))


def test_varlen_config_sampled_fp8():
    """The full FP8 varlen workload (8 sequences in [512, 4096], 32 heads),
    checked on sampled rows."""
    from tests.test_gpu_prefill import sample_rows
    inp = W.varlen_causal_prefill_fp8()
    out, lse = run_fp8(inp)
    rows = sample_rows(inp, 768, 3)
    q, k, v = dequantised(inp)
    o_ref, l_ref = oracle.attention_rows_ref(q, k, v, inp.cu_seqlens, inp.causal, inp.scale, rows)
    it = np.array([r[0] for r in rows])
    ih = np.array([r[1] for r in rows])
    compare(out.float().cpu().numpy()[it, ih].astype(np.float64), lse.cpu().numpy()[it, ih], o_ref, l_ref,
            "fp8 varlen causal prefill (8 seqs, 32 heads)")
