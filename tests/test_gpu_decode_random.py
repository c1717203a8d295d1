"""GPU parity of the paged decode on seeded random configurations.

The other decode tests vary one parameter grid at a time.  Here every case
draws all of them at once: head size, kv heads and group size, bf16 or E4M3
cache, NHD or HND pages, split kernel, query tokens per request, split count,
spare pool pages, an explicit score scale, and lengths from 0 (a request with
no keys) through page multiples, their neighbours and a few thousand.  Each
case compares every output row with the fp64 oracle."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import bf16_to_f64, compare, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu

NUM_CASES = 32


def random_config(seed):
    """One valid configuration (the library supports every combination drawn)."""
    rng = np.random.default_rng(7000 + seed)
    d = 128 if rng.random() < 0.7 else 64
    hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 3, 4, 8, 16]))
    fp8 = bool(rng.random() < 0.45)
    layout = str(rng.choice(["NHD", "HND"]))
    kernel = str(rng.choice(["auto", "tensor_cores", "cuda_cores"])) if d == 128 else "cuda_cores"
    q_len = 1
    if d == 128 and kernel != "cuda_cores" and G <= 8 and rng.random() < 0.35:
        q_len = int(rng.choice([2, 3, 4]))
        q_len = max(1, min(q_len, 16 // G))
    B = int(rng.integers(1, 7))
    lens = rng.integers(0, 2600, size=B)
    for b in range(B):
        r = rng.random()
        if r < 0.25:
            lens[b] = 64 * int(rng.integers(1, 40)) + int(rng.integers(-1, 2))
        elif r < 0.35:
            lens[b] = 0
    if q_len > 1:
        lens = np.maximum(lens, q_len)
    splits = int(rng.choice([0, 0, 1, 2, 3, 5, 8]))
    scale = None if rng.random() < 0.6 else float(rng.uniform(0.03, 0.2))
    return dict(d=d, hkv=hkv, G=G, fp8=fp8, layout=layout, kernel=kernel, q_len=q_len,
                lens=lens.astype(np.int64), splits=splits, scale=scale,
                extra_pages=int(rng.integers(0, 3)), seed=7100 + seed)


def make_inputs(cfg):
    inp = W.make_decode(cfg["lens"], cfg["G"] * cfg["hkv"], cfg["hkv"], cfg["d"], seed=cfg["seed"],
                        layout=cfg["layout"], scale=cfg["scale"], extra_pages=cfg["extra_pages"],
                        q_len=cfg["q_len"], name="random_decode")
    return W.to_fp8_cache(inp) if cfg["fp8"] else inp


def plan_for(inp, cfg, num_sms=None):
    import exact_attention_148_b200 as fa
    return fa.decode_plan(inp.cache_seqlens, num_q_heads=inp.num_q_heads, num_kv_heads=inp.num_kv_heads,
                          head_dim=inp.head_dim, page_size=inp.page_size,
                          max_pages_per_seq=inp.block_table.shape[1], num_sms=num_sms,
                          num_splits=cfg["splits"], kv_dtype="e4m3" if cfg["fp8"] else "bf16",
                          kernel=cfg["kernel"], q_len=cfg["q_len"])


def oracle_all(inp):
    conv = {}
    if inp.kv_elem_bytes == 1:
        ks, vs = inp.extra["k_scale"], inp.extra["v_scale"]
        conv = dict(k_to_f64=lambda a: oracle.dequantize_e4m3(a, ks),
                    v_to_f64=lambda a: oracle.dequantize_e4m3(a, vs))
    if inp.q_len == 1:
        return oracle.paged_decode_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits, inp.block_table,
                                       inp.cache_seqlens, inp.scale, inp.page_size, inp.layout,
                                       to_f64=W.as_f64, **conv)
    # several query tokens: the chunked-prefill reading (the tokens are the
    # cache's last q_len entries, causally masked among themselves)
    B, QL, Hq, d = inp.q_bits.shape
    cu = np.arange(B + 1) * QL
    return oracle.paged_prefill_ref(inp.q_bits.reshape(B * QL, Hq, d), cu, inp.k_pages_bits,
                                    inp.v_pages_bits, inp.block_table, inp.cache_seqlens, True,
                                    inp.scale, inp.page_size, inp.layout, to_f64=W.as_f64, **conv)


@pytest.mark.parametrize("seed", range(NUM_CASES))
def test_random_configuration(seed):
    import torch

    import exact_attention_148_b200 as fa
    cfg = random_config(seed)
    inp = make_inputs(cfg)
    plan = plan_for(inp, cfg)
    dev_u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()
    q = to_dev_bf16(inp.q_bits)
    bt, lens = to_dev_i32(inp.block_table), to_dev_i32(inp.cache_seqlens)
    assert fa.device_status(clear=True) == 0
    if cfg["fp8"]:
        out, lse = fa.decode_paged_fp8(q, dev_u8(inp.k_pages_bits), dev_u8(inp.v_pages_bits), bt, lens,
                                       plan, k_scale=inp.extra["k_scale"], v_scale=inp.extra["v_scale"],
                                       layout=inp.layout, scale=inp.scale)
    else:
        out, lse = fa.decode_paged(q, to_dev_bf16(inp.k_pages_bits), to_dev_bf16(inp.v_pages_bits), bt,
                                   lens, plan, layout=inp.layout, scale=inp.scale)
    assert fa.device_status(clear=True) == 0
    o_ref, l_ref = oracle_all(inp)
    what = (f"seed {seed}: d={cfg['d']} Hkv={cfg['hkv']} G={cfg['G']} {'e4m3' if cfg['fp8'] else 'bf16'} "
            f"{cfg['layout']} {cfg['kernel']} q_len={cfg['q_len']} splits={cfg['splits']} "
            f"lens={cfg['lens'].tolist()} -> {plan.info.max_splits} splits, "
            f"{'tensor' if plan.info.tensor_cores else 'CUDA'} cores")
    compare(bf16_to_f64(out).reshape(-1, inp.head_dim), lse.cpu().numpy().reshape(-1),
            np.asarray(o_ref).reshape(-1, inp.head_dim), np.asarray(l_ref).reshape(-1), what)
