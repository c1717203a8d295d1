"""GPU parity of the prefill entry points on seeded random configurations.

The other prefill tests vary one parameter grid at a time.  Here every case
draws all of them at once: entry point (packed bf16, packed E4M3, or KV append
plus chunked prefill over the paged cache), head size, kv heads and group
size, causal or full attention, an explicit score scale, the schedule (grid
or persistent), page layout and spare pool pages, and sequence, prefix and
chunk lengths that fall on, next to and between 128-key tiles and 64-token
pages.  Each case compares every output row with the fp64 oracle (and, for
the chunked case, the page pool after the append bit for bit)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import (bf16_to_f64, chunked_on_gpu, compare, oracle_pool_after_append,
                            prefill_on_gpu, to_dev_i32)

pytestmark = pytest.mark.gpu

NUM_CASES = 30


def _length(rng, hi):
    r = rng.random()
    if r < 0.3:
        return int(max(1, 128 * int(rng.integers(1, max(2, hi // 128))) + int(rng.integers(-1, 2))))
    if r < 0.4:
        return 1
    return int(rng.integers(1, hi + 1))


def random_config(seed):
    rng = np.random.default_rng(9000 + seed)
    kind = str(rng.choice(["packed", "packed", "fp8", "chunked", "chunked"]))
    d = 128 if kind == "fp8" or rng.random() < 0.6 else 64
    hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 3, 4, 8]))
    B = int(rng.integers(1, 6))
    cfg = dict(kind=kind, d=d, hkv=hkv, G=G, causal=bool(rng.random() < 0.7),
               scale=None if rng.random() < 0.6 else float(rng.uniform(0.03, 0.2)),
               schedule=str(rng.choice(["grid", "persistent"])), seed=9100 + seed)
    if kind == "chunked":
        cfg.update(prefix=[0 if rng.random() < 0.2 else _length(rng, 1500) for _ in range(B)],
                   chunk=[_length(rng, 400) for _ in range(B)],
                   layout=str(rng.choice(["NHD", "HND"])), extra_pages=int(rng.integers(0, 3)))
    else:
        cfg.update(seqlens=[_length(rng, 700) for _ in range(B)])
    return cfg


def _describe(seed, cfg):
    lens = cfg.get("seqlens") or list(zip(cfg["prefix"], cfg["chunk"]))
    return (f"seed {seed}: {cfg['kind']} d={cfg['d']} Hkv={cfg['hkv']} G={cfg['G']} "
            f"causal={cfg['causal']} scale={cfg['scale']} {cfg['schedule']} lens={lens}")


@pytest.mark.parametrize("seed", range(NUM_CASES))
def test_random_configuration(seed, monkeypatch):
    import torch

    import exact_attention_148_b200 as fa
    cfg = random_config(seed)
    what = _describe(seed, cfg)
    monkeypatch.setenv("FA_PREFILL_SCHEDULE", cfg["schedule"])
    hq = cfg["G"] * cfg["hkv"]
    assert fa.device_status(clear=True) == 0
    if cfg["kind"] == "chunked":
        inp = W.make_chunked_prefill(cfg["prefix"], cfg["chunk"], hq, cfg["hkv"], cfg["d"], seed=cfg["seed"],
                                     causal=cfg["causal"], layout=cfg["layout"], scale=cfg["scale"],
                                     extra_pages=cfg["extra_pages"])
        out, lse, dev = chunked_on_gpu(inp)
        kp, vp = oracle_pool_after_append(inp)
        bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(bits(dev["k"]), kp), f"{what}: K pool after append"
        assert np.array_equal(bits(dev["v"]), vp), f"{what}: V pool after append"
        o_ref, l_ref = oracle.paged_prefill_ref(inp.q_bits, inp.cu_seqlens_q, kp, vp, inp.block_table,
                                                inp.cache_seqlens, inp.causal, inp.scale, inp.page_size,
                                                inp.layout, to_f64=W.as_f64)
    else:
        inp = W.make_prefill(cfg["seqlens"], hq, cfg["hkv"], cfg["d"], causal=cfg["causal"],
                             scale=cfg["scale"], seed=cfg["seed"])
        if cfg["kind"] == "fp8":
            f8 = W.to_fp8_prefill(inp)
            u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()
            out, lse = fa.prefill_fp8(u8(f8.q_bits), u8(f8.k_bits), u8(f8.v_bits), to_dev_i32(f8.cu_seqlens),
                                      q_scale=f8.q_scale, k_scale=f8.k_scale, v_scale=f8.v_scale,
                                      causal=f8.causal, scale=f8.scale, cu_seqlens_host=f8.cu_seqlens)
            q, k, v = (oracle.dequantize_e4m3(x, s) for x, s in ((f8.q_bits, f8.q_scale),
                                                                  (f8.k_bits, f8.k_scale),
                                                                  (f8.v_bits, f8.v_scale)))
            o_ref, l_ref = oracle.attention_ref(q, k, v, f8.cu_seqlens, f8.causal, f8.scale)
        else:
            out, lse = prefill_on_gpu(inp)
            o_ref, l_ref = oracle.attention_ref(W.as_f64(inp.q_bits), W.as_f64(inp.k_bits),
                                                W.as_f64(inp.v_bits), inp.cu_seqlens, inp.causal, inp.scale)
    assert fa.prefill_last_schedule() == cfg["schedule"], what
    assert fa.device_status(clear=True) == 0, what
    compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, what)
