"""The bounds-checked build (libexact_attention_debug.so, compiled with
FA_DEBUG): every global index the kernels compute is checked against its
buffer before the access, a failed check recorded as FA_ERR_DEBUG_INDEX.

It stands in for a race and bounds sanitizer on this GPU pool.  Two checks:
(1) its self-test kernel refuses a planted out-of-range index (kept inside the
buffer, so nothing outside it can be touched) and records the code; (2) every
entry point, on small cases that reach every kernel, leaves the status word
clean and gives bit for bit the release build's results.
"""
import numpy as np
import pytest

import workloads as W
from tests.gpu_util import chunked_on_gpu, decode_on_gpu, prefill_on_gpu, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_build():
    import exact_attention_148_b200 as fa
    from exact_attention_148_b200 import _build
    _build.build(debug=True)
    fa.select_library("debug")
    yield fa
    fa.select_library("release")


def test_selftest_refuses_the_planted_index(debug_build):
    import torch
    fa = debug_build
    buf = torch.zeros(16, dtype=torch.int32, device="cuda")
    fa.device_status(clear=True)
    assert fa.debug_selftest_index(buf) == fa.FA_OK
    torch.cuda.synchronize()
    got = buf.cpu().numpy()
    assert got[0] == 1 and not got[1:].any(), got
    assert fa.device_status(clear=True) == fa.FA_ERR_DEBUG_INDEX


def test_release_build_has_no_selftest_kernel():
    import torch
    import exact_attention_148_b200 as fa
    fa.select_library("release")
    buf = torch.zeros(16, dtype=torch.int32, device="cuda")
    assert fa.debug_selftest_index(buf) == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert not buf.cpu().numpy().any()


def every_entry_point(monkeypatch):
    """Small cases through every entry point and kernel; returns all outputs."""
    import torch
    import exact_attention_148_b200 as fa
    from tests.test_gpu_cascade import run as cascade_run
    from tests.test_gpu_decode_fp8 import run_fp8 as fp8_decode
    from tests.test_gpu_decode_mtp import run as mtp_run
    from tests.test_gpu_prefill_fp8 import run_fp8 as fp8_prefill
    outs = []

    def keep(res, what):
        torch.cuda.synchronize()
        assert fa.device_status(clear=True) == 0, what
        outs.extend(t.clone() for t in res if t is not None)

    lens = [1, 127, 128, 129, 300, 513]
    for sched in ("persistent", "grid"):
        monkeypatch.setenv("FA_PREFILL_SCHEDULE", sched)
        for d, hq, hkv, causal in ((128, 8, 2, True), (64, 3, 1, False), (128, 4, 4, True)):
            keep(prefill_on_gpu(W.make_prefill(lens, hq, hkv, d, causal=causal, seed=700 + d + hq)),
                 f"prefill {sched} d={d}")
        keep(fp8_prefill(W.to_fp8_prefill(W.make_prefill(lens, 4, 2, 128, seed=710))), f"fp8 prefill {sched}")
        keep(chunked_on_gpu(W.tiny_chunked_prefill())[:2], f"append + chunked prefill {sched}")
        keep(chunked_on_gpu(W.poison_chunked(W.tiny_chunked_prefill(64, "HND")))[:2],
             f"chunked prefill, NaN page tails {sched}")
    monkeypatch.delenv("FA_PREFILL_SCHEDULE", raising=False)
    dec = W.make_decode([70, 1500, 129, 0, 4097], 8, 2, 128, seed=720, extra_pages=3)
    for kernel in ("tensor_cores", "cuda_cores"):
        for s in (0, 1, 5):
            keep(decode_on_gpu(dec, s, kernel=kernel)[:2], f"decode {kernel} splits={s}")
    keep(decode_on_gpu(W.make_decode([300, 65], 4, 4, 64, seed=721), 3)[:2], "decode d=64")
    keep(fp8_decode(W.to_fp8_cache(dec), 3), "fp8 decode")
    keep(mtp_run(W.make_decode([300, 1200, 64], 8, 2, 128, seed=722, q_len=2), 3), "multi-token decode")
    keep(cascade_run(W.make_cascade(777, [5, 300, 0, 129], 8, 2, 128, seed=723)), "cascade decode")
    g = torch.Generator(device="cuda").manual_seed(724)
    parts_o = torch.randn(3, 5, 4, 128, device="cuda", generator=g)
    parts_l = torch.randn(3, 5, 4, device="cuda", generator=g)
    parts_l[1, 2] = float("-inf")
    keep(fa.merge_states(parts_o, parts_l), "merge_states")
    return outs


def test_debug_build_matches_release_bit_for_bit(debug_build, monkeypatch):
    import torch
    fa = debug_build
    fa.select_library("release")
    fa.device_status(clear=True)
    release = every_entry_point(monkeypatch)
    fa.select_library("debug")
    fa.device_status(clear=True)
    debug = every_entry_point(monkeypatch)
    assert len(release) == len(debug)
    for i, (a, b) in enumerate(zip(release, debug)):
        assert torch.equal(a, b), f"output {i} differs between the release and bounds-checked builds"
