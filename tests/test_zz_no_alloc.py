"""fa_decode_paged_static: paged decode for callers that cannot allocate.

Some callers are not allowed to call cudaMalloc — code hosted inside a
framework that owns all device memory through its own allocator, serving loops
that must not pay for an allocation (cudaMalloc/cudaFree can synchronise the
device), processes with a device-memory budget fixed at start-up.  For them
the library offers a decode entry point with no workspace argument: the split
partials go to one static 16 MiB device array inside the library.

These tests call that entry point through the C ABI on two calls in a row with
different inputs, so whatever the first call left in the shared array cannot
leak into the second.  The static and workspace entry points run the same
kernels with the same plan, so their results must agree bit for bit; the
static result is also checked against the fp64 oracle.  This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import bf16_to_f64, compare, decode_device_inputs

pytestmark = pytest.mark.gpu


def _static_call(lib, dev, inp, plan, out, lse):
    import torch
    import exact_attention_148_b200 as fa
    ps, ts, hs = fa.page_strides(dev["k"], inp.layout)
    return lib.fa_decode_paged_static(
        ctypes.c_void_p(dev["q"].data_ptr()), ctypes.c_void_p(dev["k"].data_ptr()),
        ctypes.c_void_p(dev["v"].data_ptr()), dev["k"].shape[0], ps, ts, hs,
        ctypes.c_void_p(dev["bt"].data_ptr()), ctypes.c_void_p(dev["lens"].data_ptr()), plan.handle,
        float("nan"), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("kernel", ["auto", "cuda_cores"])
def test_static_scratch_decode_matches_workspace_decode(kernel):
    import torch
    import exact_attention_148_b200 as fa
    lib = fa.library()
    cases = [([70, 1500, 4097, 129], 8, 2, 11), ([5000, 64, 3000], 4, 4, 12)]
    for call, (lens, hq, hkv, seed) in enumerate(cases):
        inp = W.make_decode(lens, hq, hkv, 128, seed=seed)
        dev = decode_device_inputs(inp)
        plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                              max_pages_per_seq=inp.block_table.shape[1], num_splits=4,
                              kernel=kernel)
        assert 0 < plan.workspace_bytes <= fa.STATIC_SCRATCH_BYTES
        ref_out, ref_lse = fa.decode_paged(dev["q"], dev["k"], dev["v"], dev["bt"], dev["lens"], plan)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        status = _static_call(lib, dev, inp, plan, out, lse)
        assert status == fa.FA_OK, fa.strerror(status)
        torch.cuda.synchronize()
        what = f"static-scratch decode ({kernel}), call {call + 1}"
        assert torch.equal(out, ref_out), f"{what}: O differs from the workspace entry point"
        assert torch.equal(lse, ref_lse), f"{what}: LSE differs from the workspace entry point"
        o_ref, l_ref = oracle.paged_decode_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits,
                                               inp.block_table, inp.cache_seqlens, inp.scale,
                                               inp.page_size, inp.layout, to_f64=W.as_f64)
        compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, what + " vs oracle")
        assert fa.device_status(clear=True) == 0


def test_static_scratch_rejects_plans_larger_than_the_array():
    import exact_attention_148_b200 as fa
    lib = fa.library()
    lens = np.full(64, 32768, dtype=np.int32)
    plan = fa.decode_plan(lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                          max_pages_per_seq=512, num_splits=64)
    assert plan.workspace_bytes > fa.STATIC_SCRATCH_BYTES
    A = ctypes.c_void_p(0x10000)   # never touched: the size check comes first
    status = lib.fa_decode_paged_static(A, A, A, 100, 64 * 8 * 128, 8 * 128, 128, A, A, plan.handle,
                                        float("nan"), A, None, None)
    assert status == fa.FA_ERR_WORKSPACE


def test_static_scratch_rejects_an_e4m3_plan_before_any_launch():
    """The static entry point reads a bf16 cache; a plan made for an E4M3 cache
    is refused with FA_ERR_PLAN_MISMATCH and nothing is written."""
    import torch
    import exact_attention_148_b200 as fa
    lib = fa.library()
    inp = W.make_decode([300, 900], 8, 2, 128, seed=13)
    dev = decode_device_inputs(inp)
    plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                          max_pages_per_seq=inp.block_table.shape[1], num_splits=2, kv_dtype="e4m3")
    assert plan.workspace_bytes <= fa.STATIC_SCRATCH_BYTES
    out = torch.full((inp.batch, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((inp.batch, 8), 7.0, dtype=torch.float32, device="cuda")
    status = _static_call(lib, dev, inp, plan, out, lse)
    assert status == fa.FA_ERR_PLAN_MISMATCH, fa.strerror(status)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0) and torch.all(lse == 7.0)
    assert fa.device_status(clear=True) == 0
