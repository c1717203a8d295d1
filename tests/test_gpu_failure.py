"""Failure detection on the GPU without a GPU fault: a bounded wait is made to
run out (a barrier nothing arrives at), the kernel records FA_ERR_TIMEOUT in
the device status word and returns, and the context stays usable."""
import pytest

import workloads as W
from tests.gpu_util import bf16_to_f64, compare, decode_on_gpu
import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import exact_attention_148_b200 as fa
    fa.device_status(clear=True)
    assert fa.selftest_wait_timeout(20000) == fa.FA_ERR_TIMEOUT
    assert fa.device_status(clear=True) == 0
    # the same process keeps working: a normal decode still matches the oracle
    inp = W.make_decode([300, 77], 4, 2, 128, seed=1300)
    out, lse, _ = decode_on_gpu(inp, 2)
    o_ref, l_ref = oracle.paged_decode_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits,
                                           inp.block_table, inp.cache_seqlens, inp.scale, 64,
                                           inp.layout, to_f64=W.as_f64)
    compare(bf16_to_f64(out), lse.cpu().numpy(), o_ref, l_ref, "decode after timeout self-test")
    assert fa.device_status(clear=True) == 0
