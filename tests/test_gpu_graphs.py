"""Every run entry point can be captured into a CUDA graph (no host
synchronisation or allocation inside the calls once the plan exists): the
graph replays give the eager results bit for bit, also after the inputs are
refreshed in place."""
import numpy as np
import pytest

import workloads as W
from tests.gpu_util import chunked_device_inputs, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


def _capture(fn):
    import torch
    fn()                                   # eager warm-up (kernel attributes, tensor-map encoder)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.synchronize()
    return g


def test_prefill_and_decode_in_one_graph():
    import torch
    import exact_attention_148_b200 as fa
    pre = W.make_prefill([300, 1000, 77], 8, 2, 128, causal=True, seed=2000)
    q, k, v = (to_dev_bf16(x) for x in (pre.q_bits, pre.k_bits, pre.v_bits))
    cu = to_dev_i32(pre.cu_seqlens)
    o1 = torch.empty_like(q)
    l1 = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    dec = W.make_decode([70, 5000, 129, 2048], 8, 2, 128, seed=2001)
    dq, dk, dv = (to_dev_bf16(x) for x in (dec.q_bits, dec.k_pages_bits, dec.v_pages_bits))
    bt, lens = to_dev_i32(dec.block_table), to_dev_i32(dec.cache_seqlens)
    plans = [fa.decode_plan(dec.cache_seqlens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                            max_pages_per_seq=dec.block_table.shape[1], num_splits=3, kernel=kern)
             for kern in ("tensor_cores", "cuda_cores")]
    ws = [torch.empty(max(p.workspace_bytes, 256), dtype=torch.uint8, device=q.device) for p in plans]
    outs = [(torch.empty_like(dq), torch.empty(dq.shape[:2], dtype=torch.float32, device=q.device))
            for _ in plans]

    def step():
        fa.prefill(q, k, v, cu, causal=True, scale=pre.scale, out=o1, lse=l1,
                   cu_seqlens_host=pre.cu_seqlens, stream=torch.cuda.current_stream())
        for p, w, (o, l) in zip(plans, ws, outs):
            fa.decode_paged(dq, dk, dv, bt, lens, p, scale=dec.scale, out=o, lse=l, workspace=w,
                            stream=torch.cuda.current_stream())

    step()
    torch.cuda.synchronize()
    want = [o1.clone(), l1.clone()] + [t.clone() for pair in outs for t in pair]
    for t in [o1, l1] + [t for pair in outs for t in pair]:
        t.zero_()
    g = _capture(step)
    for t in [o1, l1] + [t for pair in outs for t in pair]:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    got = [o1, l1] + [t for pair in outs for t in pair]
    assert all(torch.equal(a, b) for a, b in zip(want, got))
    # new query values, same shapes: the replay follows the inputs
    dq.copy_(torch.flip(dq, dims=[0]))
    g.replay()
    torch.cuda.synchronize()
    for p, w, (o, l) in zip(plans, ws, outs):
        o2, l2 = fa.decode_paged(dq, dk, dv, bt, lens, p, scale=dec.scale, workspace=w)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(l, l2)
    assert fa.device_status(clear=True) == 0


def test_append_chunked_prefill_and_cascade_in_graphs():
    import torch
    import exact_attention_148_b200 as fa
    inp = W.tiny_chunked_prefill()
    dev = chunked_device_inputs(inp)
    out = torch.empty_like(dev["q"])
    lse = torch.empty(dev["q"].shape[:2], dtype=torch.float32, device=out.device)

    def chunk_step():
        fa.append_kv(dev["k_new"], dev["v_new"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"],
                     stream=torch.cuda.current_stream())
        fa.prefill_paged(dev["q"], dev["cu"], dev["k"], dev["v"], dev["bt"], dev["lens"], out=out, lse=lse,
                         scale=inp.scale, cu_seqlens_q_host=inp.cu_seqlens_q,
                         cache_seqlens_host=inp.cache_seqlens, stream=torch.cuda.current_stream())

    chunk_step()
    torch.cuda.synchronize()
    want = (out.clone(), lse.clone())
    g = _capture(chunk_step)
    out.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, want[0]) and torch.equal(lse, want[1])

    cas = W.make_cascade(1000, [0, 70, 300, 2000], 8, 2, 128, seed=2002)
    cq = to_dev_bf16(cas.q_bits)
    ck, cv = to_dev_bf16(cas.k_pages_bits), to_dev_bf16(cas.v_pages_bits)
    pre, cbt, clen = (to_dev_i32(x) for x in (cas.prefix_block_table, cas.block_table, cas.suffix_lens))
    plan = fa.decode_plan(cas.suffix_lens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                          max_pages_per_seq=cas.block_table.shape[1])
    cws = torch.empty(fa.cascade_workspace_bytes(plan, cas.prefix_len), dtype=torch.uint8, device=cq.device)
    co = torch.empty_like(cq)
    cl = torch.empty(cq.shape[:2], dtype=torch.float32, device=cq.device)

    def cascade_step():
        fa.cascade_decode(cq, ck, cv, pre, cas.prefix_len, cbt, clen, plan, scale=cas.scale, out=co,
                          lse=cl, workspace=cws, stream=torch.cuda.current_stream())

    cascade_step()
    torch.cuda.synchronize()
    want = (co.clone(), cl.clone())
    g2 = _capture(cascade_step)
    co.zero_()
    cl.zero_()
    g2.replay()
    torch.cuda.synchronize()
    assert torch.equal(co, want[0]) and torch.equal(cl, want[1])
    assert fa.device_status(clear=True) == 0


def test_prefill_fp8_in_a_graph():
    import torch
    import exact_attention_148_b200 as fa
    inp = W.to_fp8_prefill(W.make_prefill([129, 700], 4, 2, 128, causal=True, seed=2002))
    q, k, v = (torch.from_numpy(x).cuda() for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    cu = to_dev_i32(inp.cu_seqlens)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    l = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)

    def step():
        fa.prefill_fp8(q, k, v, cu, q_scale=inp.q_scale, k_scale=inp.k_scale, v_scale=inp.v_scale,
                       causal=True, scale=inp.scale, out=o, lse=l, cu_seqlens_host=inp.cu_seqlens,
                       stream=torch.cuda.current_stream())

    step()
    torch.cuda.synchronize()
    want = (o.clone(), l.clone())
    g = _capture(step)
    o.zero_()
    l.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, want[0]) and torch.equal(l, want[1])
    k.copy_(torch.flip(k, dims=[0]))        # new keys in place: the replay follows them
    g.replay()
    o2, l2 = fa.prefill_fp8(q, k, v, cu, q_scale=inp.q_scale, k_scale=inp.k_scale,
                            v_scale=inp.v_scale, causal=True, scale=inp.scale,
                            cu_seqlens_host=inp.cu_seqlens)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(l, l2)
    assert fa.device_status(clear=True) == 0
