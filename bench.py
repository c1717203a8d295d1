#!/usr/bin/env python3
"""Benchmark of the exact-attention hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  1. causal varlen prefill (8 sequences, lengths U[512, 4096], 32 heads, d=128)
     through fa_prefill, then
  2. Flash-Decoding of a paged batch (64 requests, cache lengths U[1024, 32768],
     32 q / 8 kv heads, d=128, shuffled 64-token pages) through fa_decode_plan's
     plan and fa_decode_paged (split kernel + merge kernel).
The line's ``value`` is the prefill throughput in TFLOP/s (causal algorithmic
FLOPs); the decode half reports HBM GB/s under ``decode``.  At one GPU the
default run then times the other configurations alone, each under ``legs``
with its own time, roofline and clock record: the 32K GQA causal prefill, the
long split decode (4 x 131072, the planner's split count plus a sweep of fixed
counts) and the ragged split decode (1 x 131072 + 63 x 2048).  ``--workload``
selects a single configuration instead (one line for that configuration);
``chunked_prefill_batch`` times a chunked-prefill step (fa_append_kv of the
chunk's K/V into the paged cache, then fa_prefill_paged over the whole cache).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torch.distributed.run; every rank runs an independent
replica of the step (no collective on the data path; "replicas only").
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "causal prefill TFLOP/s and paged-decode HBM GB/s on 1 B200 vs roofline"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}

PREFILL_WORKLOADS = {"varlen_causal_prefill", "long_gqa_prefill", "tiny_causal_prefill",
                     "varlen_causal_prefill_fp8"}
DECODE_WORKLOADS = {"paged_decode_batch", "long_split_decode", "ragged_split_decode",
                    "paged_decode_batch16", "paged_decode_batch_fp8", "paged_decode_gqa8",
                    "paged_decode_gqa16", "speculative_decode_batch"}
CHUNKED_WORKLOADS = {"chunked_prefill_batch", "tiny_chunked_prefill"}
CASCADE_WORKLOADS = {"cascade_decode_batch"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- device inputs

def _dev_bf16(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def _dev_i32(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32))).to(device)


class PrefillCase:
    def __init__(self, inp: W.PrefillInputs, device):
        import torch
        self.inp = inp
        self.fp8 = isinstance(inp, W.Fp8PrefillInputs)
        if self.fp8:
            self.q, self.k, self.v = (torch.from_numpy(x).to(device) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
            self.h_q, self.h_k, self.h_v = (torch.from_numpy(x).pin_memory()
                                            for x in (inp.q_bits, inp.k_bits, inp.v_bits))
        else:
            self.q = _dev_bf16(inp.q_bits, device)
            self.k = _dev_bf16(inp.k_bits, device)
            self.v = _dev_bf16(inp.v_bits, device)
            # pinned host copies for the end-to-end leg
            self.h_q, self.h_k, self.h_v = (torch.from_numpy(x.view(np.int16)).pin_memory()
                                            for x in (inp.q_bits, inp.k_bits, inp.v_bits))
        self.cu = _dev_i32(inp.cu_seqlens, device)
        self.h_cu = torch.from_numpy(np.ascontiguousarray(inp.cu_seqlens, dtype=np.int32)).pin_memory()
        self.out = torch.empty(self.q.shape, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=device)
        self.flops = inp.causal_flops()
        # one launch per 2048 (sequence, kv head) groups
        self.launches = -(-len(inp.seqlens) * inp.num_kv_heads // 2048)
        self.h_out = torch.empty(self.q.shape, dtype=torch.int16).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def run(self):
        import exact_attention_148_b200 as fa
        i = self.inp
        if self.fp8:
            fa.prefill_fp8(self.q, self.k, self.v, self.cu, q_scale=i.q_scale, k_scale=i.k_scale,
                           v_scale=i.v_scale, causal=i.causal, scale=i.scale, out=self.out,
                           lse=self.lse, cu_seqlens_host=i.cu_seqlens)
        else:
            fa.prefill(self.q, self.k, self.v, self.cu, causal=i.causal, scale=i.scale,
                       out=self.out, lse=self.lse, cu_seqlens_host=i.cu_seqlens)
        # the schedule the library actually launched (it uses the grid form while
        # a stream is being captured, or when it has no counter left)
        self.schedule = fa.prefill_last_schedule()

    def run_e2e(self):
        """Host buffers in, host buffers out: H2D copies, the C-ABI call, D2H copies."""
        import torch
        for d, h in ((self.q, self.h_q), (self.k, self.h_k), (self.v, self.h_v)):
            (d if self.fp8 else d.view(torch.int16)).copy_(h, non_blocking=True)
        self.cu.copy_(self.h_cu, non_blocking=True)
        self.run()
        self.h_out.copy_(self.out.view(torch.int16), non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def e2e_fields(self):
        """(device attribute, pinned host attribute, copy as int16) of each
        step's inputs and outputs."""
        bits = not self.fp8
        return ([("q", "h_q", bits), ("k", "h_k", bits), ("v", "h_v", bits), ("cu", "h_cu", False)],
                [("out", "h_out", True), ("lse", "h_lse", False)])

    def h2d_bytes(self):
        eb = 1 if self.fp8 else 2
        return eb * (self.inp.q_bits.size + self.inp.k_bits.size + self.inp.v_bits.size) + \
            4 * self.inp.cu_seqlens.size

    def d2h_bytes(self):
        return 2 * self.inp.q_bits.size + 4 * self.lse.numel()

    def describe(self):
        i = self.inp
        return {"workload": i.name, "batch": int(len(i.seqlens)), "seqlens_total": int(i.seqlens.sum()),
                "num_q_heads": i.num_q_heads, "num_kv_heads": i.num_kv_heads,
                "head_dim": i.head_dim, "causal": bool(i.causal),
                "inputs": "e4m3 q/k/v, per-tensor scales" if self.fp8 else "bf16",
                "schedule": getattr(self, "schedule", None),
                "algorithmic_tflop": round(self.flops / 1e12, 4)}


class DecodeCase:
    def __init__(self, inp: W.DecodeInputs, device, num_splits=0, kernel="auto"):
        import torch
        import exact_attention_148_b200 as fa
        self.inp = inp
        self.fp8 = inp.kv_elem_bytes == 1
        self.q = _dev_bf16(inp.q_bits, device)
        if self.fp8:
            self.kp = torch.from_numpy(inp.k_pages_bits).to(device)
            self.vp = torch.from_numpy(inp.v_pages_bits).to(device)
        else:
            self.kp = _dev_bf16(inp.k_pages_bits, device)
            self.vp = _dev_bf16(inp.v_pages_bits, device)
        self.bt = _dev_i32(inp.block_table, device)
        self.lens = _dev_i32(inp.cache_seqlens, device)
        self._plan(num_splits, kernel)
        self.ws = torch.empty(max(self.plan.workspace_bytes, 256), dtype=torch.uint8, device=device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:-1], dtype=torch.float32, device=device)
        self.bytes = inp.algorithmic_bytes()
        self.launches = 1 + (1 if self.plan.info.max_splits > 1 else 0)
        self.h_q = torch.from_numpy(inp.q_bits.view(np.int16)).pin_memory()
        self.h_bt = torch.from_numpy(inp.block_table).pin_memory()
        self.h_lens = torch.from_numpy(inp.cache_seqlens).pin_memory()
        self.h_out = torch.empty(self.q.shape, dtype=torch.int16).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def _plan(self, num_splits, kernel):
        """Plan on the host; plan_first_ms is the first call (one-time set-up
        included), plan_ms the median of five more, as in a serving loop that
        plans every step."""
        import exact_attention_148_b200 as fa
        inp = self.inp
        times = []
        for _ in range(6):
            t0 = time.perf_counter()
            self.plan = fa.decode_plan(inp.cache_seqlens, num_q_heads=inp.num_q_heads,
                                       num_kv_heads=inp.num_kv_heads, head_dim=inp.head_dim,
                                       page_size=inp.page_size, max_pages_per_seq=inp.block_table.shape[1],
                                       num_splits=num_splits, kv_dtype="e4m3" if self.fp8 else "bf16",
                                       kernel=kernel, q_len=inp.q_len)
            times.append((time.perf_counter() - t0) * 1e3)
        self.plan_first_ms = times[0]
        self.plan_ms = float(np.median(times[1:]))

    def replan(self, num_splits=0, kernel="auto"):
        """A new plan (and workspace) over the same device-resident inputs."""
        import torch
        import exact_attention_148_b200 as fa
        self._plan(num_splits, kernel)
        self.ws = torch.empty(max(self.plan.workspace_bytes, 256), dtype=torch.uint8, device=self.q.device)
        self.launches = 1 + (1 if self.plan.info.max_splits > 1 else 0)

    def run(self):
        import exact_attention_148_b200 as fa
        if self.fp8:
            fa.decode_paged_fp8(self.q, self.kp, self.vp, self.bt, self.lens, self.plan,
                                k_scale=self.inp.extra["k_scale"], v_scale=self.inp.extra["v_scale"],
                                layout=self.inp.layout, scale=self.inp.scale, out=self.out,
                                lse=self.lse, workspace=self.ws)
            return
        fa.decode_paged(self.q, self.kp, self.vp, self.bt, self.lens, self.plan, layout=self.inp.layout,
                        scale=self.inp.scale, out=self.out, lse=self.lse, workspace=self.ws)

    def run_e2e(self):
        """A decode step's inputs are its query rows, block table and cache
        lengths; the paged KV cache is state the earlier steps wrote, resident
        in HBM across steps (as in serving), so it is not copied per step."""
        import torch
        self.q.view(torch.int16).copy_(self.h_q, non_blocking=True)
        self.bt.copy_(self.h_bt, non_blocking=True)
        self.lens.copy_(self.h_lens, non_blocking=True)
        self.run()
        self.h_out.copy_(self.out.view(torch.int16), non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def e2e_fields(self):
        return ([("q", "h_q", True), ("bt", "h_bt", False), ("lens", "h_lens", False)],
                [("out", "h_out", True), ("lse", "h_lse", False)])

    def h2d_bytes(self):
        i = self.inp
        return 2 * i.q_bits.size + 4 * (i.block_table.size + i.cache_seqlens.size)

    def d2h_bytes(self):
        return 2 * self.inp.q_bits.size + 4 * self.lse.numel()

    def describe(self):
        i = self.inp
        info = self.plan.info
        return {"workload": i.name, "batch": i.batch, "q_len": i.q_len,
                "cache_tokens_total": int(i.cache_seqlens.sum()),
                "num_q_heads": i.num_q_heads, "num_kv_heads": i.num_kv_heads, "head_dim": i.head_dim,
                "page_size": i.page_size, "layout": i.layout,
                "kv_dtype": "e4m3 (per-tensor scales)" if self.fp8 else "bf16",
                "chunk_tokens": info.chunk_tokens,
                "max_splits": info.max_splits, "work_items": info.num_work_items,
                "split_kernel": "tensor cores (tcgen05)" if info.tensor_cores else "CUDA cores",
                "plan_ms": round(self.plan_ms, 3), "plan_first_ms": round(self.plan_first_ms, 3),
                "algorithmic_gb": round(self.bytes / 1e9, 4)}


class ChunkedState:
    """Device buffers of one chunked-prefill step: the chunk's q / k / v, the
    paged cache (prefix resident across steps) and the outputs."""

    def __init__(self, inp: W.ChunkedPrefillInputs, device):
        import torch
        self.inp = inp
        self.q = _dev_bf16(inp.q_bits, device)
        self.k_new = _dev_bf16(inp.k_new_bits, device)
        self.v_new = _dev_bf16(inp.v_new_bits, device)
        self.cu = _dev_i32(inp.cu_seqlens_q, device)
        self.kp = _dev_bf16(inp.k_pages_bits, device)
        self.vp = _dev_bf16(inp.v_pages_bits, device)
        self.bt = _dev_i32(inp.block_table, device)
        self.lens = _dev_i32(inp.cache_seqlens, device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=device)
        self.h_q = torch.from_numpy(inp.q_bits.view(np.int16)).pin_memory()
        self.h_k = torch.from_numpy(inp.k_new_bits.view(np.int16)).pin_memory()
        self.h_v = torch.from_numpy(inp.v_new_bits.view(np.int16)).pin_memory()
        self.h_cu = torch.from_numpy(inp.cu_seqlens_q).pin_memory()
        self.h_lens = torch.from_numpy(inp.cache_seqlens).pin_memory()
        self.h_bt = torch.from_numpy(inp.block_table).pin_memory()
        self.h_out = torch.empty(self.q.shape, dtype=torch.int16).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()


class AppendCase:
    """fa_append_kv of the chunk's K/V rows into the paged cache."""

    def __init__(self, st: ChunkedState):
        self.st = st
        self.inp = st.inp
        self.bytes = st.inp.append_bytes()
        self.launches = 1

    def run(self):
        import exact_attention_148_b200 as fa
        s = self.st
        fa.append_kv(s.k_new, s.v_new, s.cu, s.kp, s.vp, s.bt, s.lens, layout=s.inp.layout)

    def run_e2e(self):
        """The step's inputs (chunk q/k/v and its table rows) come from pinned
        host memory; the cached prefix is resident state."""
        import torch
        s = self.st
        s.q.view(torch.int16).copy_(s.h_q, non_blocking=True)
        s.k_new.view(torch.int16).copy_(s.h_k, non_blocking=True)
        s.v_new.view(torch.int16).copy_(s.h_v, non_blocking=True)
        s.cu.copy_(s.h_cu, non_blocking=True)
        s.lens.copy_(s.h_lens, non_blocking=True)
        s.bt.copy_(s.h_bt, non_blocking=True)
        self.run()

    def h2d_bytes(self):
        i = self.inp
        return 2 * (i.q_bits.size + i.k_new_bits.size + i.v_new_bits.size) + \
            4 * (i.cu_seqlens_q.size + i.cache_seqlens.size + i.block_table.size)

    def d2h_bytes(self):
        return 0

    def describe(self):
        return {"kernel": "fa_append_kv_kernel", "new_tokens": int(self.inp.cu_seqlens_q[-1]),
                "algorithmic_gb": round(self.bytes / 1e9, 4)}


class ChunkedAttnCase:
    """fa_prefill_paged: the chunk's queries against each whole paged cache."""

    def __init__(self, st: ChunkedState):
        self.st = st
        self.inp = st.inp
        self.flops = st.inp.causal_flops()
        self.launches = -(-sum(-(-int(L) // 128) for L in st.inp.chunk_lens) // 2048)

    def run(self):
        import exact_attention_148_b200 as fa
        s = self.st
        fa.prefill_paged(s.q, s.cu, s.kp, s.vp, s.bt, s.lens, causal=s.inp.causal, scale=s.inp.scale,
                         layout=s.inp.layout, out=s.out, lse=s.lse,
                         cu_seqlens_q_host=s.inp.cu_seqlens_q, cache_seqlens_host=s.inp.cache_seqlens)
        # the schedule the library actually launched (see PrefillCase.run)
        self.schedule = fa.prefill_last_schedule()

    def run_e2e(self):
        import torch
        s = self.st
        self.run()
        s.h_out.copy_(s.out.view(torch.int16), non_blocking=True)
        s.h_lse.copy_(s.lse, non_blocking=True)

    def h2d_bytes(self):
        return 0

    def d2h_bytes(self):
        return 2 * self.inp.q_bits.size + 4 * self.st.lse.numel()

    def describe(self):
        i = self.inp
        return {"workload": i.name, "batch": i.batch, "chunk_tokens_total": int(i.chunk_lens.sum()),
                "prefix_tokens_total": int(i.prefix_lens.sum()), "num_q_heads": i.num_q_heads,
                "num_kv_heads": i.num_kv_heads, "head_dim": i.head_dim, "page_size": i.page_size,
                "layout": i.layout, "causal": bool(i.causal), "schedule": getattr(self, "schedule", None),
                "algorithmic_tflop": round(self.flops / 1e12, 4)}


class CascadeCase:
    """fa_cascade_decode: shared prefix read once for the batch + own suffixes."""

    def __init__(self, inp: W.CascadeInputs, device, kernel="auto"):
        import torch
        import exact_attention_148_b200 as fa
        self.inp = inp
        self.q = _dev_bf16(inp.q_bits, device)
        self.kp = _dev_bf16(inp.k_pages_bits, device)
        self.vp = _dev_bf16(inp.v_pages_bits, device)
        self.pre = _dev_i32(inp.prefix_block_table, device)
        self.bt = _dev_i32(inp.block_table, device)
        self.lens = _dev_i32(inp.suffix_lens, device)
        self.plan = fa.decode_plan(inp.suffix_lens, num_q_heads=inp.num_q_heads,
                                   num_kv_heads=inp.num_kv_heads, head_dim=inp.head_dim,
                                   max_pages_per_seq=inp.block_table.shape[1], kernel=kernel)
        self.ws = torch.empty(max(fa.cascade_workspace_bytes(self.plan, inp.prefix_len), 256),
                              dtype=torch.uint8, device=device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:-1], dtype=torch.float32, device=device)
        self.bytes = inp.algorithmic_bytes()
        self.launches = 3 + (1 if self.plan.info.max_splits > 1 else 0)
        self.h_q = torch.from_numpy(inp.q_bits.view(np.int16)).pin_memory()
        self.h_out = torch.empty(self.q.shape, dtype=torch.int16).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def run(self):
        import exact_attention_148_b200 as fa
        fa.cascade_decode(self.q, self.kp, self.vp, self.pre, self.inp.prefix_len, self.bt, self.lens,
                          self.plan, layout=self.inp.layout, scale=self.inp.scale, out=self.out,
                          lse=self.lse, workspace=self.ws)

    def run_e2e(self):
        """The step's input is the batch's query rows; the paged cache is resident."""
        import torch
        self.q.view(torch.int16).copy_(self.h_q, non_blocking=True)
        self.run()
        self.h_out.copy_(self.out.view(torch.int16), non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def h2d_bytes(self):
        return 2 * self.inp.q_bits.size

    def d2h_bytes(self):
        return 2 * self.inp.q_bits.size + 4 * self.lse.numel()

    def describe(self):
        i = self.inp
        return {"workload": i.name, "batch": i.batch, "prefix_len": i.prefix_len,
                "suffix_tokens_total": int(i.suffix_lens.sum()), "num_q_heads": i.num_q_heads,
                "num_kv_heads": i.num_kv_heads, "head_dim": i.head_dim,
                "algorithmic_gb": round(self.bytes / 1e9, 4),
                "suffix_split_kernel": "tensor cores (tcgen05)" if self.plan.info.tensor_cores
                else "CUDA cores"}


# ----------------------------------------------------------------------------- timing

def time_cases(cases, steps, warmup, flush, dist_ctx, e2e=False):
    """Per case: total device ms over `steps` timed steps (each case of a step
    bracketed by its own CUDA events on the current stream; L2 flushed before
    every step outside the events).  Returns (per-case ms list, total ms)."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for c in cases:
            (c.run_e2e if e2e else c.run)()
    torch.cuda.synchronize()
    if dist_ctx is not None:
        dist_ctx.barrier()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in cases] for _ in range(steps)]
    for s in range(steps):
        flush.zero_()
        for ci, c in enumerate(cases):
            evs[s][ci][0].record(stream)
            (c.run_e2e if e2e else c.run)()
            evs[s][ci][1].record(stream)
    torch.cuda.synchronize()
    if dist_ctx is not None:
        dist_ctx.barrier()
    torch.cuda.synchronize()
    per_case = [sum(evs[s][ci][0].elapsed_time(evs[s][ci][1]) for s in range(steps)) for ci in range(len(cases))]
    if dist_ctx is not None:
        per_case = dist_ctx.max_over_ranks(per_case)
    return per_case


def time_e2e_overlapped(case, steps, warmup, dist_ctx):
    """End-to-end time per step of one case with consecutive steps overlapped:
    step s's host->device copies (stream A), its C-ABI call (the current
    stream) and its device->host copies (stream B) run while steps s-1 and
    s+1 are in other stages.  Inputs and outputs are double-buffered on the
    device; events order each buffer's reuse (copy-in after the compute two
    steps back, compute after the copy-out two steps back).  Every step still
    copies all of its inputs in and its outputs out.  Returns ms per step
    (device time, max over ranks)."""
    import torch
    fin, fout = case.e2e_fields()
    slots = [{}, {}]
    for dev_attr, _, _ in fin + fout:
        t = getattr(case, dev_attr)
        slots[0][dev_attr] = t
        slots[1][dev_attr] = torch.empty_like(t)
    host_out = [{h: getattr(case, h) for _, h, _ in fout},
                {h: torch.empty_like(getattr(case, h)).pin_memory() for _, h, _ in fout}]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    out_done = [torch.cuda.Event(), torch.cuda.Event()]
    used = [False, False]

    def view(t, bits):
        return t.view(torch.int16) if bits else t

    def one(step):
        b = step % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(comp_done[b])
            for dev_attr, h, bits in fin:
                view(slots[b][dev_attr], bits).copy_(getattr(case, h), non_blocking=True)
            in_done[b].record(s_in)
        comp.wait_event(in_done[b])
        if used[b]:
            comp.wait_event(out_done[b])
        for dev_attr in slots[b]:
            setattr(case, dev_attr, slots[b][dev_attr])
        case.run()
        comp_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for dev_attr, h, bits in fout:
                host_out[b][h].copy_(view(slots[b][dev_attr], bits), non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True

    try:
        for i in range(warmup):
            one(i)
        torch.cuda.synchronize()
        if dist_ctx is not None:
            dist_ctx.barrier()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(comp)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(steps):
            one(warmup + i)
        comp.wait_event(out_done[(warmup + steps - 1) % 2])
        end.record(comp)
        torch.cuda.synchronize()
    finally:
        # the case keeps its own buffers even when a call raised part way
        torch.cuda.synchronize()
        for dev_attr in slots[0]:
            setattr(case, dev_attr, slots[0][dev_attr])
    ms = start.elapsed_time(end) / steps
    if dist_ctx is not None:
        ms = dist_ctx.max_over_ranks([ms])[0]
    return ms


class DistCtx:
    """One process per GPU (NCCL), or CPU ranks over gloo for tests.  Ranks are
    independent replicas: the only collectives are the barriers around the
    timed region and the max over ranks of the measured times."""

    def __init__(self, backend="nccl", timeout_s=300):
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        self.dist = dist
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s))
        self.rank = dist.get_rank()
        self.world = dist.get_world_size()
        self.local = int(os.environ.get("LOCAL_RANK", 0))
        self.device = "cpu"
        if backend == "nccl":
            torch.cuda.set_device(self.local)
            self.device = "cuda"

    def barrier(self):
        self.dist.barrier()

    def max_over_ranks(self, vals):
        import torch
        t = torch.tensor(vals, dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return t.tolist()

    def close(self):
        self.dist.destroy_process_group()


# ----------------------------------------------------------------------------- CPU oracle legs

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name and logical core count (/proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return f"{ln.split(':', 1)[1].strip()}, {os.cpu_count()} logical cores"
    except OSError:
        pass
    return f"unknown, {os.cpu_count()} logical cores"


def oracle_prefill_sample(inp: W.PrefillInputs, budget_s: float):
    """Run the oracle on whole (sequence, head) blocks until about budget_s has
    passed; returns (flops done, seconds, description)."""
    import oracle
    order = np.argsort(inp.seqlens)          # shortest sequences first
    flops, secs, done = 0.0, 0.0, []
    d = inp.head_dim
    G = inp.num_q_heads // inp.num_kv_heads
    for h in range(inp.num_q_heads):         # one (sequence, head) block at a time
        for b in order:
            s0, s1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
            L = s1 - s0
            g = h // G
            if isinstance(inp, W.Fp8PrefillInputs):
                q = oracle.dequantize_e4m3(inp.q_bits[s0:s1, h:h + 1], inp.q_scale)
                k = oracle.dequantize_e4m3(inp.k_bits[s0:s1, g:g + 1], inp.k_scale)
                v = oracle.dequantize_e4m3(inp.v_bits[s0:s1, g:g + 1], inp.v_scale)
            else:
                q = W.as_f64(inp.q_bits[s0:s1, h:h + 1])
                k = W.as_f64(inp.k_bits[s0:s1, g:g + 1])
                v = W.as_f64(inp.v_bits[s0:s1, g:g + 1])
            t0 = time.perf_counter()
            oracle.attention_ref(q, k, v, [0, L], inp.causal, inp.scale)
            secs += time.perf_counter() - t0
            pairs = L * (L + 1) // 2 if inp.causal else L * L
            flops += 4.0 * d * pairs
            done.append((h, L))
            if secs >= budget_s:
                break
        if secs >= budget_s:
            break
    heads = sorted({h for h, _ in done})
    return flops, secs, (f"oracle attention_ref on {len(done)} (sequence, head) blocks, heads "
                         f"{heads[0]}-{heads[-1]}, sequence lengths {sorted({L for _, L in done})}")


def oracle_decode_sample(inp: W.DecodeInputs, budget_s: float):
    import oracle
    flops_bytes, secs, rows = 0.0, 0.0, []
    G = inp.num_q_heads // inp.num_kv_heads
    conv = {}
    if inp.kv_elem_bytes == 1:
        ks, vs = inp.extra["k_scale"], inp.extra["v_scale"]
        conv = dict(k_to_f64=lambda a: oracle.dequantize_e4m3(a, ks),
                    v_to_f64=lambda a: oracle.dequantize_e4m3(a, vs))
    QL = inp.q_len
    for b in range(inp.batch):
        heads = list(range(0, inp.num_q_heads, G))[:2]              # two kv heads' first q head
        t0 = time.perf_counter()
        if QL == 1:
            oracle.paged_decode_rows_ref(inp.q_bits, inp.k_pages_bits, inp.v_pages_bits,
                                         inp.block_table, inp.cache_seqlens, inp.scale,
                                         [(b, h) for h in heads], inp.page_size, inp.layout,
                                         to_f64=W.as_f64, **conv)
        else:   # multi-token decode: the chunked-prefill oracle on the packed tokens
            qp = inp.q_bits.reshape(inp.batch * QL, inp.num_q_heads, inp.head_dim)
            cu = np.arange(inp.batch + 1) * QL
            oracle.paged_prefill_rows_ref(qp, cu, inp.k_pages_bits, inp.v_pages_bits, inp.block_table,
                                          inp.cache_seqlens, True, inp.scale,
                                          [(b * QL + t, h) for h in heads for t in range(QL)],
                                          inp.page_size, inp.layout, to_f64=W.as_f64)
        secs += time.perf_counter() - t0
        flops_bytes += len(rws) * 2.0 * int(inp.cache_seqlens[b]) * inp.head_dim * inp.kv_elem_bytes
        rows.append(b)
        if secs >= budget_s:
            break
    return flops_bytes, secs, f"oracle paged_decode_rows_ref, 2 kv heads of requests {rows}"


def oracle_chunked_sample(inp: W.ChunkedPrefillInputs, budget_s: float):
    """The oracle's chunked prefill on one (request, query head) at a time,
    shortest requests first, until about budget_s has passed."""
    import oracle
    kp_all, vp_all = oracle.append_kv_ref(inp.k_pages_bits, inp.v_pages_bits, inp.k_new_bits,
                                          inp.v_new_bits, inp.cu_seqlens_q, inp.block_table,
                                          inp.cache_seqlens, inp.page_size, inp.layout)
    head_axis = 2 if inp.layout == "NHD" else 1
    kp = np.take(kp_all, [0], axis=head_axis)
    vp = np.take(vp_all, [0], axis=head_axis)
    flops, secs, done = 0.0, 0.0, []
    cu = inp.cu_seqlens_q
    for b in np.argsort(inp.cache_seqlens):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n, k = s1 - s0, int(inp.cache_seqlens[b])
        t0 = time.perf_counter()
        oracle.paged_prefill_ref(inp.q_bits[s0:s1, 0:1], [0, n], kp, vp, inp.block_table[b:b + 1],
                                 inp.cache_seqlens[b:b + 1], inp.causal, inp.scale, inp.page_size,
                                 inp.layout, to_f64=W.as_f64)
        secs += time.perf_counter() - t0
        pairs = n * (k - n) + n * (n + 1) // 2 if inp.causal else n * k
        flops += 4.0 * inp.head_dim * pairs
        done.append((k - n, n))
        if secs >= budget_s:
            break
    return flops, secs, (f"oracle paged_prefill_ref on query head 0 of requests with "
                         f"(prefix, chunk) = {done}")


def oracle_cascade_sample(inp: W.CascadeInputs, budget_s: float):
    """The oracle's cascade decode, one request at a time, until about budget_s;
    work is counted in the cascade's own algorithmic bytes per request."""
    import oracle
    secs, done = 0.0, []
    per_req = inp.algorithmic_bytes() / inp.batch
    for b in range(inp.batch):
        t0 = time.perf_counter()
        oracle.cascade_decode_ref(inp.q_bits[b:b + 1], inp.k_pages_bits, inp.v_pages_bits,
                                  inp.prefix_block_table, inp.prefix_len, inp.block_table[b:b + 1],
                                  inp.suffix_lens[b:b + 1], inp.scale, inp.page_size, inp.layout,
                                  to_f64=W.as_f64)
        secs += time.perf_counter() - t0
        done.append(b)
        if secs >= budget_s:
            break
    return per_req * len(done), secs, f"oracle cascade_decode_ref on requests {done}"


# ----------------------------------------------------------------------------- main

def decode_inputs(workload, heads=None):
    """A decode workload, optionally with its query / kv head counts replaced
    (same cache lengths, seeded draws): heads = "HQ:HKV"."""
    inp = W.CONFIGS[workload]()
    if heads:
        hq, hkv = (int(x) for x in heads.split(":"))
        inp = W.make_decode(inp.cache_seqlens, hq, hkv, inp.head_dim, seed=hq * 1000 + hkv,
                            name=f"{workload}_h{hq}x{hkv}")
    return inp


def build_cases(workload, device, num_splits, kernel="auto", heads=None):
    if workload == "default":
        return [PrefillCase(W.varlen_causal_prefill(), device),
                DecodeCase(W.paged_decode_batch(), device, 0, kernel)]
    if workload in PREFILL_WORKLOADS:
        return [PrefillCase(W.CONFIGS[workload](), device)]
    if workload in DECODE_WORKLOADS:
        return [DecodeCase(decode_inputs(workload, heads), device, num_splits, kernel)]
    if workload in CHUNKED_WORKLOADS:
        st = ChunkedState(W.CONFIGS[workload](), device)
        return [AppendCase(st), ChunkedAttnCase(st)]
    if workload in CASCADE_WORKLOADS:
        inp = W.CONFIGS[workload]()
        return [CascadeCase(inp, device, kernel), DecodeCase(inp.as_plain_decode(), device, 0, kernel)]
    raise SystemExit(f"unknown workload {workload}")


def kernel_source_hash(kind):
    import hashlib
    files = {"prefill": ["ptx_sm100.cuh", "prefill_pp_sm100.cuh"],
             "prefill_persist": ["ptx_sm100.cuh", "prefill_pp_sm100.cuh", "prefill_persist_sm100.cuh"],
             "decode": ["ptx_sm100.cuh", "decode_sm100.cuh"],
             "decode_tc": ["ptx_sm100.cuh", "decode_sm100.cuh", "decode_tc_sm100.cuh"],
             "append": ["ptx_sm100.cuh", "append_sm100.cuh"]}[kind]
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_attention_148_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def pages_shared(inp) -> bool:
    """True when some page id sits in more than one used block-table slot (a
    prefix shared by several requests): such pages are fetched once and then
    re-read from L2, so DRAM bytes no longer follow the K/V bytes."""
    ps = inp.page_size
    used = [inp.block_table[b, :(int(L) + ps - 1) // ps] for b, L in enumerate(inp.cache_seqlens)]
    ids = np.concatenate(used) if used else np.zeros(0, np.int32)
    return len(np.unique(ids)) != len(ids)


def measured_traffic(kind, workload, case=None):
    """(DRAM bytes per launch, how it was obtained) from profiles/dram_traffic.md,
    or (None, None) when no capture matches the current kernel source.  A decode
    workload without its own row uses the 16-request capture of the same split
    kernel scaled by K/V bytes (every decode capture reads its K/V bytes one for
    one), unless its requests share pages; the full-size workloads are too large
    for a multi-pass capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None, None
    rows = {}
    for ln in lines:
        parts = [x.strip() for x in ln.strip().strip("|").split("|")]
        if len(parts) >= 5 and parts[0] in ("prefill", "prefill_persist", "decode", "decode_tc", "append") \
                and parts[3].isdigit():
            rows[(parts[0], parts[1])] = (parts[2], int(parts[3]) + int(parts[4]))
    sha = kernel_source_hash(kind)
    if (kind, workload) in rows and rows[(kind, workload)][0] == sha:
        return rows[(kind, workload)][1], "ncu capture of this workload"
    if kind in ("decode", "decode_tc") and case is not None and not case.fp8 and \
            (kind, "paged_decode_batch16") in rows and not pages_shared(case.inp):
        h, t16 = rows[(kind, "paged_decode_batch16")]
        if h == sha:
            kv16 = 2.0 * float(np.sum(W.paged_decode_batch16_lengths())) * 8 * 128 * 2
            return int(t16 * case.inp.kv_bytes() / kv16), \
                "16-request ncu capture of the same split kernel, scaled by K/V bytes"
    return None, None


def aggregate_throughput(work_per_replica: float, ms_max: float, n_replicas: int, scale: float) -> float:
    """Whole-job throughput of N independent replicas: every replica does the
    same work; the job takes as long as the slowest replica (max over ranks)."""
    return n_replicas * work_per_replica / (ms_max * 1e-3) / scale


def roofline_entry(kind, algorithmic, ms_per_launch, peaks, peak_src, traffic=(None, None), fp8_qk=False):
    traffic, traffic_src = traffic
    if kind == "tensor":
        achieved = algorithmic / (ms_per_launch * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        src = f"{peak_src} bf16 dense (burst)"
        spec = SPEC_PEAKS["bf16_tflops"]
        if fp8_qk:
            # half the FLOPs (Q K^T) at the E4M3 rate, nominally 2x bf16, the
            # other half (P V, f16) at the bf16 rate: 2 / (1/2 + 1) = 4/3
            peak, spec = round(peak * 4.0 / 3.0, 1), spec * 4.0 / 3.0
            src += " x 4/3 (Q K^T at the fp8 rate = 2 x bf16 nominal, P V at the f16 rate)"
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_source": traffic_src,
                "peak_source": src, "frac_of_spec": round(achieved / spec, 4)}
    achieved = algorithmic / (ms_per_launch * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_source": traffic_src,
            "peak_source": f"{peak_src} HBM copy", "frac_of_spec": round(achieved / SPEC_PEAKS["hbm_gbs"], 4)}


# The other configurations of the benchmark, timed in the default run after the
# headline step: (workload, split counts swept besides the planner's choice).
LEGS = [("long_gqa_prefill", ()), ("long_split_decode", (1, 2, 4, 8, 16, 32, 64)),
        ("ragged_split_decode", ())]


def case_roofline(c, ms, peaks, peak_src):
    """Roofline entry of one case's kernel(s) at `ms` per call."""
    if isinstance(c, PrefillCase):
        pers = getattr(c, "schedule", None) == "persistent"
        e = roofline_entry("tensor", c.flops, ms / c.launches, peaks, peak_src,
                           measured_traffic("prefill_persist" if pers else "prefill", c.inp.name),
                           fp8_qk=c.fp8)
        e["kernel"] = "%s<%d%s>" % ("fa_prefill_persist_kernel" if pers else "fa_prefill_pp_kernel",
                                    c.inp.head_dim, ", e4m3" if c.fp8 else "")
        return e
    e = roofline_entry("hbm", c.bytes, ms, peaks, peak_src,
                       measured_traffic("decode_tc" if c.plan.info.tensor_cores else "decode",
                                        c.inp.name, c))
    e["kernel"] = ("fa_decode_tc_kernel" if c.plan.info.tensor_cores else "fa_decode_split_kernel") + \
        ("<e4m3>" if c.fp8 else "") + " + fa_merge_kernel (one decode call)"
    return e


def run_legs(args, device, flush, peaks, peak_src):
    """Time every other configuration once on this GPU (rank 0's replica):
    value, ms, roofline and clocks per leg; the long split decode also over a
    sweep of split counts.  Each leg's inputs are freed before the next."""
    import torch
    legs = []
    steps = max(3, min(args.steps, 10))
    for workload, sweep in LEGS:
        c = build_cases(workload, device, 0)[0]
        sampler = ClockSampler(device.index if device.index is not None else 0)
        sampler.start()
        ms = time_cases([c], steps, 3, flush, None)[0] / steps
        rows = []
        for ns in sweep:
            c.replan(ns)
            t = time_cases([c], steps, 2, flush, None)[0] / steps
            rows.append({"num_splits": ns, "max_splits": c.plan.info.max_splits, "ms": round(t, 4),
                         "gbs": round(c.bytes / (t * 1e-3) / 1e9, 1)})
        clocks = sampler.stop()
        if sweep:
            c.replan(0)                      # describe the planner's own choice
        prefill = isinstance(c, PrefillCase)
        leg = {"workload": workload,
               "value": round(c.flops / (ms * 1e-3) / 1e12, 3) if prefill else round(c.bytes / (ms * 1e-3) / 1e9, 1),
               "unit": "TFLOP/s" if prefill else "GB/s", "ms": round(ms, 4), "steps": steps,
               "launches_per_call": c.launches,
               "roofline": case_roofline(c, ms, peaks, peak_src), "clocks": clocks,
               "config": c.describe()}
        if sweep:
            auto = {"num_splits": "auto", "max_splits": c.plan.info.max_splits, "ms": round(ms, 4),
                    "gbs": leg["value"]}
            leg["splits_sweep"] = rows + [auto]
        legs.append(leg)
        del c
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return legs


def run_ours(args):
    import torch
    import exact_attention_148_b200 as fa  # noqa: F401  (fails loudly if the library is missing)
    fa.library()
    dist_ctx = DistCtx() if args.gpus > 1 else None
    rank = dist_ctx.rank if dist_ctx else 0
    device = torch.device("cuda", dist_ctx.local if dist_ctx else 0)
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()
    cases = build_cases(args.workload, device, args.num_splits, args.decode_kernel, args.decode_heads)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    per_case = time_cases(cases, args.steps, args.warmup, flush, dist_ctx)
    clocks = sampler.stop()
    status = fa.device_status(clear=True)

    e2e_case = None
    overlapped = not args.e2e_serial and all(hasattr(c, "e2e_fields") for c in cases)
    if not args.no_e2e:
        if overlapped:
            e2e_steps = max(2, min(args.steps, 8))
            e2e_case = [time_e2e_overlapped(c, e2e_steps, 2, dist_ctx) for c in cases]
        else:
            e2e_steps = max(1, min(args.steps, 5))
            e2e_case = time_cases(cases, e2e_steps, 1, flush, dist_ctx, e2e=True)
            e2e_case = [x / e2e_steps for x in e2e_case]

    N = args.gpus
    ms_case = [x / args.steps for x in per_case]
    ms_step = sum(ms_case)
    line = {"metric": METRIC}
    launches = sum(c.launches for c in cases) * args.steps
    main = cases[0]
    rooflines = []
    for c, ms in zip(cases, ms_case):
        if isinstance(c, PrefillCase):
            e = case_roofline(c, ms, peaks, peak_src)
        elif isinstance(c, ChunkedAttnCase):
            pers = getattr(c, "schedule", None) == "persistent"
            e = roofline_entry("tensor", c.flops, ms / c.launches, peaks, peak_src,
                               measured_traffic("prefill_persist" if pers else "prefill", c.inp.name))
            e["kernel"] = "%s<%d, paged>" % ("fa_prefill_persist_kernel" if pers else "fa_prefill_pp_kernel",
                                             c.inp.head_dim)
        elif isinstance(c, CascadeCase):
            e = roofline_entry("hbm", c.bytes, ms, peaks, peak_src)
            e["kernel"] = "fa_prefill_pp_kernel<paged, key ranges> + decode split + fa_cascade_merge_kernel"
        elif isinstance(c, AppendCase):
            e = roofline_entry("hbm", c.bytes, ms, peaks, peak_src,
                               measured_traffic("append", c.inp.name))
            e["kernel"] = "fa_append_kv_kernel<%d>" % c.inp.head_dim
        else:
            e = case_roofline(c, ms, peaks, peak_src)
        e["workload"] = c.inp.name
        e["ms_per_launch"] = round(ms / c.launches, 4)
        rooflines.append(e)
    chunked = isinstance(main, AppendCase)
    cascade = isinstance(main, CascadeCase)
    if cascade:
        value = aggregate_throughput(main.bytes, ms_case[0], N, 1e9)
        unit = "GB/s"
    elif chunked:
        # the whole chunked step (append + attention) against the attention FLOPs
        value = aggregate_throughput(cases[1].flops, ms_step, N, 1e12)
        unit = "TFLOP/s"
    elif isinstance(main, PrefillCase):
        value = aggregate_throughput(main.flops, ms_case[0], N, 1e12)
        unit = "TFLOP/s"
    else:
        value = aggregate_throughput(main.bytes, ms_case[0], N, 1e9)
        unit = "GB/s"
    # `roofline` is the kernel with the largest share of the measured step time;
    # the cascade's step is the cascade call alone (the plain decode beside it
    # is a comparison, reported with its own roofline under its own key).
    rl = rooflines[0] if cascade else rooflines[int(np.argmax(ms_case))]
    line.update({"value": round(value, 3), "unit": unit, "n_gpus": N, "steps": args.steps,
                 "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
                 "scaling": "weak", "vs_baseline": None,
                 "dtype": "e4m3 in, fp32 accumulate" if getattr(main, "fp8", False) else "bf16",
                 "data": "synthetic (seeded N(0,1) rounded to bf16; see workloads/)"})
    cfg = {"workload": cases[1].inp.name + " (append + chunked prefill)" if chunked else
           " + ".join(c.inp.name for c in cases),
           "l2": "flushed before every step (256 MiB write), outside the timed events; "
                 "inputs also exceed L2",
           "parallelism": f"replicas x{N}" if N > 1 else "single GPU"}
    for i, c in enumerate(cases):
        key = {PrefillCase: "prefill", DecodeCase: "decode", AppendCase: "append",
               ChunkedAttnCase: "chunked_prefill", CascadeCase: "cascade"}[type(c)]
        cfg[key] = c.describe()
    line["config"] = cfg
    line["roofline"] = rl
    if cascade:
        line["plain_decode_same_contexts"] = {
            "ms": round(ms_case[1], 4), "speedup_of_cascade": round(ms_case[1] / ms_case[0], 3),
            "roofline": rooflines[1],
            "note": "fa_decode_paged over prefix+suffix table rows (prefix read per request; "
                    "its repeated prefix reads hit L2, so it can exceed the copy peak)"}
        line["ms_per_step"] = round(ms_case[0], 4)
    elif chunked:
        line["append"] = {"value": round(N * main.bytes / (ms_case[0] * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "ms": round(ms_case[0], 4), "roofline": rooflines[0]}
        line["chunked_prefill_ms"] = round(ms_case[1], 4)
        line["chunked_prefill_tflops"] = round(N * cases[1].flops / (ms_case[1] * 1e-3) / 1e12, 2)
    elif len(cases) > 1:
        dc = cases[1]
        line["decode"] = {"value": round(N * dc.bytes / (ms_case[1] * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "ms": round(ms_case[1], 4), "roofline": rooflines[1],
                          "timed_over": "fa_decode_paged call (split kernel + merge kernel)"}
        line["prefill_ms"] = round(ms_case[0], 4)
        line["prefill_roofline"] = rooflines[0]
    if e2e_case is not None:
        if cascade:
            e2e_v = N * main.bytes / (e2e_case[0] * 1e-3) / 1e9
        elif chunked:
            e2e_v = N * cases[1].flops / (sum(e2e_case) * 1e-3) / 1e12
        elif isinstance(main, PrefillCase):
            e2e_v = N * main.flops / (e2e_case[0] * 1e-3) / 1e12
        else:
            e2e_v = N * main.bytes / (e2e_case[0] * 1e-3) / 1e9
        line["e2e"] = {"value": round(e2e_v, 3), "unit": unit,
                       "h2d_bytes_per_step": int(sum(c.h2d_bytes() for c in cases)),
                       "d2h_bytes_per_step": int(sum(c.d2h_bytes() for c in cases)),
                       "ms_per_step": round(sum(e2e_case), 3),
                       "path": "pinned host -> device copies of each step's inputs (prefill q/k/v; "
                               "decode q, block table, lengths), C-ABI calls, device -> pinned host "
                               "copies of O and LSE; the paged KV cache is resident state",
                       "steps": ("overlapped: step s+1 copies in and step s-1 copies out while step s "
                                 "computes (double-buffered device inputs and outputs)" if overlapped
                                 else "serial: copy in, compute, copy out, one step after another")}
    if args.workload == "default" and N == 1 and not args.no_legs:
        line["legs"] = run_legs(args, device, flush, peaks, peak_src)
        line["legs_device_status"] = fa.device_status(clear=True)
        line["legs_note"] = ("the benchmark's other configurations, each timed alone after the "
                             "headline step (CUDA events, L2 flushed before every step); not part of "
                             "value, ms_per_step or gpu_launches")
    line["gpu_launches"] = int(launches)
    line["clocks"] = clocks
    line["device_status"] = status
    if rank == 0 and N == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cases[1] if chunked else main, args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_ctx is not None:
        dist_ctx.close()


def cpu_baseline(case, budget):
    threads = blas_threads()
    if isinstance(case, PrefillCase):
        work, secs, desc = oracle_prefill_sample(case.inp, budget)
        val, unit = work / secs / 1e12, "TFLOP/s"
    elif isinstance(case, ChunkedAttnCase):
        work, secs, desc = oracle_chunked_sample(case.inp, budget)
        val, unit = work / secs / 1e12, "TFLOP/s"
    elif isinstance(case, CascadeCase):
        work, secs, desc = oracle_cascade_sample(case.inp, budget)
        val, unit = work / secs / 1e9, "GB/s"
    else:
        work, secs, desc = oracle_decode_sample(case.inp, budget)
        val, unit = work / secs / 1e9, "GB/s"
    return {"value": val, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": f"{desc}; {secs:.1f} s of CPU time", "cpu": cpu_model()}


def run_reference(args):
    """The oracle, as it stands, timed on the host cores on a bounded sample
    of the same workload (rank 0 only; other ranks exit without work)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    main = args.workload
    if main == "default":
        inp = W.varlen_causal_prefill()
        is_prefill = True
    elif main in PREFILL_WORKLOADS or main in CHUNKED_WORKLOADS:
        inp = W.CONFIGS[main]()
        is_prefill = True
    else:
        inp = W.CONFIGS[main]()
        is_prefill = False
    per_step = max(1.0, args.cpu_budget / max(1, args.steps))
    fn = oracle_prefill_sample if is_prefill else oracle_decode_sample
    if main in CHUNKED_WORKLOADS:
        fn = oracle_chunked_sample
    if main in CASCADE_WORKLOADS:
        fn = oracle_cascade_sample
    for _ in range(args.warmup and 1):
        fn(inp, 0.0)
    work, secs = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        w, s, desc = fn(inp, per_step)
        work += w
        secs += s
    if is_prefill:
        value, unit = work / secs / 1e12, "TFLOP/s"
    else:
        value, unit = work / secs / 1e9, "GB/s"
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) rounded to bf16; see workloads/)",
            "config": {"workload": inp.name if not (main == "default") else
                       "varlen_causal_prefill + paged_decode_batch (prefill half sampled)"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                             "sample": desc, "cpu": cpu_model()},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=int(os.environ.get("WORLD_SIZE", "1")))
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="default",
                    help="default | " + " | ".join(sorted(PREFILL_WORKLOADS | DECODE_WORKLOADS |
                                                          CHUNKED_WORKLOADS | CASCADE_WORKLOADS)))
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--decode-kernel", default="auto", choices=["auto", "cuda_cores", "tensor_cores"])
    ap.add_argument("--decode-heads", default=None, help="HQ:HKV override for a decode workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="default workload: skip the other configurations' legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time")
    ap.add_argument("--e2e-serial", action="store_true",
                    help="end-to-end leg without overlap: copy in, compute, copy out, one step after "
                         "another (default: consecutive steps' copies overlap the compute)")
    ap.add_argument("--prefill-schedule", default=None, choices=["grid", "persistent"],
                    help="packed prefill: one CTA per work item (grid) or one per SM (persistent); "
                         "default: the library's (FA_PREFILL_SCHEDULE, else persistent)")
    args = ap.parse_args()
    if args.prefill_schedule is not None:
        os.environ["FA_PREFILL_SCHEDULE"] = args.prefill_schedule
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
