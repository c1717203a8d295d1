"""exact_attention_148_b200 — B200 (sm_100a) exact attention forward.

Thin Python binding over the C ABI in ``include/exact_attention.h``: it only
marshals arguments (device pointers, sizes, the current CUDA stream) into
``libexact_attention.so``; every step of the computation runs in that
library's CUDA kernels.  PyTorch provides device memory and streams.

There is no CPU fallback: if the shared library is missing, or a tensor is not
a CUDA tensor, the call raises.

``FA_LIBRARY=debug`` in the environment (or ``select_library("debug")``) loads
the bounds-checked build ``libexact_attention_debug.so`` instead: the same
kernels with every computed global index checked against its buffer, a
failure recorded as FA_ERR_DEBUG_INDEX in the device status word.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

__all__ = [
    "FAError", "library", "lib_path", "prefill", "decode_plan", "DecodePlan", "decode_paged",
    "decode_paged_static", "merge_states", "device_status", "strerror", "EXPORTED_SYMBOLS",
    "append_kv", "prefill_paged", "prefill_fp8", "decode_paged_fp8", "cascade_decode", "cascade_workspace_bytes",
    "prefill_last_schedule", "select_library", "debug_selftest_index",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
release_lib_path = os.path.join(_PKG_DIR, "libexact_attention.so")
debug_lib_path = os.path.join(_PKG_DIR, "libexact_attention_debug.so")
lib_path = debug_lib_path if os.environ.get("FA_LIBRARY") == "debug" else release_lib_path

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_WORKSPACE = -3
FA_ERR_CUDA = -4
FA_ERR_TIMEOUT = -5
FA_ERR_PLAN_MISMATCH = -6
FA_ERR_BAD_PAGE = -7
FA_ERR_DEBUG_INDEX = -8

EXPORTED_SYMBOLS = [
    "fa_prefill", "fa_decode_plan", "fa_plan_get_info", "fa_plan_free", "fa_decode_paged",
    "fa_merge_states", "fa_strerror", "fa_last_cuda_error", "fa_get_device_status", "fa_version",
    "fa_decode_paged_static", "fa_selftest_wait_timeout", "fa_append_kv", "fa_prefill_paged",
    "fa_decode_paged_fp8", "fa_decode_plan_kv", "fa_decode_plan_ex", "fa_cascade_workspace_bytes",
    "fa_cascade_decode", "fa_prefill_fp8", "fa_prefill_last_schedule", "fa_debug_selftest_index",
]

FA_KV_BF16, FA_KV_E4M3 = 0, 1
FA_DECODE_AUTO, FA_DECODE_CUDA_CORES, FA_DECODE_TENSOR_CORES = 0, 1, 2
FA_SCHEDULE_GRID, FA_SCHEDULE_PERSISTENT = 0, 1
_KV_DTYPES = {"bf16": FA_KV_BF16, "e4m3": FA_KV_E4M3}
_KERNELS = {"auto": FA_DECODE_AUTO, "cuda_cores": FA_DECODE_CUDA_CORES,
            "tensor_cores": FA_DECODE_TENSOR_CORES}

# Size of the library's static decode scratch (FA_STATIC_SCRATCH_BYTES).
STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {strerror(status)} ({status})"
        if status == FA_ERR_CUDA:
            msg += f", cuda error {library().fa_last_cuda_error()}"
        super().__init__(msg)


class _PlanInfo(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("page_size", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int),
        ("chunk_tokens", ctypes.c_int), ("max_splits", ctypes.c_int), ("heads_per_cta", ctypes.c_int),
        ("num_work_items", ctypes.c_int), ("max_seqlen", ctypes.c_int),
        ("workspace_bytes", ctypes.c_size_t), ("kv_dtype", ctypes.c_int),
        ("tensor_cores", ctypes.c_int), ("q_len", ctypes.c_int),
    ]


class _DecodeOptions(ctypes.Structure):
    _fields_ = [("kv_dtype", ctypes.c_int), ("kernel", ctypes.c_int), ("q_len", ctypes.c_int)]


_lib = None


def library() -> ctypes.CDLL:
    """Load the in-tree shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(lib_path):
        raise RuntimeError(f"{lib_path} is missing; build it with "
                           "`python -m exact_attention_148_b200._build`")
    L = ctypes.CDLL(lib_path)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    L.fa_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp, vp]
    L.fa_prefill.restype = i32
    L.fa_prefill_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32, f32,
                                 vp, vp, vp]
    L.fa_prefill_fp8.restype = i32
    L.fa_decode_plan.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                 ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_size_t)]
    L.fa_decode_plan.restype = i32
    L.fa_decode_plan_kv.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, i32,
                                    ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_size_t)]
    L.fa_decode_plan_kv.restype = i32
    L.fa_decode_plan_ex.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                    ctypes.POINTER(_DecodeOptions), ctypes.POINTER(vp),
                                    ctypes.POINTER(ctypes.c_size_t)]
    L.fa_decode_plan_ex.restype = i32
    L.fa_cascade_workspace_bytes.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_size_t)]
    L.fa_cascade_workspace_bytes.restype = i32
    L.fa_cascade_decode.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, i32, vp, vp, vp, f32, vp, vp,
                                    vp, ctypes.c_size_t, vp]
    L.fa_cascade_decode.restype = i32
    L.fa_plan_get_info.argtypes = [vp, ctypes.POINTER(_PlanInfo)]
    L.fa_plan_get_info.restype = i32
    L.fa_plan_free.argtypes = [vp]
    L.fa_plan_free.restype = None
    L.fa_decode_paged.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, f32, vp, vp, vp,
                                  ctypes.c_size_t, vp]
    L.fa_decode_paged.restype = i32
    L.fa_merge_states.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
    L.fa_merge_states.restype = i32
    L.fa_strerror.argtypes = [i32]
    L.fa_strerror.restype = ctypes.c_char_p
    L.fa_last_cuda_error.argtypes = []
    L.fa_last_cuda_error.restype = i32
    L.fa_get_device_status.argtypes = [vp, ctypes.POINTER(i32), i32]
    L.fa_get_device_status.restype = i32
    L.fa_version.argtypes = []
    L.fa_version.restype = i32
    L.fa_decode_paged_static.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, f32, vp, vp, vp]
    L.fa_decode_paged_static.restype = i32
    L.fa_selftest_wait_timeout.argtypes = [i64, vp]
    L.fa_selftest_wait_timeout.restype = i32
    L.fa_append_kv.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, i64, i64, i64, i64, i32, vp,
                               i32, vp, vp]
    L.fa_append_kv.restype = i32
    L.fa_prefill_paged.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, vp, vp, i32,
                                   i32, i32, i32, i32, i32, f32, vp, vp, vp]
    L.fa_prefill_paged.restype = i32
    L.fa_decode_paged_fp8.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, f32, f32, f32, vp,
                                      vp, vp, ctypes.c_size_t, vp]
    L.fa_decode_paged_fp8.restype = i32
    L.fa_prefill_last_schedule.argtypes = []
    L.fa_prefill_last_schedule.restype = i32
    L.fa_debug_selftest_index.argtypes = [vp, i32, vp]
    L.fa_debug_selftest_index.restype = i32
    _lib = L
    return L


def select_library(variant: str) -> None:
    """"release" or "debug" (bounds-checked): the build later calls load.
    Plans made with one build must not be passed to the other."""
    global lib_path, _lib
    lib_path = {"release": release_lib_path, "debug": debug_lib_path}[variant]
    _lib = None


def debug_selftest_index(buf, stream=None) -> int:
    """Bounds-checked build only: a kernel writes buf[0] and then tries an
    index past half of buf, which its check must refuse (the refused index is
    still inside buf).  Returns the call's status (FA_ERR_UNSUPPORTED on the
    release build, which launches nothing)."""
    torch = _torch()
    _require_cuda(buf)
    if buf.dtype != torch.int32 or buf.numel() < 4:
        raise ValueError("buf must be an int32 CUDA tensor of at least 4 elements")
    return library().fa_debug_selftest_index(_ptr(buf), int(buf.numel()), _stream_ptr(stream))


def strerror(status: int) -> str:
    return library().fa_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("exact_attention_148_b200 runs on CUDA tensors only "
                             "(no CPU fallback)")


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _scale_arg(scale):
    return float("nan") if scale is None else float(scale)


# ----------------------------------------------------------------------------- prefill

def prefill(q, k, v, cu_seqlens, *, causal: bool = True, scale: float | None = None,
            out=None, lse=None, cu_seqlens_host=None, return_lse: bool = True, stream=None):
    """Exact attention over packed variable-length sequences.

    q [T, Hq, d], k/v [T, Hkv, d] bf16 CUDA tensors (contiguous); cu_seqlens
    [B+1] int32 CUDA tensor.  Returns (out [T, Hq, d] bf16, lse [T, Hq] fp32 or
    None).  ``cu_seqlens_host`` (a sequence of ints / numpy array) avoids a
    device-to-host copy of the offsets.
    """
    torch = _torch()
    _require_cuda(q, k, v, cu_seqlens, out, lse)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D bfloat16 tensor")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().numpy()
    cu_h = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
    batch = len(cu_h) - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    st = library().fa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                              cu_h.ctypes.data_as(ctypes.c_void_p), batch, Hq, Hkv, d,
                              1 if causal else 0, _scale_arg(scale), _ptr(out), _ptr(lse),
                              _stream_ptr(stream))
    _check(st, "fa_prefill")
    return out, lse


def prefill_last_schedule() -> str | None:
    """"persistent" or "grid": the schedule the calling thread's last prefill,
    prefill_fp8 or prefill_paged launched (None if that call failed or there
    was none)."""
    return {FA_SCHEDULE_GRID: "grid", FA_SCHEDULE_PERSISTENT: "persistent"}.get(
        library().fa_prefill_last_schedule())


def prefill_fp8(q, k, v, cu_seqlens, *, q_scale: float, k_scale: float, v_scale: float,
                causal: bool = True, scale: float | None = None, out=None, lse=None,
                cu_seqlens_host=None, return_lse: bool = True, stream=None):
    """``prefill`` over E4M3 inputs: q [T, Hq, 128], k/v [T, Hkv, 128] uint8
    (or float8_e4m3fn) tensors of E4M3 codes, dequantised as q_scale * q8,
    k_scale * k8 and v_scale * v8.  Returns (out [T, Hq, 128] bf16, lse fp32)."""
    torch = _torch()
    _require_cuda(q, k, v, cu_seqlens, out, lse)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.element_size() != 1 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D tensor of one-byte E4M3 codes")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().numpy()
    cu_h = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
    batch = len(cu_h) - 1
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    st = library().fa_prefill_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                  cu_h.ctypes.data_as(ctypes.c_void_p), batch, Hq, Hkv, d,
                                  1 if causal else 0, _scale_arg(scale), float(q_scale),
                                  float(k_scale), float(v_scale), _ptr(out), _ptr(lse),
                                  _stream_ptr(stream))
    _check(st, "fa_prefill_fp8")
    return out, lse


# ----------------------------------------------------------------------------- decode

@dataclass
class PlanInfo:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    max_pages_per_seq: int
    chunk_tokens: int
    max_splits: int
    heads_per_cta: int
    num_work_items: int
    max_seqlen: int
    workspace_bytes: int
    kv_dtype: int
    tensor_cores: int
    q_len: int


class DecodePlan:
    """Host-side split plan (owns an ``fa_plan``; freed with the object)."""

    def __init__(self, handle: ctypes.c_void_p, workspace_bytes: int):
        self._h = handle
        self.workspace_bytes = int(workspace_bytes)
        info = _PlanInfo()
        _check(library().fa_plan_get_info(self._h, ctypes.byref(info)), "fa_plan_get_info")
        self.info = PlanInfo(**{f: getattr(info, f) for f, _ in _PlanInfo._fields_})

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h is not None and self._h.value:
            library().fa_plan_free(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def decode_plan(cache_seqlens_host, *, num_q_heads: int, num_kv_heads: int, head_dim: int,
                page_size: int = 64, max_pages_per_seq: int, num_sms: int | None = None,
                num_splits: int = 0, kv_dtype: str = "bf16", kernel: str = "auto",
                q_len: int = 1) -> DecodePlan:
    """Plan the split of every request's cached context (host only, no GPU needed
    when ``num_sms`` is given).  ``kv_dtype``: "bf16" (for decode_paged) or
    "e4m3" (for decode_paged_fp8); ``kernel``: "auto", "cuda_cores" or
    "tensor_cores"; ``q_len`` > 1: multi-token decode (q [B, q_len, Hq, d])."""
    lens = np.ascontiguousarray(np.asarray(cache_seqlens_host, dtype=np.int32))
    if num_sms is None:
        torch = _torch()
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    opts = _DecodeOptions(_KV_DTYPES[kv_dtype], _KERNELS[kernel], int(q_len))
    st = library().fa_decode_plan_ex(lens.ctypes.data_as(ctypes.c_void_p), len(lens), num_q_heads,
                                     num_kv_heads, head_dim, page_size, max_pages_per_seq, num_sms,
                                     num_splits, ctypes.byref(opts), ctypes.byref(h), ctypes.byref(ws))
    _check(st, "fa_decode_plan_ex")
    return DecodePlan(h, ws.value)


def page_strides(k_pages, layout: str):
    """(page_stride, token_stride, head_stride) in elements for NHD / HND pools."""
    P, a, b, d = k_pages.shape
    if layout == "NHD":     # [P, page, Hkv, d]
        return a * b * d, b * d, d
    if layout == "HND":     # [P, Hkv, page, d]
        return a * b * d, d, b * d
    raise ValueError(layout)


def _check_q_rows(q, plan: DecodePlan):
    """q is [B, Hq, d], or [B, q_len, Hq, d] for a multi-token plan."""
    i = plan.info
    want = (i.batch, i.num_q_heads, i.head_dim) if i.q_len == 1 and q.dim() == 3 else \
        (i.batch, i.q_len, i.num_q_heads, i.head_dim)
    if tuple(q.shape) != want:
        raise ValueError(f"q has shape {tuple(q.shape)}, the plan expects {want}")


def decode_paged(q, k_pages, v_pages, block_table, cache_seqlens, plan: DecodePlan, *,
                 layout: str = "NHD", scale: float | None = None, out=None, lse=None,
                 workspace=None, return_lse: bool = True, stream=None):
    """One query token per request against a paged KV cache (Flash-Decoding).

    q [B, Hq, d] bf16; k_pages/v_pages [P, page, Hkv, d] (NHD) or
    [P, Hkv, page, d] (HND) bf16; block_table [B, max_pages] int32;
    cache_seqlens [B] int32 (device).  Returns (out, lse).
    """
    torch = _torch()
    _require_cuda(q, k_pages, v_pages, block_table, cache_seqlens, out, lse, workspace)
    if k_pages.dtype != torch.bfloat16 or v_pages.dtype != torch.bfloat16 or q.dtype != torch.bfloat16:
        raise ValueError("q, k_pages and v_pages must be bfloat16")
    if not (k_pages.is_contiguous() and v_pages.is_contiguous() and q.is_contiguous()
            and block_table.is_contiguous()):
        raise ValueError("tensors must be contiguous")
    if k_pages.shape != v_pages.shape:
        raise ValueError("k_pages and v_pages must have the same shape")
    _check_q_rows(q, plan)
    ps, ts, hs = page_strides(k_pages, layout)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if workspace is None and plan.workspace_bytes > 0:
        workspace = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=q.device)
    st = library().fa_decode_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], ps, ts, hs, _ptr(block_table),
        _ptr(cache_seqlens), plan.handle, _scale_arg(scale), _ptr(out), _ptr(lse), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(st, "fa_decode_paged")
    return out, lse


def decode_paged_fp8(q, k_pages, v_pages, block_table, cache_seqlens, plan: DecodePlan, *,
                     k_scale: float, v_scale: float, layout: str = "NHD",
                     scale: float | None = None, out=None, lse=None, workspace=None,
                     return_lse: bool = True, stream=None):
    """``decode_paged`` over an FP8 E4M3 cache: k_pages / v_pages are uint8
    (or float8_e4m3fn) tensors of E4M3 codes, dequantised as k_scale * k8 and
    v_scale * v8.  Returns (out bf16, lse fp32)."""
    torch = _torch()
    _require_cuda(q, k_pages, v_pages, block_table, cache_seqlens, out, lse, workspace)
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bfloat16")
    if k_pages.element_size() != 1 or v_pages.element_size() != 1:
        raise ValueError("k_pages and v_pages must hold one-byte E4M3 codes")
    if not (k_pages.is_contiguous() and v_pages.is_contiguous() and q.is_contiguous()
            and block_table.is_contiguous()):
        raise ValueError("tensors must be contiguous")
    if k_pages.shape != v_pages.shape:
        raise ValueError("k_pages and v_pages must have the same shape")
    _check_q_rows(q, plan)
    ps, ts, hs = page_strides(k_pages, layout)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if workspace is None and plan.workspace_bytes > 0:
        workspace = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=q.device)
    st = library().fa_decode_paged_fp8(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], ps, ts, hs, _ptr(block_table),
        _ptr(cache_seqlens), plan.handle, _scale_arg(scale), float(k_scale), float(v_scale),
        _ptr(out), _ptr(lse), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(st, "fa_decode_paged_fp8")
    return out, lse


def decode_paged_static(q, k_pages, v_pages, block_table, cache_seqlens, plan: DecodePlan, *,
                        layout: str = "NHD", scale: float | None = None, out=None, lse=None,
                        return_lse: bool = True, stream=None):
    """``decode_paged`` without a workspace, for callers that cannot allocate
    device memory: the split partials use the library's static 16 MiB device
    scratch (``STATIC_SCRATCH_BYTES``), shared by every call on a device, so
    calls that overlap on the GPU race and must be ordered by the caller.
    Pass preallocated ``out`` (and ``lse``) to keep the call allocation-free."""
    torch = _torch()
    _require_cuda(q, k_pages, v_pages, block_table, cache_seqlens, out, lse)
    _check_q_rows(q, plan)
    ps, ts, hs = page_strides(k_pages, layout)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    st = library().fa_decode_paged_static(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], ps, ts, hs, _ptr(block_table),
        _ptr(cache_seqlens), plan.handle, _scale_arg(scale), _ptr(out), _ptr(lse), _stream_ptr(stream))
    _check(st, "fa_decode_paged_static")
    return out, lse


def _check_pool(k_pages, v_pages, block_table):
    torch = _torch()
    if k_pages.dtype != torch.bfloat16 or v_pages.dtype != torch.bfloat16:
        raise ValueError("k_pages and v_pages must be bfloat16")
    if not (k_pages.is_contiguous() and v_pages.is_contiguous() and block_table.is_contiguous()):
        raise ValueError("k_pages, v_pages and block_table must be contiguous")
    if k_pages.shape != v_pages.shape or k_pages.dim() != 4:
        raise ValueError("k_pages and v_pages must be 4-D with the same shape")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise ValueError("block_table must be a 2-D int32 tensor")


def append_kv(k_new, v_new, cu_seqlens_new, k_pages, v_pages, block_table, cache_seqlens, *,
              layout: str = "NHD", stream=None):
    """Write new K/V rows into the paged cache (in place).

    k_new/v_new [T_new, Hkv, d] bf16 packed by cu_seqlens_new [B+1] int32;
    cache_seqlens [B] int32 are the lengths after the append: request b's new
    rows go to logical positions cache_seqlens[b] - n_b ... cache_seqlens[b] - 1.
    """
    torch = _torch()
    _require_cuda(k_new, v_new, cu_seqlens_new, k_pages, v_pages, block_table, cache_seqlens)
    _check_pool(k_pages, v_pages, block_table)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D bfloat16 tensor")
    if k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new must have the same shape")
    if cu_seqlens_new.dtype != torch.int32 or cache_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens_new and cache_seqlens must be int32")
    T, Hkv, d = k_new.shape
    ps, ts, hs = page_strides(k_pages, layout)
    page_size = k_pages.shape[1] if layout == "NHD" else k_pages.shape[2]
    st = library().fa_append_kv(
        _ptr(k_new), _ptr(v_new), _ptr(cu_seqlens_new), T, cu_seqlens_new.numel() - 1, Hkv, d,
        _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], ps, ts, hs, page_size, _ptr(block_table),
        block_table.shape[1], _ptr(cache_seqlens), _stream_ptr(stream))
    _check(st, "fa_append_kv")


def prefill_paged(q, cu_seqlens_q, k_pages, v_pages, block_table, cache_seqlens, *,
                  causal: bool = True, scale: float | None = None, layout: str = "NHD",
                  out=None, lse=None, cu_seqlens_q_host=None, cache_seqlens_host=None,
                  return_lse: bool = True, stream=None):
    """Chunked prefill: new queries [Tq, Hq, d] (packed by cu_seqlens_q) against
    each request's whole paged cache of cache_seqlens[b] keys; causal queries
    are the last q_len positions of their sequence.  Returns (out, lse)."""
    torch = _torch()
    _require_cuda(q, cu_seqlens_q, k_pages, v_pages, block_table, cache_seqlens, out, lse)
    _check_pool(k_pages, v_pages, block_table)
    if q.dtype != torch.bfloat16 or not q.is_contiguous() or q.dim() != 3:
        raise ValueError("q must be a contiguous 3-D bfloat16 tensor")
    if cu_seqlens_q.dtype != torch.int32 or cache_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens_q and cache_seqlens must be int32")
    T, Hq, d = q.shape
    Hkv = k_pages.shape[2] if layout == "NHD" else k_pages.shape[1]
    page_size = k_pages.shape[1] if layout == "NHD" else k_pages.shape[2]
    if cu_seqlens_q_host is None:
        cu_seqlens_q_host = cu_seqlens_q.cpu().numpy()
    if cache_seqlens_host is None:
        cache_seqlens_host = cache_seqlens.cpu().numpy()
    cu_h = np.ascontiguousarray(np.asarray(cu_seqlens_q_host, dtype=np.int32))
    len_h = np.ascontiguousarray(np.asarray(cache_seqlens_host, dtype=np.int32))
    batch = len(cu_h) - 1
    if len(len_h) != batch:
        raise ValueError("cache_seqlens must have one entry per request")
    ps, ts, hs = page_strides(k_pages, layout)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    st = library().fa_prefill_paged(
        _ptr(q), _ptr(cu_seqlens_q), cu_h.ctypes.data_as(ctypes.c_void_p), _ptr(k_pages),
        _ptr(v_pages), k_pages.shape[0], ps, ts, hs, _ptr(block_table), block_table.shape[1],
        _ptr(cache_seqlens), len_h.ctypes.data_as(ctypes.c_void_p), batch, Hq, Hkv, d, page_size,
        1 if causal else 0, _scale_arg(scale), _ptr(out), _ptr(lse), _stream_ptr(stream))
    _check(st, "fa_prefill_paged")
    return out, lse


def cascade_workspace_bytes(plan: DecodePlan, prefix_len: int) -> int:
    n = ctypes.c_size_t()
    _check(library().fa_cascade_workspace_bytes(plan.handle, int(prefix_len), ctypes.byref(n)),
           "fa_cascade_workspace_bytes")
    return n.value


def cascade_decode(q, k_pages, v_pages, prefix_block_table, prefix_len: int, block_table,
                   cache_seqlens, plan: DecodePlan, *, layout: str = "NHD",
                   scale: float | None = None, out=None, lse=None, workspace=None,
                   return_lse: bool = True, stream=None):
    """Decode where every request's context is a shared prefix (prefix_len
    tokens in the pages of prefix_block_table) followed by its own suffix
    (cache_seqlens[b] tokens through block_table[b]).  ``plan`` is a bf16 plan
    for the suffix lengths.  Returns (out, lse)."""
    torch = _torch()
    _require_cuda(q, k_pages, v_pages, prefix_block_table, block_table, cache_seqlens, out, lse,
                  workspace)
    _check_pool(k_pages, v_pages, block_table)
    _check_q_rows(q, plan)
    ps, ts, hs = page_strides(k_pages, layout)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    need = cascade_workspace_bytes(plan, prefix_len)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = library().fa_cascade_decode(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], ps, ts, hs, _ptr(prefix_block_table),
        int(prefix_len), _ptr(block_table), _ptr(cache_seqlens), plan.handle, _scale_arg(scale),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream))
    _check(st, "fa_cascade_decode")
    return out, lse


def merge_states(o_parts, lse_parts, *, out=None, lse=None, stream=None):
    """Merge states by LSE.  o_parts [S, rows, H, d] fp32, lse_parts [S, rows, H] fp32."""
    torch = _torch()
    _require_cuda(o_parts, lse_parts, out, lse)
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise ValueError("o_parts and lse_parts must be float32")
    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("o_parts and lse_parts must be contiguous")
    S, R, H, d = o_parts.shape
    if out is None:
        out = torch.empty((R, H, d), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((R, H), dtype=torch.float32, device=o_parts.device)
    st = library().fa_merge_states(_ptr(o_parts), _ptr(lse_parts), S, R, H, d, _ptr(out), _ptr(lse),
                                   _stream_ptr(stream))
    _check(st, "fa_merge_states")
    return out, lse


def device_status(clear: bool = True, stream=None) -> int:
    """Synchronise and return (optionally clear) the device status word."""
    v = ctypes.c_int(0)
    _check(library().fa_get_device_status(_stream_ptr(stream), ctypes.byref(v), 1 if clear else 0),
           "fa_get_device_status")
    return v.value


def selftest_wait_timeout(limit_us: int = 20000, stream=None) -> int:
    """Run the bounded-wait self-test kernel and return the device status it
    leaves (FA_ERR_TIMEOUT when the failure path works); clears the status."""
    _check(library().fa_selftest_wait_timeout(int(limit_us), _stream_ptr(stream)),
           "fa_selftest_wait_timeout")
    return device_status(clear=True, stream=stream)


def version() -> int:
    return library().fa_version()
