"""Host-side checks of the C ABI library (no GPU needed).

The library must load, export every function include/exact_attention.h
declares, and its host-only parts (planner, argument validation that fails
before any CUDA call) must behave as documented.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import exact_attention_148_b200 as fa
from exact_attention_148_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "exact_attention.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return fa.library()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_api():
    fns = header_functions()
    for name in ["fa_prefill", "fa_decode_plan", "fa_decode_paged", "fa_merge_states",
                 "fa_plan_free", "fa_strerror", "fa_get_device_status"]:
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), f"{name} declared in the header but not exported"
    assert sorted(header_functions()) == sorted(fa.EXPORTED_SYMBOLS)


def test_only_api_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", fa.lib_path], capture_output=True, text=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if " T " in line}
    fa_names = {n for n in names if n.startswith("fa_")}
    assert fa_names == set(header_functions())


def test_bounds_checked_build_exports_the_same_symbols():
    import subprocess
    path = _build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {n for n in names if n.startswith("fa_")} == set(header_functions())


def test_release_build_refuses_the_index_selftest(lib):
    # no CUDA call is made: the release build returns before any launch
    fake = ctypes.c_void_p(0x10000)
    assert lib.fa_debug_selftest_index(fake, 16, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_debug_selftest_index(fake, 2, None) == fa.FA_ERR_INVALID_ARG
    assert fa.strerror(fa.FA_ERR_DEBUG_INDEX).startswith("index outside")


def test_version_and_strerror(lib):
    assert fa.version() == 100
    assert fa.strerror(0) == "ok"
    assert "workspace" in fa.strerror(-3)
    assert fa.strerror(12345) == "unknown status"


def _plan(lens, hq=32, hkv=8, d=128, max_pages=None, num_sms=148, splits=0, kv_dtype="bf16",
          kernel="auto"):
    lens = np.asarray(lens, dtype=np.int32)
    if max_pages is None:
        max_pages = max(1, int(np.max((lens + 63) // 64)))
    return fa.decode_plan(lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                          max_pages_per_seq=max_pages, num_sms=num_sms, num_splits=splits,
                          kv_dtype=kv_dtype, kernel=kernel)


def _splits(L, chunk):
    return max(1, -(-int(L) // chunk))


@pytest.mark.parametrize("lens", [[1024, 32768, 5000, 64], [131072] * 4, [131072] + [2048] * 63,
                                  [0, 0, 7], [1], list(range(1, 300, 7))])
def test_plan_covers_every_key_once(lib, lens):
    p = _plan(lens)
    info = p.info
    assert info.chunk_tokens % 64 == 0 and info.chunk_tokens >= 64
    assert info.max_splits == max(1, max(_splits(L, info.chunk_tokens) for L in lens))
    for L in lens:
        # splits [s*chunk, min(L, (s+1)*chunk)) tile [0, L) exactly, no overlap
        n = _splits(L, info.chunk_tokens)
        covered = []
        for s in range(n):
            lo, hi = s * info.chunk_tokens, min(L, (s + 1) * info.chunk_tokens)
            assert lo < hi or L == 0
            covered.extend(range(lo, hi))
        assert covered == list(range(L))
    units = info.num_kv_heads * (info.num_q_heads // info.num_kv_heads // info.heads_per_cta)
    assert info.num_work_items == units * sum(_splits(L, info.chunk_tokens) for L in lens)


def test_plan_workspace_size(lib):
    p = _plan([131072] * 4, hq=32, hkv=32, splits=16)
    i = p.info
    assert i.max_splits == 16
    rows = 4 * 32
    o_bytes = 16 * rows * 128 * 4
    lse_bytes = 16 * rows * 4
    assert p.workspace_bytes >= o_bytes + lse_bytes
    assert p.workspace_bytes % 256 == 0
    assert p.workspace_bytes < o_bytes + lse_bytes + 512
    # no split -> no workspace
    q = _plan([100, 200], splits=1)
    assert q.info.max_splits == 1 and q.workspace_bytes == 0


@pytest.mark.parametrize("s", [1, 2, 3, 4, 7, 8, 16, 32, 64])
def test_plan_override_caps_splits(lib, s):
    p = _plan([131072] * 4, hq=32, hkv=32, splits=s)
    assert p.info.max_splits <= s
    if 2048 % s == 0:
        assert p.info.max_splits == s


def test_plan_is_deterministic(lib):
    lens = np.random.default_rng(3).integers(1024, 32769, size=64)
    a = _plan(lens).info
    b = _plan(lens).info
    assert a == b


def test_plan_heads_per_cta(lib):
    cc = dict(kernel="cuda_cores")
    assert _plan([100], hq=32, hkv=8).info.heads_per_cta == 4
    assert _plan([100], hq=32, hkv=32).info.heads_per_cta == 1
    assert _plan([100], hq=32, hkv=2, **cc).info.heads_per_cta == 8     # 16 per kv head -> 2 CTAs
    assert _plan([100], hq=12, hkv=4).info.heads_per_cta == 1     # group 3
    assert _plan([100], hq=12, hkv=2, **cc).info.heads_per_cta == 2     # group 6
    assert _plan([100], hq=12, hkv=2).info.heads_per_cta == 6     # tensor cores: whole group


def test_plan_kernel_choice(lib):
    """Tensor cores for an E4M3 cache or a group of 4..16 heads at d = 128."""
    p = _plan([100], hq=32, hkv=8)
    assert p.info.tensor_cores == 1 and p.info.kv_dtype == fa.FA_KV_BF16
    assert _plan([100], hq=32, hkv=16).info.tensor_cores == 0               # group 2
    assert _plan([100], hq=32, hkv=32).info.tensor_cores == 0               # group 1
    p = _plan([100], hq=32, hkv=8, kv_dtype="e4m3")
    assert p.info.tensor_cores == 1 and p.info.kv_dtype == fa.FA_KV_E4M3 and p.info.heads_per_cta == 4
    p = _plan([100], hq=32, hkv=2)
    assert p.info.tensor_cores == 1 and p.info.heads_per_cta == 16
    assert _plan([100], hq=64, hkv=2).info.tensor_cores == 0                 # group 32
    assert _plan([100], hq=16, hkv=2, d=64).info.tensor_cores == 0           # d = 64
    assert _plan([100], hq=32, hkv=16, kernel="tensor_cores").info.tensor_cores == 1
    assert _plan([100], hq=32, hkv=8, kv_dtype="e4m3", kernel="cuda_cores").info.tensor_cores == 0
    with pytest.raises(fa.FAError) as e:
        _plan([100], hq=64, hkv=2, kernel="tensor_cores")
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_plan_dtype_must_match_entry_point(lib):
    A = 0x10000
    p = _plan([1000, 3000], hq=8, hkv=2, kv_dtype="bf16")
    st = lib.fa_decode_paged_fp8(_fake(A), _fake(A), _fake(A), 100, 64 * 2 * 128, 2 * 128, 128,
                                 _fake(A), _fake(A), p.handle, float("nan"), 1.0, 1.0, _fake(A), None,
                                 _fake(A), p.workspace_bytes, None)
    assert st == fa.FA_ERR_PLAN_MISMATCH
    p8 = _plan([1000, 3000], hq=8, hkv=2, kv_dtype="e4m3")
    st = lib.fa_decode_paged(_fake(A), _fake(A), _fake(A), 100, 64 * 2 * 128, 2 * 128, 128,
                             _fake(A), _fake(A), p8.handle, float("nan"), _fake(A), None,
                             _fake(A), p8.workspace_bytes, None)
    assert st == fa.FA_ERR_PLAN_MISMATCH


def test_plan_rejects_cache_overflow(lib):
    with pytest.raises(fa.FAError) as e:
        _plan([65], max_pages=1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FAError):
        _plan([-1], max_pages=1)


@pytest.mark.parametrize("kw,status", [
    (dict(hq=30, hkv=8), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(num_sms=0), fa.FA_ERR_INVALID_ARG),
])
def test_plan_rejects_bad_shapes(lib, kw, status):
    with pytest.raises(fa.FAError) as e:
        _plan([100], **kw)
    assert e.value.status == status


def test_plan_rejects_other_page_sizes(lib):
    lens = np.array([100], dtype=np.int32)
    with pytest.raises(fa.FAError) as e:
        fa.decode_plan(lens, num_q_heads=4, num_kv_heads=4, head_dim=128, page_size=16,
                       max_pages_per_seq=8, num_sms=148)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_prefill_fp8_validation_before_any_cuda_call(lib):
    cu = np.array([0, 128], dtype=np.int32)
    cuh = cu.ctypes.data_as(ctypes.c_void_p)
    A = 0x10000   # never dereferenced: validation fails first
    call = lambda q=A, d=128, qs=1.0, ks=1.0, vs=1.0, cuh=cuh: lib.fa_prefill_fp8(
        _fake(q), _fake(A), _fake(A), _fake(A), cuh, 1, 4, 2, d, 1, float("nan"), qs, ks, vs,
        _fake(A), None, None)
    assert call(q=0) == fa.FA_ERR_INVALID_ARG
    assert call(d=64) == fa.FA_ERR_UNSUPPORTED                      # E4M3 inputs: d = 128 only
    for bad_scale in (0.0, -1.0, float("nan"), float("inf")):
        assert call(qs=bad_scale) == fa.FA_ERR_INVALID_ARG
        assert call(ks=bad_scale) == fa.FA_ERR_INVALID_ARG
        assert call(vs=bad_scale) == fa.FA_ERR_INVALID_ARG
    assert call(q=A + 8) == fa.FA_ERR_INVALID_ARG                   # 16-byte alignment
    bad = np.array([0, 0], dtype=np.int32)
    assert call(cuh=bad.ctypes.data_as(ctypes.c_void_p)) == fa.FA_ERR_INVALID_ARG


def test_prefill_validation_before_any_cuda_call(lib):
    cu = np.array([0, 128], dtype=np.int32)
    cuh = cu.ctypes.data_as(ctypes.c_void_p)
    A = 0x10000   # never dereferenced: validation fails first
    call = lambda q=A, hq=4, hkv=4, d=128, scale=float("nan"), cuh=cuh, out=A, k=A: lib.fa_prefill(
        _fake(q), _fake(k), _fake(A), _fake(A), cuh, 1, hq, hkv, d, 1, scale, _fake(out), None, None)
    assert call(q=0) == fa.FA_ERR_INVALID_ARG
    assert call(q=A + 2) == fa.FA_ERR_INVALID_ARG                 # misaligned
    assert call(hq=6, hkv=4) == fa.FA_ERR_INVALID_ARG              # Hq % Hkv
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert call(scale=float("inf")) == fa.FA_ERR_INVALID_ARG
    bad = np.array([0, 0], dtype=np.int32)                          # empty sequence
    assert call(cuh=bad.ctypes.data_as(ctypes.c_void_p)) == fa.FA_ERR_INVALID_ARG
    bad2 = np.array([5, 10], dtype=np.int32)                        # must start at 0
    assert call(cuh=bad2.ctypes.data_as(ctypes.c_void_p)) == fa.FA_ERR_INVALID_ARG
    # T * Hq * d must stay below 2^40: two 2^22-token sequences, 1024 heads, d = 128
    big = np.array([0, 1 << 22, 1 << 23], dtype=np.int32)
    big_call = lambda hq: lib.fa_prefill(_fake(A), _fake(A), _fake(A), _fake(A),
                                         big.ctypes.data_as(ctypes.c_void_p), 2, hq, hq, 128, 1,
                                         float("nan"), _fake(A), None, None)
    assert big_call(1024) == fa.FA_ERR_UNSUPPORTED


def test_decode_validation_before_any_cuda_call(lib):
    p = _plan([1000, 3000], hq=8, hkv=2, splits=4)
    assert p.workspace_bytes > 0
    A = 0x10000
    def call(ws=A, ws_bytes=None, q=A, strides=(64 * 2 * 128, 2 * 128, 128), npages=100, plan=p.handle):
        return lib.fa_decode_paged(_fake(q), _fake(A), _fake(A), npages, *strides, _fake(A), _fake(A),
                                   plan, float("nan"), _fake(A), None, _fake(ws),
                                   p.workspace_bytes if ws_bytes is None else ws_bytes, None)
    assert call(ws_bytes=p.workspace_bytes - 1) == fa.FA_ERR_WORKSPACE
    assert call(ws=0) == fa.FA_ERR_INVALID_ARG
    assert call(ws=A + 16) == fa.FA_ERR_INVALID_ARG                  # workspace not 256-aligned
    assert call(q=A + 8) == fa.FA_ERR_INVALID_ARG
    assert call(strides=(64 * 2 * 128, 2 * 128, 100)) == fa.FA_ERR_INVALID_ARG
    assert call(npages=0) == fa.FA_ERR_INVALID_ARG
    assert call(plan=None) == fa.FA_ERR_INVALID_ARG


def test_merge_validation_before_any_cuda_call(lib):
    A = 0x10000
    f = lambda S=2, d=128, o=A: lib.fa_merge_states(_fake(o), _fake(A), S, 4, 2, d, _fake(A), None, None)
    assert f(S=0) == fa.FA_ERR_INVALID_ARG
    assert f(d=32) == fa.FA_ERR_UNSUPPORTED
    assert f(o=A + 4) == fa.FA_ERR_INVALID_ARG


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(128, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 128], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        fa.prefill(q, q, q, cu)


def test_prefill_paged_validation_before_any_cuda_call(lib):
    cu = np.array([0, 100, 300], dtype=np.int32)
    lens = np.array([150, 200], dtype=np.int32)
    A = 0x10000
    strides = (64 * 2 * 128, 2 * 128, 128)

    def call(q=A, cu=cu, lens=lens, hq=4, hkv=2, d=128, ps=64, max_pages=4, npages=10,
             strides=strides, scale=float("nan"), bt=A):
        return lib.fa_prefill_paged(
            _fake(q), _fake(A), cu.ctypes.data_as(ctypes.c_void_p), _fake(A), _fake(A), npages,
            *strides, _fake(bt), max_pages, _fake(A), lens.ctypes.data_as(ctypes.c_void_p),
            len(cu) - 1, hq, hkv, d, ps, 1, scale, _fake(A), None, None)
    assert call(q=0) == fa.FA_ERR_INVALID_ARG
    assert call(bt=0) == fa.FA_ERR_INVALID_ARG
    assert call(q=A + 2) == fa.FA_ERR_INVALID_ARG
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(ps=16) == fa.FA_ERR_UNSUPPORTED
    assert call(hq=6, hkv=4) == fa.FA_ERR_INVALID_ARG
    assert call(npages=0) == fa.FA_ERR_INVALID_ARG
    assert call(strides=(64 * 2 * 128, 2 * 128, 100)) == fa.FA_ERR_INVALID_ARG
    assert call(scale=-2.0) == fa.FA_ERR_INVALID_ARG
    # cache shorter than the chunk, and a cache past the table's capacity
    assert call(lens=np.array([99, 200], dtype=np.int32)) == fa.FA_ERR_INVALID_ARG
    assert call(max_pages=3) == fa.FA_ERR_INVALID_ARG               # 200 > 3 * 64
    assert call(max_pages=(1 << 24) + 1) == fa.FA_ERR_INVALID_ARG   # capacity past 2^30 keys
    assert call(cu=np.array([0, 0, 300], dtype=np.int32)) == fa.FA_ERR_INVALID_ARG


def test_append_validation_before_any_cuda_call(lib):
    A = 0x10000
    strides = (64 * 2 * 128, 2 * 128, 128)

    def call(k=A, total=10, d=128, ps=64, npages=10, strides=strides, bt=A, kp=A):
        return lib.fa_append_kv(_fake(k), _fake(A), _fake(A), total, 2, 2, d, _fake(kp), _fake(A),
                                npages, *strides, ps, _fake(bt), 4, _fake(A), None)
    assert call(k=0) == fa.FA_ERR_INVALID_ARG
    assert call(kp=0) == fa.FA_ERR_INVALID_ARG
    assert call(k=A + 8) == fa.FA_ERR_INVALID_ARG
    assert call(total=-1) == fa.FA_ERR_INVALID_ARG
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(ps=32) == fa.FA_ERR_UNSUPPORTED
    assert call(npages=0) == fa.FA_ERR_INVALID_ARG
    assert call(strides=(64 * 2 * 128, 2 * 128, 12)) == fa.FA_ERR_INVALID_ARG
    assert call(total=0) == fa.FA_OK                                 # nothing to enqueue


def test_decode_fp8_validation_before_any_cuda_call(lib):
    p = _plan([1000, 3000], hq=8, hkv=2, splits=4, kv_dtype="e4m3")
    A = 0x10000

    def call(strides=(64 * 2 * 128, 2 * 128, 128), ks=0.5, vs=0.5):
        return lib.fa_decode_paged_fp8(_fake(A), _fake(A), _fake(A), 100, *strides, _fake(A),
                                       _fake(A), p.handle, float("nan"), ks, vs, _fake(A), None,
                                       _fake(A), p.workspace_bytes, None)
    assert call(ks=0.0) == fa.FA_ERR_INVALID_ARG
    assert call(vs=-1.0) == fa.FA_ERR_INVALID_ARG
    assert call(ks=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert call(vs=float("nan")) == fa.FA_ERR_INVALID_ARG
    # byte strides must be multiples of 16 (8 is fine for bf16 elements, not for bytes)
    assert call(strides=(64 * 2 * 128, 2 * 128, 8)) == fa.FA_ERR_INVALID_ARG


def test_build_tracks_every_source_file():
    """Every file under csrc/ is a build input, so editing any of them rebuilds."""
    csrc = os.path.join(ROOT, "exact_attention_148_b200", "csrc")
    assert sorted(os.listdir(csrc)) == sorted(_build.SOURCES + _build.HEADERS)


def test_multi_token_plans(lib):
    mk = lambda **kw: fa.decode_plan(np.array([100, 2000], dtype=np.int32), num_q_heads=kw.get("hq", 8),
                                     num_kv_heads=kw.get("hkv", 2), head_dim=kw.get("d", 128),
                                     max_pages_per_seq=40, num_sms=148, num_splits=kw.get("s", 0),
                                     q_len=kw.get("q_len", 1), kernel=kw.get("kernel", "auto"),
                                     kv_dtype=kw.get("kv", "bf16"))
    p = mk(q_len=4)
    assert p.info.q_len == 4 and p.info.tensor_cores == 1
    p1 = mk(q_len=1, s=4, kernel="tensor_cores")
    p4 = mk(q_len=4, s=4)
    assert p4.workspace_bytes >= 4 * p1.workspace_bytes - 1024            # partials scale with q_len
    assert mk(q_len=4, kv="e4m3").info.tensor_cores == 1
    for kw, status in [(dict(q_len=3, hq=16, hkv=2), fa.FA_ERR_UNSUPPORTED),   # 24 rows > 16
                       (dict(q_len=2, d=64), fa.FA_ERR_UNSUPPORTED),
                       (dict(q_len=2, kernel="cuda_cores"), fa.FA_ERR_UNSUPPORTED),
                       (dict(q_len=0), fa.FA_ERR_INVALID_ARG),
                       (dict(q_len=17), fa.FA_ERR_INVALID_ARG)]:
        with pytest.raises(fa.FAError) as e:
            mk(**kw)
        assert e.value.status == status, kw
    with pytest.raises(fa.FAError) as e:      # a cache shorter than the chunk
        fa.decode_plan(np.array([3, 2000], dtype=np.int32), num_q_heads=8, num_kv_heads=2,
                       head_dim=128, max_pages_per_seq=40, num_sms=148, q_len=4)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


def test_cascade_validation_before_any_cuda_call(lib):
    A = 0x10000
    p = _plan([100, 2000], hq=8, hkv=2)
    n = ctypes.c_size_t()
    assert lib.fa_cascade_workspace_bytes(p.handle, 1000, ctypes.byref(n)) == fa.FA_OK
    n0 = ctypes.c_size_t()
    assert lib.fa_cascade_workspace_bytes(p.handle, 0, ctypes.byref(n0)) == fa.FA_OK
    assert n.value > n0.value >= p.workspace_bytes
    assert lib.fa_cascade_workspace_bytes(p.handle, -1, ctypes.byref(n)) == fa.FA_ERR_INVALID_ARG

    def call(plan=p.handle, ws_bytes=None, prefix=1000, pre=A, ws=A):
        return lib.fa_cascade_decode(_fake(A), _fake(A), _fake(A), 100, 64 * 2 * 128, 2 * 128, 128,
                                     _fake(pre), prefix, _fake(A), _fake(A), plan, float("nan"),
                                     _fake(A), None, _fake(ws), n.value if ws_bytes is None else ws_bytes,
                                     None)
    n.value = 0
    lib.fa_cascade_workspace_bytes(p.handle, 1000, ctypes.byref(n))
    assert call(ws_bytes=n.value - 256) == fa.FA_ERR_WORKSPACE
    assert call(pre=0) == fa.FA_ERR_INVALID_ARG
    assert call(ws=A + 16) == fa.FA_ERR_INVALID_ARG
    p8 = _plan([100, 2000], hq=8, hkv=2, kv_dtype="e4m3")
    assert call(plan=p8.handle) == fa.FA_ERR_PLAN_MISMATCH


def _batch64():
    # the paged decode batch's lengths (workloads.paged_decode_batch and its variants)
    return np.random.default_rng(3).integers(1024, 32768 + 1, size=64)


@pytest.mark.parametrize("name,lens,hq,hkv,q_len,kv,chunk,splits,tensor_cores", [
    ("paged_decode_batch", _batch64(), 32, 8, 1, "bf16", 3200, 10, 1),
    ("ragged_split_decode", [131072] + [2048] * 63, 32, 32, 1, "bf16", 16384, 8, 0),
    ("long_split_decode", [131072] * 4, 32, 32, 1, "bf16", 65536, 2, 0),
    ("paged_decode_gqa8", _batch64(), 64, 8, 1, "bf16", 3200, 10, 1),
    ("paged_decode_gqa16", _batch64(), 32, 2, 1, "bf16", 5376, 6, 1),
    ("paged_decode_batch_fp8", _batch64(), 32, 8, 1, "e4m3", 4032, 8, 1),
    ("speculative_decode_batch", _batch64(), 32, 8, 4, "bf16", 10688, 3, 1),
])
def test_planner_choices_for_the_benchmark_batches(name, lens, hq, hkv, q_len, kv, chunk, splits, tensor_cores):
    """The automatic plans the measured decode numbers were taken with (148
    SMs): a change to the planner's search or model that moves one of them
    shows up here, to be measured again."""
    lens = np.asarray(lens, dtype=np.int32)
    p = fa.decode_plan(lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                       max_pages_per_seq=int(((lens + 63) // 64).max()), num_sms=148, kv_dtype=kv, q_len=q_len)
    assert (p.info.chunk_tokens, p.info.max_splits, p.info.tensor_cores) == (chunk, splits, tensor_cores), name


def _random_lengths(rng):
    kind = rng.integers(0, 4)
    B = int(rng.integers(1, 257))
    if kind == 0:      # uniform over a wide range
        return rng.integers(0, 1 << 17, size=B)
    if kind == 1:      # a few long requests among short ones
        lens = rng.integers(1, 4096, size=B)
        lens[rng.integers(0, B, size=max(1, B // 16))] = rng.integers(1 << 16, 1 << 20)
        return lens
    if kind == 2:      # page multiples and their neighbours
        return np.clip(64 * rng.integers(0, 600, size=B) + rng.integers(-1, 2, size=B), 0, None)
    return rng.integers(0, 600, size=B)   # all within the minimum chunk


def test_plan_invariants_on_random_batches(lib):
    """Seeded batch mixes (lengths 0 to 2^20, 1-256 requests, every head
    group, both cache types, 1-4 query tokens, automatic and forced splits):
    the plan tiles every request's keys in page-multiple chunks within the
    split limit, sizes the workspace for its splits, and picks the kernel by
    the documented rule."""
    rng = np.random.default_rng(2024)
    for case in range(300):
        lens = _random_lengths(rng).astype(np.int32)
        hkv = int(rng.choice([1, 2, 4, 8]))
        G = int(rng.choice([1, 2, 3, 4, 8, 16]))
        d = int(rng.choice([64, 128]))
        kv = "e4m3" if rng.random() < 0.3 else "bf16"
        q_len = int(rng.choice([1, 1, 2, 4])) if d == 128 and G <= 8 else 1
        if q_len * G > 16:
            q_len = 1
        L = int(lens.max())
        splits = 0 if rng.random() < 0.6 else int(rng.integers(1, 200))
        max_pages = max(1, (L + 63) // 64)
        if q_len > 1:
            lens = np.maximum(lens, q_len).astype(np.int32)
            L = int(lens.max())
            max_pages = max(1, (L + 63) // 64)
        p = fa.decode_plan(lens, num_q_heads=G * hkv, num_kv_heads=hkv, head_dim=d,
                           max_pages_per_seq=max_pages, num_sms=148, num_splits=splits,
                           kv_dtype=kv, q_len=q_len)
        i = p.info
        where = f"case {case}: B={len(lens)} max={L} G={G} d={d} {kv} q_len={q_len} splits={splits}"
        chunk = i.chunk_tokens
        assert chunk % 64 == 0 and chunk >= 64, where
        assert 1 <= i.max_splits <= 128, where
        assert i.max_splits == max(_splits(x, chunk) for x in lens), where
        if splits:
            assert i.max_splits <= splits, where
        elif L > 512:
            assert chunk >= min(512, L) or i.max_splits == 128, where
        tc_ok = d == 128 and q_len * G <= 16
        assert bool(i.tensor_cores) == (q_len > 1 or (tc_ok and (kv == "e4m3" or G >= 4))), where
        hpc = G if i.tensor_cores else next(g for g in (8, 4, 2, 1) if G % g == 0)
        assert i.heads_per_cta == hpc, where
        units = hkv * (G // hpc)
        assert i.num_work_items == units * sum(_splits(x, chunk) for x in lens), where
        if i.max_splits == 1:
            assert p.workspace_bytes == 0, where
        else:
            rows = len(lens) * q_len * G * hkv
            need = i.max_splits * rows * (d * 4 + 4)
            assert need <= p.workspace_bytes < need + 512 and p.workspace_bytes % 256 == 0, where
