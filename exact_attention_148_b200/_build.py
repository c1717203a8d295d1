"""Build the in-tree shared library ``libexact_attention.so`` for sm_100a.

Run ``python -m exact_attention_148_b200._build`` (or ``__graft_entry__.build()``);
``--debug`` builds the bounds-checked variant ``libexact_attention_debug.so``
(compiled with FA_DEBUG: every global index a kernel computes is checked
against its buffer before the access).  nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it has no link-time dependency on libcuda.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_NAME = "libexact_attention.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libexact_attention_debug.so")

SOURCES = ["fa_api.cu", "planner.cpp"]
HEADERS = ["ptx_sm100.cuh", "prefill_pp_sm100.cuh", "decode_sm100.cuh", "decode_tc_sm100.cuh",
           "append_sm100.cuh", "prefill_persist_sm100.cuh", "planner.h"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_input_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    paths.append(os.path.join(ROOT, "include", "exact_attention.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths)


def needs_build(debug: bool = False) -> bool:
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    return not os.path.exists(path) or os.path.getmtime(path) < _newest_input_mtime()


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug: bool = False) -> str:
    out = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not needs_build(debug):
        return out
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-std=c++17", "-lineinfo",
        "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"),
        "-o", out + ".tmp",
    ]
    if debug:
        cmd += ["-DFA_DEBUG=1"]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    cmd += ["-ldl", "-lpthread", "-lrt"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building " + os.path.basename(out))
    if ptxas_info or verbose:
        sys.stderr.write(res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="-v" in sys.argv,
                debug="--debug" in sys.argv))
