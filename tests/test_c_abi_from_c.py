"""The boundary is a C ABI: a plain C11 program (no Python, no torch) compiles
against include/exact_attention.h, links the shared library and uses its
host-only entry points — version, status strings, the decode planner and the
validation that rejects bad arguments before any CUDA call.  No GPU needed."""
import os
import shutil
import subprocess

import pytest

from exact_attention_148_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <stdint.h>
#include "exact_attention.h"

int main(void) {
  printf("version %d\n", fa_version());
  printf("ok '%s'\n", fa_strerror(FA_OK));
  /* 4 requests (the last one empty), 32 q / 8 kv heads, d = 128, 64-token pages */
  const int32_t lens[4] = {1000, 40000, 64, 0};
  fa_plan* plan = NULL;
  size_t ws = 0;
  int st = fa_decode_plan(lens, 4, 32, 8, 128, 64, 1024, 148, 0, &plan, &ws);
  printf("plan %d\n", st);
  if (st != FA_OK) return 1;
  fa_plan_info info;
  st = fa_plan_get_info(plan, &info);
  printf("info %d chunk %d splits %d items %d heads_per_cta %d tc %d ws_match %d\n", st,
         info.chunk_tokens, info.max_splits, info.num_work_items, info.heads_per_cta,
         info.tensor_cores, info.workspace_bytes == ws);
  fa_plan_free(plan);
  /* invalid arguments are refused before any CUDA call */
  printf("bad_heads %d\n", fa_decode_plan(lens, 4, 30, 8, 128, 64, 1024, 148, 0, &plan, &ws));
  printf("bad_page %d\n", fa_decode_plan(lens, 4, 32, 8, 128, 32, 1024, 148, 0, &plan, &ws));
  printf("overflow %d\n", fa_decode_plan(lens, 4, 32, 8, 128, 64, 10, 148, 0, &plan, &ws));
  const int32_t cu[3] = {0, 5, 9};
  printf("null_q %d\n", fa_prefill(NULL, (void*)0x10000, (void*)0x10000, (const int32_t*)0x10000, cu, 2,
                                   4, 4, 128, 1, NAN, (void*)0x10000, NULL, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    _build.build()
    return os.path.dirname(_build.LIB_PATH)


def test_plain_c_program_uses_the_library(tmp_path, lib_dir):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_abi"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", lib_dir, "-lexact_attention", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert lines["version"] == "100"
    assert lines["ok"] == "'ok'"
    assert lines["plan"] == "0"
    info = lines["info"].split()
    fields = dict(zip(info[1::2], info[2::2]))
    assert info[0] == "0"
    chunk, splits = int(fields["chunk"]), int(fields["splits"])
    assert chunk % 64 == 0 and splits == -(-40000 // chunk)
    # 8 kv heads x (splits of each request; an empty request still has one item)
    assert int(fields["items"]) == 8 * sum(max(1, -(-L // chunk)) for L in (1000, 40000, 64, 0))
    assert fields["heads_per_cta"] == "4" and fields["tc"] == "1" and fields["ws_match"] == "1"
    assert int(lines["bad_heads"]) == -1       # FA_ERR_INVALID_ARG: Hq % Hkv != 0
    assert int(lines["bad_page"]) == -2        # FA_ERR_UNSUPPORTED: page size other than 64
    assert int(lines["overflow"]) == -1        # cache longer than the block table can address
    assert int(lines["null_q"]) == -1
