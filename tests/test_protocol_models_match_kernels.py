"""The host protocol models (tests/*_protocol_model.py) restate each kernel's
barrier arrival counts, ring depths and shared-memory aliasing.  This test
ties those numbers to the kernel sources: if a kernel changes one of them,
the matching line here fails and the model has to be revisited."""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "exact_attention_148_b200", "csrc")


def _source(name):
    with open(os.path.join(CSRC, name)) as f:
        return re.sub(r"\s+", " ", f.read())


# (kernel source, text it must contain, what the model assumes)
FACTS = [
    # persistent prefill (tests/persist_protocol_model.py)
    ("prefill_persist_sm100.cuh", "constexpr int kPersistQueue = 4;", "queue depth QD = 4"),
    ("prefill_persist_sm100.cuh", "constexpr int NS = B::NS;", "the grid form's ring depths 5 and 8"),
    ("prefill_persist_sm100.cuh", "CONSUMERS = 1 + 8 + (F8 ? 2 : 0);", "item_empty arrivals: MMA + 8 softmax + 2 converters"),
    ("prefill_persist_sm100.cuh", "mbar_init(bar_kv_empty(i), (F8 && (i & 1)) ? 2 : 1);", "E4M3 V slots freed by both converters"),
    ("prefill_persist_sm100.cuh", "mbar_init(bar_p_full(k), 4);", "p_full: four softmax warps per slot"),
    ("prefill_persist_sm100.cuh", "mbar_init(bar_p_half(k), 4);", "p_half: four softmax warps per slot"),
    ("prefill_persist_sm100.cuh", "mbar_init(bar_vh_full(k), 2);", "vh_full: two converter warps"),
    # grid prefill (tests/prefill_grid_protocol_model.py)
    ("prefill_pp_sm100.cuh", "NS = F8 ? 8 : (D == 128) ? 5 : 8;", "ring depths 5 and 8"),
    ("prefill_pp_sm100.cuh", "mbar_init(bar_kv_empty(i), (F8 && (i & 1)) ? 2 : 1);", "E4M3 V slots freed by both converters"),
    ("prefill_pp_sm100.cuh", "mbar_init(bar_p_full(k), 4);", "p_full: four softmax warps per slot"),
    ("prefill_pp_sm100.cuh", "mbar_init(bar_p_half(k), 4);", "p_half: four softmax warps per slot"),
    ("prefill_pp_sm100.cuh", "mbar_init(bar_vh_full(k), 2);", "vh_full: two converter warps"),
    ("prefill_pp_sm100.cuh", "if (ok) tc_commit(bar_kv_empty(0));", "K_0 freed after both slots' first S"),
    # tensor-core decode (tests/decode_protocol_model.py, simulate)
    ("decode_tc_sm100.cuh", "CTAS_PER_SM = NPAD == 8 ? 2 : 1;", "8 padded rows: two CTAs per SM"),
    ("decode_tc_sm100.cuh", "ITEMS = (CTAS_PER_SM == 2 ? 96 : 192) * 1024 / KV_BYTES;", "ring of 3/6 (bf16) or 6/12 (E4M3) items"),
    ("decode_tc_sm100.cuh", "mbar_init(bar_q, KV8 ? 4 : 1);", "E4M3: the four softmax warps build Q"),
    ("decode_tc_sm100.cuh", "mbar_init(bar_p_full(k), 4);", "p_full: four softmax warps"),
    ("decode_tc_sm100.cuh", "mbar_wait(bar_kv_empty(it), item_par(it) ^ 1, abort_flag)", "producer waits one phase back"),
    # CUDA-core decode (tests/decode_protocol_model.py, simulate_cc)
    ("decode_sm100.cuh", "STAGES = KV8 ? 6 : 3;", "ring of 3 (bf16) or 6 (E4M3) pages"),
    ("decode_sm100.cuh", "mbar_init(bar_empty(st), 4);", "a page slot is freed by the four consumer warps"),
    ("decode_sm100.cuh", "CMB_O = 0;", "the combine scratch starts at the K ring"),
    ("decode_sm100.cuh", "CMB_M = 4 * GC * D * 4;", "combine maxima after the four warps' O"),
    ("decode_sm100.cuh", "CMB_L = CMB_M + 4 * GC * 4;", "combine sums after the maxima"),
]


@pytest.mark.parametrize("source,text,assumption", FACTS, ids=[f"{s}:{a}" for s, _, a in FACTS])
def test_kernel_matches_model_assumption(source, text, assumption):
    assert re.sub(r"\s+", " ", text) in _source(source), \
        f"{source} no longer has `{text}` ({assumption}): revisit the protocol model"


def test_models_use_the_same_numbers():
    from tests import decode_protocol_model as dm
    from tests import persist_protocol_model as pm
    from tests import prefill_grid_protocol_model as gm
    # the random cases draw the kernels' ring depths only
    assert {gm.random_case(s)[1] for s in range(200)} == {5, 8}
    assert {(pm.random_case(s)[2], pm.random_case(s)[3]) for s in range(200)} == \
        {(5, False), (8, False), (8, True)}
    assert {(dm.random_case(s)[1], dm.random_case(s)[2]) for s in range(200)} == \
        {(3, False), (6, False), (6, True), (12, True)}
