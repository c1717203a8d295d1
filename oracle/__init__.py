"""CPU oracle for exact attention forward — TEST INFRASTRUCTURE, not product code.

Plain, slow, float64 NumPy restatements of what the CUDA path computes.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  It shares no code with
``exact_attention_148_b200`` and never imports it.

Parity pins: every public function here is checked in ``tests/test_oracle_*.py``
against closed forms, hand-derived fixtures (``tests/golden/``), brute force in
exact/extended arithmetic, and PyTorch's CPU ``scaled_dot_product_attention``
in float64; none is "parity unpinned".
"""
from .attention import (  # noqa: F401
    append_kv_ref,
    attention_probs_ref,
    attention_ref,
    attention_rows_ref,
    cascade_decode_ref,
    gather_paged_kv,
    kv_head_of,
    merge_states_ref,
    paged_decode_ref,
    paged_decode_rows_ref,
    paged_prefill_ref,
    paged_prefill_rows_ref,
    partial_state_ref,
    visible_key_count,
)
from .fp8 import dequantize_e4m3, e4m3_to_f64  # noqa: F401
