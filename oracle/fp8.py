"""FP8 E4M3 decoding, float64 — oracle (test infrastructure only).

FP8 inference kernels are listed among the inference library's capabilities
(wsisp.com "FIA / FlashAttention", section 三, comparison table, FP8 row; FA-3's
FP8 support, section 一 table).  The pages do not define the format; this
module follows the E4M3 encoding of the OCP 8-bit floating point
specification (the "FN" variant KV caches use): 1 sign bit s, 4 exponent bits
e with bias 7, 3 mantissa bits m, no infinities,

    e == 0:             (-1)^s * 2^-6 * (m / 8)          (subnormal, incl. +-0)
    0 < e, not NaN:     (-1)^s * 2^(e - 7) * (1 + m / 8)
    e == 15, m == 7:    NaN

so the largest finite magnitude is 448 (e = 15, m = 6).

Reading taken for the quantised KV cache: one scale per
tensor, k = k_scale * E4M3(k8), v = v_scale * E4M3(v8); the query stays bf16.
"""
from __future__ import annotations

import numpy as np


def e4m3_to_f64(bits) -> np.ndarray:
    """E4M3 bit patterns (uint8) -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where(s == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def dequantize_e4m3(bits, scale: float) -> np.ndarray:
    """Per-tensor dequantisation: scale * E4M3(bits)."""
    return float(scale) * e4m3_to_f64(bits)
