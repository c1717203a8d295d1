"""The prefill kernel's FMA-pipe exp2 (Cody-Waite reduction + degree-3 Remez
polynomial), emulated in float32 on the CPU with the constants read from the
kernel source, against numpy's exp2 and the fit's stated error bound."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_148_b200", "csrc", "prefill_pp_sm100.cuh")


def kernel_coefficients():
    body = open(SRC).read().split("float exp2_poly(float x)")[1].split("\n}")[0]
    nums = [float(x) for x in re.findall(r"([0-9]+\.[0-9]+)f", body)]
    # clamp, +magic, -magic, then fmaf(c3, f, c2); fmaf(p, f, c1); fmaf(p, f, c0)
    assert nums[:3] == [125.0, 12582912.0, 12582912.0], nums
    c3, c2, c1, c0 = nums[3:7]
    return c0, c1, c2, c3


def emulate(x):
    """Bit-faithful float32 emulation of the device function's steps."""
    c0, c1, c2, c3 = (np.float32(c) for c in kernel_coefficients())
    magic = np.float32(12582912.0)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)          # float32 add, round to nearest even
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    fma = lambda a, b, c: (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)
    p = fma(c3, f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = (p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error_bound():
    x = np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4, rel.max()


def test_exp2_poly_exact_at_integers_within_bound():
    x = np.arange(-124, 9, dtype=np.float32)
    rel = np.abs(emulate(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4


def test_exp2_poly_is_far_below_bf16_rounding():
    # P is stored as bf16 (relative rounding up to 2^-9); the polynomial must be
    # at least 10x more accurate than that.
    x = np.random.default_rng(0).uniform(-30, 8, 100000).astype(np.float32)
    rel = np.abs(emulate(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2.0 ** -9 / 10


def test_fit_script_reproduces_kernel_coefficients():
    from exact_attention_148_b200.tools.fit_exp2_poly import remez_rel
    c, err = remez_rel()
    assert err < 8e-5
    for a, b in zip(c, kernel_coefficients()):
        assert abs(a - b) < 1e-8


def test_exp2_poly_rounding_uses_nearest_integer():
    # f must stay within [-1/2, 1/2] for the fit's bound to apply
    x = np.linspace(-124.0, 8.0, 100001, dtype=np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    assert np.all(np.abs(x - n) <= 0.5)
    assert np.array_equal(n, np.rint(x))
