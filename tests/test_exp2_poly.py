"""The prefill kernel's FMA-pipe exp2 (Cody-Waite reduction + degree-3 Remez
polynomial), emulated in float32 on the CPU with the constants read from the
kernel source, against numpy's exp2 and the fit's stated error bound.

The constants themselves are re-derived here: 2^x = 2^n * 2^f with
n = round(x), f = x - n in [-1/2, 1/2] (Cody & Waite, "Software Manual for the
Elementary Functions", 1980), and p(f) the degree-3 polynomial of least
maximum relative error on that interval, found by the Remez exchange
algorithm."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_148_b200", "csrc", "prefill_pp_sm100.cuh")


def kernel_coefficients():
    body = open(SRC).read().split("float2 exp2_poly2(float2 x)")[1].split("\n}")[0]
    nums = [float(x) for x in re.findall(r"([0-9]+\.[0-9]+)f", body)]
    # clamp (x2), +magic (x2), -magic (x2), -1 (x2), then the packed
    # fma(c3, f, c2); fma(p, f, c1); fma(p, f, c0), each constant twice
    assert nums[:8] == [125.0, 125.0, 12582912.0, 12582912.0, 12582912.0, 12582912.0, 1.0, 1.0], nums
    c = nums[8:16]
    assert c[0::2] == c[1::2], c
    c3, c2, c1, c0 = c[0::2]
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


def remez_rel(deg=3, iters=40, a=-0.5, b=0.5):
    """Minimax-relative-error polynomial for 2^f on [a, b] (Remez exchange).
    Returns (coefficients c0..c_deg, max relative error)."""
    n = deg + 2
    xs = 0.5 * (a + b) - 0.5 * (b - a) * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(a, b, 200001)
    target = np.exp2(grid)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i} on the reference points
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x)
        c = np.linalg.solve(A, np.exp2(xs))[:deg + 1]
        err = (np.polyval(c[::-1], grid) - target) / target
        # new reference: the largest error of each sign run, n of them alternating
        s = np.sign(err)
        idx, start = [], 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or s[k] != s[start]:
                seg = np.arange(start, k)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        if len(idx) >= n:
            while len(idx) > n:
                idx.pop(0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1)
            xs = grid[idx]
    return c, np.max(np.abs(err))


def test_kernel_coefficients_are_the_remez_fit():
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
