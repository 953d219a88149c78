"""The FMA-pipe 2^x helper of sm100_primitives.cuh, checked on the CPU.

exp2_poly2 computes 2^x without the special-function unit: x = n + f,
n = round(x) via the 1.5 * 2^23 constant, 2^f from a cubic, 2^n added to the
exponent bits.  The shipped kernels do not call it (moving a half or a quarter
of the softmax exponentials onto it measured slower); it is kept correct for
kernels that are bound by the special-function unit.  This test replays those
float32 steps in numpy with the coefficients read from the kernel source and
bounds the relative error against numpy.exp2 (float64), which must stay far
below the bf16 resolution (2^-9) of the probabilities it feeds.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_stats_b200", "csrc", "sm100_primitives.cuh")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("exp2_poly2"):]
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, "
                  r"c3 = ([0-9.e+-]+)f", body)
    return [np.float32(float(g)) for g in m.groups()]


def exp2_poly_f32(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    r = np.float32(12582912.0)
    y = (x + r).astype(np.float32)
    n = (y - r).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4
    # far below bf16 resolution of the probabilities
    assert rel.max() < 2.0 ** -9 / 16


def test_integer_points_and_underflow():
    for k in range(-100, 9):
        v = float(exp2_poly_f32(np.float32(k)))
        assert abs(v / 2.0 ** k - 1) < 1e-4
    tiny = exp2_poly_f32(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)
