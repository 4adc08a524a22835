"""Pins of the oracle's fused decode + matrix-vector product (float64) to exact
arithmetic: Python fractions on small cases, unit vectors, and the orientation
of both operands (a transposed W or swapped x rows fails)."""
from fractions import Fraction

import numpy as np

from test_oracle_pins import bf16_as_f32


def rand_bf16(rng, shape, std):
    f = (rng.standard_normal(shape) * std).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def test_gemv_exact_rationals(orc):
    rng = np.random.default_rng(31)
    rows, cols, B = 3, 256, 128
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (2, cols), 1.0)
    y, absum = orc.gemv(orc.compress(W, B), rows, cols, B, x)
    Wf, xf = bf16_as_f32(W).astype(np.float64), bf16_as_f32(x).astype(np.float64)
    for j in range(2):
        for r in range(rows):
            exact = sum(Fraction(Wf[r, c]) * Fraction(xf[j, c]) for c in range(cols))
            bound = cols * 2.0 ** -53 * float(sum(abs(Fraction(Wf[r, c]) * Fraction(xf[j, c]))
                                                  for c in range(cols)))
            assert abs(Fraction(y[j, r]) - exact) <= Fraction(bound)
            assert absum[j, r] >= abs(y[j, r])


def test_gemv_unit_vectors_pick_columns(orc):
    rng = np.random.default_rng(32)
    rows, cols, B = 5, 512, 256
    W = rand_bf16(rng, (rows, cols), 0.02)
    stream = orc.compress(W, B)
    for c in (0, 1, 255, 256, 511):
        x = np.zeros((1, cols), np.uint16)
        x[0, c] = 0x3F80  # 1.0
        y, _ = orc.gemv(stream, rows, cols, B, x)
        assert np.array_equal(y[0], bf16_as_f32(W[:, c]).astype(np.float64))


def test_gemv_orientation(orc):
    rows, cols, B = 2, 128, 128
    W = np.zeros((rows, cols), np.uint16)
    W[0, :] = 0x3F80          # row 0: all ones
    W[1, 0] = 0x4000          # row 1: 2.0 in column 0
    x = np.zeros((2, cols), np.uint16)
    x[0, :] = 0x3F80          # x0: all ones
    x[1, 0] = 0x4040          # x1: 3.0 in column 0
    y, _ = orc.gemv(orc.compress(W, B), rows, cols, B, x)
    assert y.tolist() == [[128.0, 2.0], [3.0, 6.0]]
