"""Error bound of the FMA-pipe 2^x used for part of the softmax (CPU).

The attention kernel evaluates a quarter of its exponentials as
2^x = 2^n * p(f) (n nearest integer to x, f = x - n in [-1/2, 1/2], p a
degree-3 polynomial).  This test reads the coefficients from the kernel
source, replays the same float32 steps in numpy and checks the relative error
against 2^x stays below 1e-4 (well under the 2^-9 rounding of the bf16
probabilities it feeds), that masked scores (-inf) give a value far below any
real probability, and that nothing turns into NaN or a negative number.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_attention_long_moga_b200", "csrc", "attention.cu")


def coefficients():
    text = open(SRC).read()
    return [np.float32(float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1))) for i in range(4)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def poly_exp2(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma32(fma32(fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f,
              np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.9, 9.0, 2_000_001, dtype=np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_masked_and_extreme_inputs():
    out = poly_exp2(np.array([-np.inf, -1e30, -126.0, -200.0], dtype=np.float32))
    assert np.all(np.isfinite(out)) and np.all(out >= 0) and np.all(out < 1e-37)
    assert poly_exp2(np.array([0.0], dtype=np.float32))[0] == np.float32(poly_exp2(np.array([0.0]))[0])
    np.testing.assert_allclose(poly_exp2(np.array([0.0, 1.0, -1.0, 8.0], dtype=np.float32)),
                               [1.0, 2.0, 0.5, 256.0], rtol=1e-4)
