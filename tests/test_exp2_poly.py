"""The FMA-pipe exponential of the prefill kernel (2^x = 2^rint(x) * cubic(f),
f = x - rint(x)), restated in numpy float32 with the coefficients the kernel
compiles (csrc/exp2_poly.h): its relative error against numpy's exp2 stays
far below the bf16 rounding of P (2^-9), over the whole input range the
kernel feeds it (x in [-125, 8]; smaller inputs are clamped to -125)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "query_adaptive_chunk_b200", "csrc", "exp2_poly.h")


def coeffs():
    txt = open(HDR).read()
    return [np.float32(float(re.search(rf"CSA_EXP2_C{i} ([-0-9.eE+]+)f", txt).group(1)))
            for i in range(4)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_fma(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    jf = (t - magic).astype(np.float32)
    f = (x - jf).astype(np.float32)
    c0, c1, c2, c3 = coeffs()
    q = fma32(f, c3, c2)
    q = fma32(q, f, c1)
    q = fma32(q, f, c0)
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_kernel_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_003, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, -1e-7, 8.0, -125.0, -124.5])])
    got = exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 2e-4, rel.max()


def test_integers_are_exact_powers_of_two_up_to_the_cubic_at_zero():
    x = np.arange(-125, 9, dtype=np.float32)
    got = exp2_fma(x).astype(np.float64)
    c0 = float(coeffs()[0])
    np.testing.assert_allclose(got, c0 * np.exp2(x.astype(np.float64)), rtol=1e-7)


def test_clamp_below_the_range():
    got = exp2_fma(np.float32([-126.0, -1000.0, -np.inf]))
    assert np.all(got > 0) and np.all(got < 3e-38)
