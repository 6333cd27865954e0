"""The FMA-pipe 2^x of the softmax anchor kernel (gla_softmax_anchor.cuh),
emulated in numpy float32 / int32 from the constants read out of the header:
the degree-3 fit stays within 1e-4 relative error of 2^x over the range P
takes (x in [-125, 8]: below that P is under 1e-37 and only its size
matters), including the exponent-field arithmetic, and the clamp turns -inf
into a value no sum notices."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "gated_linear_attention_frame_b200", "csrc",
                   "gla_softmax_anchor.cuh")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1)))
            for i in range(4)]


def exp2_poly3(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (x - (t - magic)).astype(np.float32)
    p = ((c3 * r + c2) * r + c1) * r + c0
    bits = p.astype(np.float32).view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_range_of_p():
    x = np.linspace(-125.0, 8.0, 400001, dtype=np.float32)
    got = exp2_poly3(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1e-4


def test_integers_and_halves():
    x = np.arange(-125, 9, dtype=np.float32)
    np.testing.assert_allclose(exp2_poly3(x), np.exp2(x.astype(np.float64)), rtol=1e-4)
    h = x[:-1] + np.float32(0.5)
    np.testing.assert_allclose(exp2_poly3(h), np.exp2(h.astype(np.float64)), rtol=1e-4)


def test_masked_keys_vanish():
    v = exp2_poly3(np.array([-np.inf, -1e30, -200.0, -126.0, -125.7], dtype=np.float32))
    assert np.all(np.isfinite(v)) and np.all(v >= 0) and np.all(v < 1e-37)
