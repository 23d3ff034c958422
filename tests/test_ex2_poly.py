"""The forward kernel computes one exponential in four on the FMA pipe
(ex2_poly2 in csrc/common.cuh).  This restates its steps in float32 numpy
(round-to-nearest by adding 1.5 * 2^23, the cubic, the exponent-field add)
with the constants read from the header, and checks the result against
2^x: relative error at most 1.02e-4 over the softmax's range, exact zeros
for masked scores, exactly 1 at x = 0."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_blockwise_long_b200", "csrc",
                   "common.cuh")


def constants():
    txt = open(HDR).read()
    m = re.search(r"kEx2C1 = ([0-9.e+-]+)f, kEx2C2 = ([0-9.e+-]+)f, kEx2C3 = ([0-9.e+-]+)f", txt)
    return tuple(np.float32(float(v)) for v in m.groups())


def ex2_poly(x):
    c1, c2, c3 = constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    shift = np.float32(12582912.0)
    jm = (x + shift).astype(np.float32)
    j = (jm - shift).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + np.float32(1.0)
    p = p.astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (jm.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) <= 1.03e-4


def test_special_values():
    assert ex2_poly(np.float32(0.0)) == np.float32(1.0)
    assert ex2_poly(np.float32(-np.inf)) == 0.0          # masked score
    assert ex2_poly(np.float32(-127.0)) == 0.0
    tiny = ex2_poly(np.linspace(-127.0, -120.0, 10001, dtype=np.float32))
    assert np.all(tiny >= 0.0) and np.all(np.isfinite(tiny))  # no wrapped exponent near the clamp
    assert np.all(np.diff(tiny.astype(np.float64)) >= -1e-45 * 4)
    whole = ex2_poly(np.arange(-126, 9, dtype=np.float32))
    np.testing.assert_array_equal(whole, np.exp2(np.arange(-126, 9)).astype(np.float32))  # integers are exact


def test_fit_is_a_minimax_cubic():
    """Refit 2^f on [-1/2, 1/2] (relative error, p(0) = 1) by Lawson
    reweighting: the committed constants reach the same maximum error."""
    f = np.linspace(-0.5, 0.5, 100001)
    y = np.exp2(f)
    A = np.stack([f, f ** 2, f ** 3], 1) / y[:, None]
    b = (y - 1) / y
    w = np.ones_like(f)
    for _ in range(200):
        c, *_ = np.linalg.lstsq(A * w[:, None], b * w, rcond=None)
        e = (1 + c[0] * f + c[1] * f ** 2 + c[2] * f ** 3 - y) / y
        w = w * (np.abs(e) / np.abs(e).max()) ** 0.3 + 1e-12
    best = np.abs(e).max()
    c1, c2, c3 = (float(v) for v in constants())
    ours = np.abs((1 + c1 * f + c2 * f ** 2 + c3 * f ** 3 - y) / y).max()
    assert ours <= best * 1.01 and best < 1.1e-4
