"""Host emulation of the FMA-pipe 2^x used by the tensor-core row pass.

The kernel evaluates 2^x = 2^n * p(f) with n = rint(x) taken from the
1.5 * 2^23 rounding constant, f = x - n, a degree-5 polynomial p and an
integer add of n into the exponent field.  This test replays those float32
steps with numpy, using the coefficients as written in the kernel header, and
checks the result against exp2 and the behaviour below -126.
"""

import os
import re

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(HERE, "..", "structured_sparse_attention_grid_b200", "csrc", "tc_common.cuh")


def _coefficients():
    src = open(HEADER).read()
    body = src[src.index("ex2_fma2"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([-+0-9.e]+)f,", body)]
    # Horner order in the source: c5, c4, c3, c2, c1, c0
    c5, c4, c3, c2, c1, c0 = vals[1], vals[2], vals[3], vals[4], vals[5], vals[6]
    assert vals[0] == 12582912.0
    return np.array([c0, c1, c2, c3, c4, c5], np.float32)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma_emulated(x):
    c = _coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    rc = np.float32(12582912.0)
    t = (x + rc).astype(np.float32)
    f = (x - (t - rc).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c[5]), f, np.full_like(f, c[4]))
    for k in (3, 2, 1, 0):
        p = _fma32(p, f, np.full_like(f, c[k]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    y = ex2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 3e-7, rel.max()


def test_integers_are_exact():
    n = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(ex2_fma_emulated(n), np.exp2(n.astype(np.float64)).astype(np.float32))


@pytest.mark.parametrize("x", [-np.inf, -1e30, -300.0, -127.0])
def test_far_below_range_gives_zero(x):
    assert ex2_fma_emulated(np.array([x], np.float32))[0] == 0.0


def test_between_minus_127_and_minus_126_stays_tiny_and_non_negative():
    x = np.linspace(-127.0, -126.0, 10001).astype(np.float32)
    y = ex2_fma_emulated(x)
    assert np.all(y >= 0.0) and np.all(y <= np.float32(2.0 ** -125))
