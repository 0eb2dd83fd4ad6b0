"""The kernels' exp2 on the FMA pipe (exp2_poly_pair in fa_common.cuh), checked
on the CPU.

The forward softmax computes part of its 2^x with a polynomial instead of the
MUFU unit.  This test reads the coefficients from the CUDA header, replays the
kernel's fp32 steps bit for bit in numpy (round-to-nearest via the 1.5 * 2^23
shift, the polynomial in fp32 fused multiply-adds, the exponent added as an
integer), and compares with 2^x in double precision.  The bound is the one the
kernel's comment states: relative error below 1e-4 where the result is a
normal number (x >= -125), far below the 2^-9 rounding of P to bf16; below
that it only has to stay a tiny non-negative value.
"""
import os
import re

import numpy as np
import pytest

HEADER = os.path.join(os.path.dirname(__file__), "..", "exact_io_aware_89_b200", "csrc", "fa_common.cuh")


def _coeffs():
    text = open(HEADER).read()
    c = {}
    for i in range(4):
        m = re.search(r"kExp2C%d\s*=\s*([0-9.eE+-]+)f;" % i, text)
        assert m, "coefficient %d not found" % i
        c[i] = np.float32(float(m.group(1)))
    return c


def _fma32(a, b, c):
    # exact a * b + c for fp32 inputs fits comfortably in fp64 for these
    # magnitudes; one rounding to fp32, like the hardware fused multiply-add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    c = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    j = (t - k).astype(np.float32)
    f = _fma32(j, np.full_like(j, -1.0), x)
    p = _fma32(f, np.full_like(f, c[3]), np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 16.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4, rel.max()


def test_integer_arguments_are_nearly_exact():
    x = np.arange(-125, 17, dtype=np.float32)
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    # 2^0 from the polynomial is c0; the exponent field then scales it exactly
    c0 = float(_coeffs()[0])
    np.testing.assert_allclose(got / want, c0, rtol=1e-7)


def test_below_range_clamps_to_tiny_positive():
    # scores far below the row max: below 2^-125 instead of ~0 (a row sum is >= 1)
    got = _exp2_poly(np.array([-125.1, -125.9, -126.0, -127.5, -300.0, -1e6], dtype=np.float32)).astype(np.float64)
    assert np.all(got > 0) and np.all(got < 2.0 ** -125)


@pytest.mark.parametrize("deg", [3])
def test_coefficients_are_a_minimax_fit(deg):
    # The alternation theorem: a minimax relative-error fit of degree 3 has
    # deg + 2 = 5 error extrema of equal size and alternating sign.
    c = _coeffs()
    f = np.linspace(-0.5, 0.5, 200_001)
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    err = (p - np.exp2(f)) / np.exp2(f)
    s = np.sign(err)
    idx = np.concatenate(([0], np.nonzero(np.diff(s))[0] + 1, [len(f)]))
    ext = np.array([np.abs(err[a:b]).max() for a, b in zip(idx[:-1], idx[1:])])
    assert len(ext) == deg + 2
    assert ext.max() < 8e-5
    assert ext.min() > 0.9 * ext.max()  # equioscillation, up to fp32 rounding of the coefficients
