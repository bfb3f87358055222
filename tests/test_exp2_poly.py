"""The FMA-pipe 2^x used for part of the softmax numerators (CPU check).

The constants are read from the kernel source and the device steps (clamp,
round-to-nearest split with the 1.5 * 2^23 constant, fp32 Horner, exponent
add) are replayed in fp32; the result must be within 8e-5 relative of 2^x on
[-126, 8.5] (the polynomial's minimax bound is 7.5e-5; P is then rounded to
bf16, whose half-ulp is 2^-9) and effectively zero below.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "packed_mm_rope_b200", "csrc", "attention.cuh")).read()
    c = {int(k): np.float32(float(v)) for k, v in re.findall(r"EXP2_C(\d) = ([0-9.e+-]+)f;", src)}
    return [c[i] for i in range(4)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)
    j = (x + big).astype(np.float32)
    f = (x - (j - big).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.int32).astype(np.int64) + (j.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    # results below 2^-120 can fall into fp32's subnormal range and lose bits;
    # they are zero at bf16 resolution next to numerators >= 2^-8
    x = np.linspace(-120.0, 8.5, 2_000_001).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 8e-5, rel.max()
    lo = np.linspace(-126.0, -120.0, 10001).astype(np.float32)
    assert np.abs(exp2_fma(lo).astype(np.float64) - np.exp2(lo.astype(np.float64))).max() <= 2.0 ** -130


def test_integers_and_halves():
    x = np.arange(-120, 9).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=8e-5)
    h = (np.arange(-120, 9) + 0.5).astype(np.float32)
    np.testing.assert_allclose(exp2_fma(h).astype(np.float64), np.exp2(h.astype(np.float64)), rtol=8e-5)


def test_underflow_and_masked_keys():
    got = exp2_fma(np.array([-127.0, -500.0, -np.inf], np.float32))
    assert np.all(got >= 0) and np.all(got <= 2.0 ** -125)
