"""The kernels' Box-Muller transcendentals (csrc/philox.cuh), checked on the
host over every one of their 2^24 inputs.

ln u1 and the cosine / sine of 2 pi u2 are evaluated from the 24-bit integers
the Philox words give (an exact exponent split with the atanh series, and the
quarter turn taken from the integer's top bits with Taylor series).  The test
reads the coefficients out of the header, requires them to be the series'
own, emulates the fp32 operations in the header's order (each rounded once;
fused multiply-adds once) and checks the error bounds the header states
against fp64 logarithms, cosines and sines.  The GPU parity tests then compare
the noisy gate itself with the oracle."""
import math
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "sparsely_gated_mixture_gate_b200", "csrc",
                   "philox.cuh")
f32, f64 = np.float32, np.float64


def _src():
    s = open(HDR).read()
    return s[s.index("void box_muller2("):]


def _chain(var):
    """[first, c1, c2, ...] of `float var = first; var = fmaf(var, f2, c1); ...`"""
    src = _src()
    first = float(re.search(rf"float {var} = ([-0-9.e+]+)f;", src).group(1))
    rest = [float(v) for v in re.findall(rf"{var} = fmaf\({var}, f2, ([-0-9.e+]+)f\);", src)]
    return [first] + rest


def _fma(a, b, c):
    return (a.astype(f64) * b.astype(f64) + c.astype(f64)).astype(f32)


def test_series_coefficients_are_the_taylor_series():
    hp = math.pi / 2
    sin_c = [(-1) ** k * hp ** (2 * k + 1) / math.factorial(2 * k + 1) for k in range(4, -1, -1)]
    cos_c = [(-1) ** k * hp ** (2 * k) / math.factorial(2 * k) for k in range(4, -1, -1)]
    np.testing.assert_allclose(_chain("sn"), sin_c, rtol=1e-15)
    np.testing.assert_allclose(_chain("cs"), cos_c, rtol=1e-15)
    src = _src()
    for k in (9, 7, 5, 3):
        assert f"2.0f / {k}.0f" in src
    assert "0.6931471805599453f" in src and "0x3504f3u" in src  # ln 2 and sqrt 2's mantissa


def test_cos_sin_of_every_u2():
    sc, cc = [f32(v) for v in _chain("sn")], [f32(v) for v in _chain("cs")]
    j = np.arange(1 << 24, dtype=np.uint32)
    jr = j + np.uint32(1 << 21)
    quad = (jr >> np.uint32(22)) & np.uint32(3)
    f = ((jr & np.uint32(0x3fffff)).astype(np.int64) - (1 << 21)).astype(f32) * f32(2.0 ** -22)
    f2 = (f * f).astype(f32)
    sn = np.full_like(f, sc[0])
    for c in sc[1:]:
        sn = _fma(sn, f2, np.full_like(f, c))
    sn = (sn * f).astype(f32)
    cs = np.full_like(f, cc[0])
    for c in cc[1:]:
        cs = _fma(cs, f2, np.full_like(f, c))
    odd = (quad & 1) == 1
    c0, s0 = np.where(odd, sn, cs), np.where(odd, cs, sn)
    cosv = np.where(((quad + 1) & 2) != 0, -c0, c0)
    sinv = np.where((quad & 2) != 0, -s0, s0)
    ang = 2 * np.pi * j.astype(f64) / 2 ** 24
    assert np.max(np.abs(cosv - np.cos(ang))) < 8.9e-8
    assert np.max(np.abs(sinv - np.sin(ang))) < 8.9e-8
    # the quarter turns land exactly
    for q, (c, s) in enumerate([(1, 0), (0, 1), (-1, 0), (0, -1)]):
        k = q << 22
        assert cosv[k] == c and sinv[k] == s


def test_ln_of_every_u1():
    m = np.arange(1, (1 << 24) + 1, dtype=np.int64)  # u1 = m / 2^24
    bits = m.astype(f32).view(np.uint32)
    mant = bits & np.uint32(0x7fffff)
    big = mant >= np.uint32(0x3504f3)
    e = (bits >> np.uint32(23)).astype(np.int64) - 127 - 24 + big
    g = (mant | np.where(big, np.uint32(0x3f000000), np.uint32(0x3f800000))).view(f32)
    s = (((g - f32(1)).astype(f64)) / ((g + f32(1)).astype(f64))).astype(f32)
    s2 = (s * s).astype(f32)
    p = np.full_like(s2, f32(2.0 / 9.0))
    for k in (7, 5, 3, 1):
        p = _fma(p, s2, np.full_like(s2, f32(2.0 / k)))
    lnu = _fma(e.astype(f32), np.full_like(s2, f32(math.log(2))), (p * s).astype(f32))
    ref = np.log(m.astype(f64) / 2 ** 24)
    assert lnu[-1] == 0.0  # u1 = 1
    rel = np.abs(lnu[:-1] - ref[:-1]) / np.abs(ref[:-1])
    assert rel.max() < 2.1e-7
