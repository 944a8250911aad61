"""CPU pins for the exact-division identities the 2-bit value kernel relies on.

The kernel never divides. It takes s = RN((max - min) / 3) as q = RN(a RN(1/3)),
r = fma(-3, q, a), RN(q + r RN(1/3)). It takes RN(1/s) from a one-ulp reciprocal y0
with one step RN(y0 + y0 fma(-s, y0, 1)). Both are Markstein's identities. These tests
check them against IEEE division with exact rational arithmetic (fractions) or exact
float64 emulation: the first on a sample of fp32 inputs, the second for every positive
finite fp16 s and for y0 at RN(1/s) and both neighbours.
"""

from fractions import Fraction

import numpy as np

THIRD = np.float32(1.0) / np.float32(3.0)


def rn32(fr):
    """Round a Fraction to the nearest float32, ties to even."""
    x = np.float32(float(fr))
    cands = (np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf)))
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - fr), int(np.float32(c).view(np.uint32)) & 1))
    return np.float32(best)


def test_division_by_three_sampled():
    bits = np.arange(0x00800000, 0x7F000000, 4099, dtype=np.uint64).astype(np.uint32)
    a = bits.view(np.float32)
    want = a / np.float32(3.0)
    q = (a.astype(np.float64) * np.float64(THIRD)).astype(np.float32)     # exact product, then RN32
    r64 = a.astype(np.float64) - 3.0 * q.astype(np.float64)               # exact in float64
    r = r64.astype(np.float32)
    assert np.array_equal(r.astype(np.float64), r64)                       # the residual is exact
    s = (q.astype(np.float64) + r.astype(np.float64) * np.float64(THIRD)).astype(np.float32)
    bad = np.nonzero(s != want)[0]
    # float64 may round q + r/3 before the final rounding: settle any mismatch exactly
    for i in bad:
        assert rn32(Fraction(float(q[i])) + Fraction(float(r[i])) * Fraction(float(THIRD))) == want[i]


def _f32_midpoint(x64):
    """True where a float64 value lies exactly halfway between two adjacent float32 values."""
    x32 = x64.astype(np.float32)
    lo = np.where(x32.astype(np.float64) > x64, np.nextafter(x32, np.float32(-np.inf)), x32)
    hi = np.nextafter(lo, np.float32(np.inf))
    return (lo.astype(np.float64) + hi.astype(np.float64)) * 0.5 == x64


def test_reciprocal_step_all_fp16():
    """Every positive finite fp16 s, with y0 at RN(1/s) and both neighbours.

    1 - s y0 is exact in float64 (an 11-bit by 24-bit product near 1), so e = RN32 of
    it is exact too. y0 + e y0 is formed in float64 and rounded to float32; a case
    whose float64 sum is a float32 midpoint (where double rounding could mislead) or
    that disagrees is settled with exact rationals.
    """
    s = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    y = np.float32(1.0) / s                                                 # IEEE RN(1/s)
    for y0 in (np.nextafter(y, np.float32(0)), y, np.nextafter(y, np.float32(np.inf))):
        e = (1.0 - s.astype(np.float64) * y0.astype(np.float64)).astype(np.float32)
        t64 = y0.astype(np.float64) + e.astype(np.float64) * y0.astype(np.float64)
        t = t64.astype(np.float32)
        check = np.nonzero((t != y) | _f32_midpoint(t64))[0]
        for i in check:
            ee = rn32(Fraction(1) - Fraction(float(s[i])) * Fraction(float(y0[i])))
            assert ee == e[i]
            assert rn32(Fraction(float(y0[i])) + Fraction(float(ee)) * Fraction(float(y0[i]))) == y[i]
