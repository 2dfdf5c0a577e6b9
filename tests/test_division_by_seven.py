"""The tensor-core bulk quantizer computes the group scale fl(a / 7) as
fl(a zh + fl(a zl)), zh = fl(1/7), zl = fl(1/7 - zh): division by a divisor
known in advance (Brisebarre, Muller and Raina, IEEE Trans. Computers 53(8),
2004).  The scale's definition (SRFT post, core method: the group scale is the
abs-max over the largest code) is the correctly rounded quotient, so the
two-constant form must equal it for every a in the range the kernel uses it
(2^-90 and up, finite).  Scaling a by a power of two scales every step exactly
there, so checking every significand in [1, 2) covers that range.  The check
is exact: integers, no floating-point comparison of the quotient.
"""
import numpy as np

ZH = np.float32(float.fromhex("0x1.24924ap-3"))
ZL = np.float32(float.fromhex("-0x1.b6db6ep-28"))


def test_constants_are_the_rounded_seventh_and_its_remainder():
    from fractions import Fraction
    # ZH is the float32 nearest to 1/7, ZL the float32 nearest to 1/7 - ZH
    for z, target in ((ZH, Fraction(1, 7)), (ZL, Fraction(1, 7) - Fraction(float(ZH)))):
        below = np.nextafter(z, np.float32(-np.inf))
        above = np.nextafter(z, np.float32(np.inf))
        dz = abs(Fraction(float(z)) - target)
        assert dz < abs(Fraction(float(below)) - target) and dz < abs(Fraction(float(above)) - target)


def test_two_constant_division_by_seven_is_correctly_rounded_for_every_significand():
    M = np.arange(1 << 23, 1 << 24, dtype=np.int64)   # a = M 2^-23 in [1, 2)
    a = (M.astype(np.float64) * 2.0 ** -23).astype(np.float32)
    u = (a.astype(np.float64) * np.float64(ZL)).astype(np.float32)   # exact product, one rounding
    # a zh + u is within 2^-24 ulp of a / 7, which is at least 1/14 ulp from a
    # midpoint, so the fp64 sum rounds to float32 as the fused multiply-add does
    q = (a.astype(np.float64) * np.float64(ZH) + u.astype(np.float64)).astype(np.float32)

    def scaled(v):
        """v (float32 in [2^-5, 2^-1)) times 7 * 2^50, exactly, as int64."""
        bits = v.view(np.int32).astype(np.int64)
        e = ((bits >> 23) & 0xFF) - 127 - 23
        m = (bits & 0x7FFFFF) | (1 << 23)
        return 7 * (m << (e + 50))

    target = M << 27   # (a / 7) * 7 * 2^50
    err = np.abs(scaled(q) - target)
    for nb in (np.nextafter(q, np.float32(0)), np.nextafter(q, np.float32(1))):
        assert np.all(err < np.abs(scaled(nb) - target))
