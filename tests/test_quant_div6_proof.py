"""The quantizer divides a block's amax by 6 with two FMAs instead of an IEEE
division: q = a*c, r = fma(-q, 6, a), q' = fma(r, c, q), c = RN(1/6). This
proves, with exact rational arithmetic and correct float32 rounding, that q'
equals RN(a/6) for every non-negative finite bf16 value a (the amax of a
block of bf16 inputs is always one of them)."""
import struct
from fractions import Fraction

import numpy as np


def _f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def _round_f32(x: Fraction) -> float:
    """Correctly rounded (ties to even) binary32 value of an exact rational."""
    if x == 0:
        return 0.0
    neg = x < 0
    a = -x if neg else x
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = float(np.float32(float(fl * quantum)))
    return -v if neg else v


def test_fma_refined_division_by_6_is_exact_for_every_bf16():
    c = float(np.float32(1.0) / np.float32(6.0))
    assert struct.pack("<f", c) == struct.pack("<I", 0x3E2AAAAB)
    for bits in range(0, 0x7F80):            # +0 .. largest finite bf16
        a = _f32(bits << 16)
        ref = float(np.float32(a) / np.float32(6.0))
        q = _round_f32(Fraction(a) * Fraction(c))
        r = _round_f32(Fraction(-q) * 6 + Fraction(a))
        q2 = _round_f32(Fraction(r) * Fraction(c) + Fraction(q))
        assert q2 == ref, hex(bits)
