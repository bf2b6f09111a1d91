"""Exact rational helpers used to pin the oracle independently of it:
rounding a Fraction to a binary floating-point format (round to nearest,
ties to even, gradual underflow) and decoding bit patterns by their
textbook definitions.  Shared by the CPU tests only."""
from fractions import Fraction
import math


def round_binary(x: Fraction, p: int, emin: int, emax: int) -> Fraction:
    """Nearest value of a binary format with p significant bits, minimum
    normal exponent emin and maximum exponent emax; ties to even; values at
    or beyond the overflow threshold return +-inf (as float)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix the estimate so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)                       # subnormal range shares emin's quantum
    quantum = Fraction(2) ** (e - (p - 1))
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    maxval = (2 - Fraction(2) ** (1 - p)) * Fraction(2) ** emax
    if r > maxval:
        return sign * math.inf
    return sign * r


def to_f32(x: Fraction) -> Fraction:
    return round_binary(Fraction(x), 24, -126, 127)


def to_bf16(x: Fraction) -> Fraction:
    return round_binary(Fraction(x), 8, -126, 127)


def e4m3_value(code: int) -> Fraction:
    s, e, m = code >> 7, (code >> 3) & 15, code & 7
    assert not (e == 15 and m == 7), "NaN"
    mag = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -mag if s else mag


def e2m1_value(code: int) -> Fraction:
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return -mag if s else mag


def bf16_value(bits: int) -> Fraction:
    s, e, m = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
    assert e != 0xFF
    mag = Fraction(m, 128) * Fraction(2) ** -126 if e == 0 else (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
    return -mag if s else mag


def nearest_code(x: Fraction, values: dict):
    """Brute-force nearest code among `values` (code -> Fraction); a tie goes
    to the code whose lowest bit is 0 (the even mantissa)."""
    best = min(abs(x - v) for v in values.values())
    ties = [c for c, v in values.items() if abs(x - v) == best]
    if len(ties) == 1:
        return ties[0]
    even = [c for c in ties if c % 2 == 0]
    assert len(even) == 1, ties
    return even[0]
