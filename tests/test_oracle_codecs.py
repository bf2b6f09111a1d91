"""Pins of the oracle's element codecs against definitions it does not use:
hand-worked fixtures, exhaustive brute force in exact rational arithmetic,
closed forms, and an independent library cast (torch float8_e4m3fn and
bfloat16).  CPU only."""
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from exact import bf16_value, e2m1_value, e4m3_value, nearest_code, to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            v, c = line.split()
            rows.append((float(v), int(c, 0)))
    return rows


E4M3_FINITE = {c: e4m3_value(c) for c in range(256) if (c & 0x7F) != 0x7F}
E2M1_ALL = {c: e2m1_value(c) for c in range(16)}


# ------------------------------------------------------------------ E4M3

def test_e4m3_hand_worked(orc):
    for v, code in _fixture("e4m3_hand_worked.txt"):
        assert orc.e4m3_encode(v) == code, (v, hex(orc.e4m3_encode(v)), hex(code))


def test_e4m3_decode_matches_definition(orc):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            assert math.isnan(orc.e4m3_decode(c))
        else:
            assert Fraction(orc.e4m3_decode(c)) == E4M3_FINITE[c]
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_roundtrip_all_codes(orc):
    for c in range(256):
        d = orc.e4m3_decode(c)
        if math.isnan(d):
            assert orc.e4m3_encode(d) == 0x7F
        else:
            assert orc.e4m3_encode(d) == c


def test_e4m3_encode_all_bf16_exhaustive(orc):
    """Every one of the 65,536 bf16 patterns: the oracle's encode equals a
    brute-force nearest search over all finite E4M3 codes of the input's sign
    (exact rationals, tie -> even code), with NaN -> 0x7F."""
    bad = []
    pos_vals = sorted((v, c) for c, v in E4M3_FINITE.items() if c < 0x80)
    for bits in range(65536):
        e = (bits >> 7) & 0xFF
        if e == 0xFF:
            if bits & 0x7F:                  # NaN
                assert orc.e4m3_encode(float("nan")) == 0x7F
                continue
        got = orc.e4m3_encode(orc.bf16_decode(bits))
        if e == 0xFF:
            want = 0xFE if bits >> 15 else 0x7E
        else:
            xv = bf16_value(bits)
            neg = bool(bits >> 15)
            a = abs(xv)
            if a >= 448:
                mag_code = 0x7E
            else:
                # brute force over the 127 non-negative finite codes
                best = min(abs(a - v) for v, _ in pos_vals)
                ties = [c for v, c in pos_vals if abs(a - v) == best]
                mag_code = ties[0] if len(ties) == 1 else [c for c in ties if c % 2 == 0][0]
            want = mag_code | (0x80 if neg else 0)
        if got != want:
            bad.append((hex(bits), hex(got), hex(want)))
    assert not bad, bad[:10]


def test_e4m3_against_torch_cast(orc):
    """Independent library: torch's float8_e4m3fn cast (RNE) on in-range
    fp32 values (torch does not saturate, so |v| <= 448 only)."""
    g = torch.Generator().manual_seed(7)
    v = torch.cat([
        torch.randn(20000, generator=g) * 100,
        torch.randn(20000, generator=g) * 0.01,
        torch.rand(20000, generator=g) * 2.0 ** -8,
    ]).clamp(-448, 448)
    want = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(t)) for t in v.tolist()], np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_half_ulp_bound(orc):
    """|dec(E4M3(t)) - t| <= half an E4M3 ulp at t (2^(floor(log2|t|) - 3), or
    2^-10 in the subnormal range), for |t| <= 448."""
    rng = np.random.default_rng(3)
    for t in np.concatenate([rng.uniform(-448, 448, 5000), rng.uniform(-0.02, 0.02, 5000)]):
        d = orc.e4m3_decode(orc.e4m3_encode(float(t)))
        a = abs(t)
        ulp = 2.0 ** -9 if a < 2.0 ** -6 else 2.0 ** (math.floor(math.log2(a)) - 3)
        assert abs(d - t) <= ulp / 2, (t, d)


# ------------------------------------------------------------------ E2M1

def test_e2m1_hand_worked(orc):
    for v, code in _fixture("e2m1_hand_worked.txt"):
        assert orc.e2m1_encode(v) == code, (v, orc.e2m1_encode(v), code)


def test_e2m1_all_codes(orc):
    for c in range(16):
        assert Fraction(orc.e2m1_decode(c)) == E2M1_ALL[c]
        assert orc.e2m1_encode(orc.e2m1_decode(c)) == c


def test_e2m1_brute_force_grid(orc):
    """A grid of multiples of 1/16 in [-8, 8] (it contains every tie point):
    the encode equals the brute-force nearest code of the same sign."""
    for i in range(-128, 129):
        x = Fraction(i, 16)
        neg = i < 0
        cands = {c: v for c, v in E2M1_ALL.items() if bool(c & 8) == neg}
        if abs(x) >= 6:
            want = 0xF if neg else 0x7
        else:
            want = nearest_code(x, cands)
        got = orc.e2m1_encode(float(x))
        assert got == want, (x, got, want)


# ------------------------------------------------------------------ E8M0

def test_e8m0_block_exponent_fixture(orc):
    for amax, e in _fixture("e8m0_block_exponent.txt"):
        assert orc.mx_block_exponent(amax) == e, amax


def test_e8m0_block_exponent_all_bf16(orc):
    """Every positive finite bf16 amax: the exponent equals the closed form
    ceil(log2(amax / 448)) clamped to [-127, 127] (fp64 log2 is exact at the
    powers of two that matter: amax = 448 * 2^k gives log2 = k exactly)."""
    for bits in range(1, 0x7F80):
        amax = orc.bf16_decode(bits)
        # estimate with fp64 log2, then settle the ceil in exact arithmetic:
        # the smallest e with 448 * 2^e >= amax
        e = math.ceil(math.log2(amax) - math.log2(448))
        while Fraction(2) ** (e - 1) * 448 >= Fraction(amax):
            e -= 1
        while Fraction(2) ** e * 448 < Fraction(amax):
            e += 1
        assert orc.mx_block_exponent(amax) == max(-127, min(127, e)), amax
        # and the scaled block maximum never exceeds the E4M3 range
        e = orc.mx_block_exponent(amax)
        if e > -127:
            assert 224 < Fraction(amax) / Fraction(2) ** e <= 448


def test_e8m0_decode(orc):
    assert orc.e8m0_decode(127) == 1.0
    assert orc.e8m0_decode(0) == 2.0 ** -127
    assert orc.e8m0_decode(254) == 2.0 ** 127
    assert math.isnan(orc.e8m0_decode(255))


# ------------------------------------------------------------------ bf16

def test_bf16_encode_against_torch_and_exact(orc):
    """bf16 rounding: torch's fp32->bf16 cast (RNE) as an independent library
    on random bit patterns, plus exact-rational ties and subnormals."""
    rng = np.random.default_rng(11)
    pats = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    pats = pats[((pats >> 23) & 0xFF) != 0xFF]                  # finite only
    f = pats.view(np.float32)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_encode(float(x)) for x in f], np.uint16)
    assert np.array_equal(got, want)
    # exact ties: lower half 0x8000 with even and odd upper halves
    for hi in (0x3F80, 0x3F81, 0x0001, 0x0002, 0x7F7E, 0x7F7F):
        u = (hi << 16) | 0x8000
        x = struct.unpack("<f", struct.pack("<I", u))[0]
        fx = Fraction(x)
        want_v = to_bf16(fx)
        got_v = orc.bf16_decode(orc.bf16_encode(x))
        assert (math.isinf(want_v) and math.isinf(got_v)) or Fraction(got_v) == want_v, hex(u)
