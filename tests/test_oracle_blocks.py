"""Pins of the oracle's block quantizers, dequantizers and LoRA merge:
special blocks, invariants, and brute force in exact rational arithmetic on
small inputs (a second, independent statement of each definition).  CPU only."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads
from exact import bf16_value, e2m1_value, e4m3_value, nearest_code, to_bf16, to_f32

E4M3_POS = {c: e4m3_value(c) for c in range(0x7F)}          # finite, non-negative
E4M3_NEG = {c | 0x80: -v for c, v in E4M3_POS.items()}
E2M1_POS = {c: e2m1_value(c) for c in range(8)}
E2M1_NEG = {c | 8: -v for c, v in E2M1_POS.items()}


def exact_e4m3(t: Fraction, negative: bool) -> int:
    """RNE-saturating E4M3 by brute force; `negative` carries the sign (for -0)."""
    if abs(t) >= 448:
        return 0xFE if negative else 0x7E
    return nearest_code(t, E4M3_NEG if negative else E4M3_POS)


def exact_e2m1(t: Fraction, negative: bool) -> int:
    if abs(t) >= 6:
        return 0xF if negative else 0x7
    return nearest_code(t, E2M1_NEG if negative else E2M1_POS)


def bf16_bits(vals):
    return workloads.as_u16(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def rand_bf16(shape, seed, std=1.0, outliers=0.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed, outlier_frac=outliers))


def sign_of(bits):
    return bool(int(bits) >> 15)


# ------------------------------------------------------------------ MXFP8

def test_mxfp8_special_blocks(orc):
    # all-zero block: exponent clamps to -127 (code 0), every element 0x00
    q, s = orc.quant_mxfp8(np.zeros((1, 32), np.uint16))
    assert s[0, 0] == 0 and not q.any()
    # negative zeros keep their sign
    q, s = orc.quant_mxfp8(np.full((1, 32), 0x8000, np.uint16))
    assert s[0, 0] == 0 and (q == 0x80).all()
    # single outlier: 31 zeros and one 1.0 -> e = -8 (code 119), 1.0 * 2^8 = 256 -> 0x78
    x = np.zeros((1, 32), np.uint16)
    x[0, 5] = 0x3F80
    q, s = orc.quant_mxfp8(x)
    assert s[0, 0] == 119 and q[0, 5] == 0x78 and q.sum() == 0x78
    # subnormal block: amax 2^-130 -> e clamps at -127 (code 0); x * 2^127 = 2^-3 -> 0x20
    x = np.zeros((1, 32), np.uint16)
    x[0, 0] = 0x0008                               # 2^-130 as a bf16 subnormal
    assert bf16_value(0x0008) == Fraction(2) ** -130
    q, s = orc.quant_mxfp8(x)
    assert s[0, 0] == 0 and q[0, 0] == 0x20
    # a block containing +-448 * 2^-5 = +-14 exactly: e = -5, those elements -> 0x7E / 0xFE
    x = bf16_bits([14.0, -14.0] + [0.5] * 30)[None, :]
    q, s = orc.quant_mxfp8(x)
    assert s[0, 0] == 122 and q[0, 0] == 0x7E and q[0, 1] == 0xFE
    assert q[0, 2] == exact_e4m3(Fraction(1, 2) * 32, False)


def test_mxfp8_brute_force(orc):
    x = rand_bf16((3, 96), seed=21, std=0.02, outliers=0.05)
    q, s = orc.quant_mxfp8(x)
    for r in range(3):
        for j in range(3):
            blk = [bf16_value(int(b)) for b in x[r, 32 * j:32 * j + 32]]
            amax = max(abs(v) for v in blk)
            # smallest exponent >= -127 keeping every |x| / 2^e within 448
            e = -127
            while amax / Fraction(2) ** e > 448:
                e += 1
            assert s[r, j] == e + 127
            for i, v in enumerate(blk):
                want = exact_e4m3(v / Fraction(2) ** e, sign_of(x[r, 32 * j + i]))
                assert q[r, 32 * j + i] == want


def test_mxfp8_invariants_on_outlier_matrix(orc):
    x = workloads.as_u16(workloads.mxfp8_256x512()["b"])
    q, s = orc.quant_mxfp8(x)
    deq_codes = np.vectorize(orc.e4m3_decode)(q)
    scale = np.ldexp(1.0, s.astype(np.int64) - 127)
    xs = np.vectorize(orc.bf16_decode)(x)
    for r in range(0, 256, 17):
        for j in range(16):
            blk = slice(32 * j, 32 * j + 32)
            d = deq_codes[r, blk]
            if s[r, j] > 0:
                # the scaled block max lies in (224, 448]; its E4M3 code can
                # round down onto 224 itself, never below
                assert 224 < np.max(np.abs(xs[r, blk])) / scale[r, j] <= 448
                assert 224 <= np.max(np.abs(d)) <= 448
            assert np.all(np.abs(xs[r, blk] / scale[r, j]) <= 448)   # nothing saturates
            # half-ulp bound, in fp64, before any bf16 rounding of the dequant
            t = np.abs(xs[r, blk] / scale[r, j])
            ulp = np.where(t < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, np.floor(np.log2(np.maximum(t, 1e-300))).astype(int) - 3))
            assert np.all(np.abs(d * scale[r, j] - xs[r, blk]) <= ulp / 2 * scale[r, j])


# ------------------------------------------------------------------ fp32-scale FP8

def test_fp8_1x128_special(orc):
    q, s = orc.quant_fp8_1x128(np.zeros((2, 128), np.uint16))
    assert (s == 1.0).all() and not q.any()
    x = rand_bf16((4, 256), seed=5)
    q, s = orc.quant_fp8_1x128(x)
    xs = np.vectorize(orc.bf16_decode)(x)
    for r in range(4):
        for j in range(2):
            blk = np.abs(xs[r, 128 * j:128 * j + 128])
            i = int(np.argmax(blk))
            assert q[r, 128 * j + i] & 0x7F == 0x7E          # the amax element encodes to +-448


def test_fp8_1x128_brute_force(orc):
    x = rand_bf16((3, 256), seed=31, std=0.5)
    x[1, :128] = bf16_bits(np.linspace(-1e-38, 1e-38, 128))   # a block near the fp32 subnormal range
    q, s = orc.quant_fp8_1x128(x)
    for r in range(3):
        for j in range(2):
            blk = [bf16_value(int(b)) for b in x[r, 128 * j:128 * j + 128]]
            amax = max(abs(v) for v in blk)
            sc = Fraction(1) if amax == 0 else to_f32(amax / 448)
            assert Fraction(float(s[r, j])) == sc
            for i, v in enumerate(blk):
                t = to_f32(v / sc)
                assert q[r, 128 * j + i] == exact_e4m3(t, sign_of(x[r, 128 * j + i])), (r, j, i)


def test_fp8_128x128_ragged_brute_force(orc):
    rows, cols = 200, 256                      # second block row has only 72 rows
    x = rand_bf16((rows, cols), seed=41, std=0.02)
    x[150, 200] = bf16_bits([3.0])[0]          # an outlier in block (1, 1)
    q, s = orc.quant_fp8_128x128(x)
    assert s.shape == (2, 2)
    rng = np.random.default_rng(0)
    for bi in range(2):
        for bj in range(2):
            r0, r1 = 128 * bi, min(128 * bi + 128, rows)
            amax = max(abs(bf16_value(int(b))) for b in x[r0:r1, 128 * bj:128 * bj + 128].ravel())
            sc = to_f32(amax / 448)
            assert Fraction(float(s[bi, bj])) == sc
            for _ in range(200):
                r = int(rng.integers(r0, r1))
                c = int(rng.integers(128 * bj, 128 * bj + 128))
                t = to_f32(bf16_value(int(x[r, c])) / sc)
                assert q[r, c] == exact_e4m3(t, sign_of(x[r, c]))
    assert q[150, 200] == 0x7E


def test_fp8_fp32_scale_error_bound(orc):
    """|dec(q) s - x| <= (half an E4M3 ulp of x/s + half an fp32 ulp of x/s) * s."""
    x = rand_bf16((8, 512), seed=51)
    q, s = orc.quant_fp8_1x128(x)
    xs = np.vectorize(orc.bf16_decode)(x)
    d = np.vectorize(orc.e4m3_decode)(q)
    sc = np.repeat(s.astype(np.float64), 128, axis=1)
    t = np.abs(xs / sc)
    e4 = np.where(t < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, np.floor(np.log2(np.maximum(t, 1e-300))).astype(int) - 3))
    assert np.all(np.abs(d * sc - xs) <= (e4 / 2 + t * 2.0 ** -24) * sc)


# ------------------------------------------------------------------ NVFP4

def test_nvfp4_brute_force_and_packing(orc):
    x = rand_bf16((2, 64), seed=61, std=0.02, outliers=0.05)
    q, s, g = orc.quant_nvfp4(x)
    vals = [[bf16_value(int(b)) for b in row] for row in x]
    amax_t = max(abs(v) for row in vals for v in row)
    gv = to_f32(amax_t / 2688)
    assert Fraction(float(g[0])) == gv
    for r in range(2):
        for j in range(4):
            blk = vals[r][16 * j:16 * j + 16]
            amax_b = max(abs(v) for v in blk)
            sb = exact_e4m3(to_f32(to_f32(amax_b / 6) / gv), False)
            assert s[r, j] == sb
            S = to_f32(e4m3_value(sb) * gv)
            for i in range(16):
                c = 16 * j + i
                want = 0 if S == 0 else exact_e2m1(to_f32(vals[r][c] / S), sign_of(x[r, c]))
                byte = int(q[r, c // 2])
                got = byte & 0xF if c % 2 == 0 else byte >> 4
                assert got == want, (r, c)


def test_nvfp4_packing_order_and_zero(orc):
    """Element 2i goes to the low nibble.  With x = [6, 0.5, 0, ...] the block
    scale saturates to 448 and S = fp32(448 g) is within an ulp of 1, so the
    first byte holds 6 (code 7) low and 0.5 (code 1) high: 0x17."""
    x = bf16_bits([6.0, 0.5] + [0.0] * 14)[None, :]
    q, s, g = orc.quant_nvfp4(x)
    assert s[0, 0] == 0x7E and abs(orc.e4m3_decode(0x7E) * float(g[0]) - 1.0) < 1e-6
    assert q[0, 0] == 0x17 and not q[0, 1:].any()
    q, s, g = orc.quant_nvfp4(np.zeros((1, 32), np.uint16))
    assert g[0] == 1.0 and not s.any() and not q.any()


# ------------------------------------------------------------------ dequantizers

@pytest.mark.parametrize("fmt", ["mxfp8", "1x128", "128x128", "nvfp4"])
def test_dequant_exact(orc, fmt):
    x = rand_bf16((130, 256), seed=71, std=0.3, outliers=0.01)
    if fmt == "mxfp8":
        q, s = orc.quant_mxfp8(x)
        out = orc.dequant_mxfp8(q, s)
        scale = lambda r, c: Fraction(2) ** (int(s[r, c // 32]) - 127)
        dec = lambda r, c: e4m3_value(int(q[r, c]))
    elif fmt == "1x128":
        q, s = orc.quant_fp8_1x128(x)
        out = orc.dequant_fp8_1x128(q, s)
        scale = lambda r, c: Fraction(float(s[r, c // 128]))
        dec = lambda r, c: e4m3_value(int(q[r, c]))
    elif fmt == "128x128":
        q, s = orc.quant_fp8_128x128(x)
        out = orc.dequant_fp8_128x128(q, s)
        scale = lambda r, c: Fraction(float(s[r // 128, c // 128]))
        dec = lambda r, c: e4m3_value(int(q[r, c]))
    else:
        q, s, g = orc.quant_nvfp4(x)
        out = orc.dequant_nvfp4(q, s, g)
        scale = lambda r, c: to_f32(e4m3_value(int(s[r, c // 16])) * Fraction(float(g[0])))
        dec = lambda r, c: e2m1_value((int(q[r, c // 2]) >> (4 * (c % 2))) & 0xF)
    rng = np.random.default_rng(1)
    for _ in range(400):
        r, c = int(rng.integers(0, 130)), int(rng.integers(0, 256))
        want = to_bf16(to_f32(dec(r, c) * scale(r, c)))
        assert bf16_value(int(out[r, c])) == want or (want == 0 and bf16_value(int(out[r, c])) == 0)


def test_roundtrip_of_representable_values(orc):
    """Values that are E4M3 codes times a power of two survive quant+dequant."""
    base = [orc.e4m3_decode(c) for c in range(0x40, 0x60)]          # 32 codes in [2^1, 2^4 * 1.875]
    vals = np.array(base) * 2.0 ** -3
    x = bf16_bits(list(vals))[None, :]
    q, s = orc.quant_mxfp8(x)
    assert np.array_equal(orc.dequant_mxfp8(q, s), x)


def test_batch_split_invariance(orc):
    x = rand_bf16((3, 64, 256), seed=81)
    qa, sa = orc.quant_mxfp8(x)
    for b in range(3):
        qb, sb = orc.quant_mxfp8(x[b])
        assert np.array_equal(qa[b], qb) and np.array_equal(sa[b], sb)
    qa, sa, ga = orc.quant_nvfp4(x)
    qb, sb, gb = orc.quant_nvfp4(x[1])
    assert np.array_equal(qa[1], qb) and ga[1] == gb[0]


# ------------------------------------------------------------------ LoRA merge

def test_lora_merge_exact_small(orc):
    """delta = sum_j fma(B[n,j], A[j,k], .) in fp32 (j ascending), then
    W_eff = bf16(fma(alpha/r, delta, W)); each fma is one rounding of the
    exact a*b+c, computed here with rationals."""
    n, k, r = 6, 40, 4
    w = rand_bf16((n, k), seed=91, std=0.02)
    a = rand_bf16((r, k), seed=92, std=0.01)
    b = rand_bf16((n, r), seed=93, std=0.01)
    alpha_over_r = 2.0
    got = orc.lora_merge(w, a, b, alpha_over_r)
    for i in range(n):
        for c in range(k):
            d = Fraction(0)
            for j in range(r):
                d = to_f32(bf16_value(int(b[i, j])) * bf16_value(int(a[j, c])) + d)
            m = to_f32(Fraction(alpha_over_r) * d + bf16_value(int(w[i, c])))
            assert bf16_value(int(got[i, c])) == to_bf16(m), (i, c)


def test_lora_merge_degenerate(orc):
    w = rand_bf16((4, 128), seed=95, std=0.02)
    a = rand_bf16((2, 128), seed=96)
    b = np.zeros((4, 2), np.uint16)
    assert np.array_equal(orc.lora_merge(w, a, b, 2.0), w)           # B = 0: no delta
    assert np.array_equal(orc.lora_merge(w, a, rand_bf16((4, 2), 97), 0.0), w)


def test_lora_merge_fakequant_composes(orc):
    wl = workloads.qat_forward(m=8, n=256, k=384)
    w, a, b = (workloads.as_u16(wl[t]) for t in ("w", "lora_a", "lora_b"))
    q, s, fq = orc.lora_merge_fakequant(w, a, b, wl["alpha_over_r"])
    q2, s2 = orc.quant_fp8_128x128(orc.lora_merge(w, a, b, wl["alpha_over_r"]))
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    assert np.array_equal(fq, orc.dequant_fp8_128x128(q, s))
