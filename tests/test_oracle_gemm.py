"""Pins of the oracle's GEMM reference (fp64 sum of exactly dequantized
products): exact-rational brute force on tiny shapes, an integer-exact case,
one-hot scales (scale indexing and layout), numpy's float64 matmul as an
independent library on dequantized operands, and the grouped variant.  CPU."""
from fractions import Fraction

import numpy as np
import pytest

import workloads
from exact import e2m1_value, e4m3_value

FMT = {"1x128": 0, "128x128": 1, "mxfp8": 2, "nvfp4": 3}


def rand_codes(rng, shape, lo=0x00, hi=0x7E):
    """Random finite E4M3 codes (both signs)."""
    c = rng.integers(lo, hi + 1, shape).astype(np.uint8)
    return c | (rng.integers(0, 2, shape).astype(np.uint8) << 7)


def deq_exact(fmt, q, s, g=None):
    """Dequantized operand as exact Fractions (independent of the oracle)."""
    rows = q.shape[0]
    cols = q.shape[1] * (2 if fmt == "nvfp4" else 1)
    out = [[None] * cols for _ in range(rows)]
    for r in range(rows):
        for c in range(cols):
            if fmt == "mxfp8":
                v = e4m3_value(int(q[r, c])) * Fraction(2) ** (int(s[r, c // 32]) - 127)
            elif fmt == "1x128":
                v = e4m3_value(int(q[r, c])) * Fraction(float(s[r, c // 128]))
            elif fmt == "128x128":
                v = e4m3_value(int(q[r, c])) * Fraction(float(s[r // 128, c // 128]))
            else:
                code = (int(q[r, c // 2]) >> (4 * (c % 2))) & 0xF
                v = e2m1_value(code) * e4m3_value(int(s[r, c // 16])) * Fraction(float(g))
            out[r][c] = v
    return out


def test_gemm_tiny_exact_mxfp8(orc):
    rng = np.random.default_rng(0)
    m, n, k = 5, 7, 64
    aq, bq = rand_codes(rng, (m, k)), rand_codes(rng, (n, k))
    as_ = rng.integers(110, 140, (m, k // 32)).astype(np.uint8)
    bs = rng.integers(110, 140, (n, k // 32)).astype(np.uint8)
    got = orc.gemm_full(FMT["mxfp8"], aq, as_, FMT["mxfp8"], bq, bs)
    A, B = deq_exact("mxfp8", aq, as_), deq_exact("mxfp8", bq, bs)
    for i in range(m):
        for j in range(n):
            exact = sum(A[i][t] * B[j][t] for t in range(k))
            mag = sum(abs(A[i][t] * B[j][t]) for t in range(k))
            assert abs(Fraction(got[i, j]) - exact) <= mag * Fraction(1, 2 ** 46)


def test_gemm_tiny_exact_fp32_scales(orc):
    rng = np.random.default_rng(1)
    m, n, k = 4, 130, 256                      # B has two 128-row scale blocks
    aq, bq = rand_codes(rng, (m, k)), rand_codes(rng, (n, k))
    as_ = rng.uniform(0.001, 0.01, (m, k // 128)).astype(np.float32)
    bs = rng.uniform(1e-5, 1e-4, (2, k // 128)).astype(np.float32)
    got = orc.gemm_full(FMT["1x128"], aq, as_, FMT["128x128"], bq, bs)
    A, B = deq_exact("1x128", aq, as_), deq_exact("128x128", bq, bs)
    for i in range(m):
        for j in (0, 1, 127, 128, 129):
            exact = sum(A[i][t] * B[j][t] for t in range(k))
            mag = sum(abs(A[i][t] * B[j][t]) for t in range(k))
            assert abs(Fraction(got[i, j]) - exact) <= mag * Fraction(1, 2 ** 45)


def test_gemm_integer_exact(orc):
    """Scales of one and codes for {-2, -1, 0, 1, 2}: C is an integer and the
    reference must equal it exactly (numpy int64 matmul as the check)."""
    rng = np.random.default_rng(2)
    code_of = {-2: 0xC0, -1: 0xB8, 0: 0x00, 1: 0x38, 2: 0x40}
    for v, c in code_of.items():
        assert e4m3_value(c) == v
    m, n, k = 16, 24, 256
    ia, ib = rng.integers(-2, 3, (m, k)), rng.integers(-2, 3, (n, k))
    aq = np.vectorize(code_of.get)(ia).astype(np.uint8)
    bq = np.vectorize(code_of.get)(ib).astype(np.uint8)
    ones8 = lambda r: np.full((r, k // 32), 127, np.uint8)
    got = orc.gemm_full(FMT["mxfp8"], aq, ones8(m), FMT["mxfp8"], bq, ones8(n))
    assert np.array_equal(got, (ia @ ib.T).astype(np.float64))
    got = orc.gemm_full(FMT["1x128"], aq, np.ones((m, 2), np.float32),
                        FMT["128x128"], bq, np.ones((1, 2), np.float32))
    assert np.array_equal(got, (ia @ ib.T).astype(np.float64))


@pytest.mark.parametrize("which", ["a", "b"])
def test_gemm_one_hot_scale(orc, which):
    """All scales one except a single block at 2^5: only the entries that
    touch that block change, by exactly the block's contribution times 31."""
    rng = np.random.default_rng(3)
    m, n, k = 64, 40, 128
    code_of = {-1: 0xB8, 0: 0x00, 1: 0x38}
    ia, ib = rng.integers(-1, 2, (m, k)), rng.integers(-1, 2, (n, k))
    aq = np.vectorize(code_of.get)(ia).astype(np.uint8)
    bq = np.vectorize(code_of.get)(ib).astype(np.uint8)
    as_, bs = np.full((m, 4), 127, np.uint8), np.full((n, 4), 127, np.uint8)
    r0, kb = (9, 2)
    (as_ if which == "a" else bs)[r0, kb] = 127 + 5
    got = orc.gemm_full(FMT["mxfp8"], aq, as_, FMT["mxfp8"], bq, bs)
    base = (ia @ ib.T).astype(np.float64)
    blk = slice(32 * kb, 32 * kb + 32)
    extra = (ia[:, blk] @ ib[:, blk].T) * 31.0
    want = base.copy()
    if which == "a":
        want[r0, :] += extra[r0, :]
    else:
        want[:, r0] += extra[:, r0]
    assert np.array_equal(got, want)


def test_gemm_against_numpy_on_dequantized(orc):
    """Random quantized operands from the quantizers; numpy float64 matmul of
    the oracle-independent dequantized operands agrees to fp64 rounding."""
    wl = workloads.ds_fp8_gemm(m=64, n=160, k=384)
    aq, as_ = orc.quant_fp8_1x128(workloads.as_u16(wl["a"]))
    bq, bs = orc.quant_fp8_128x128(workloads.as_u16(wl["b"]))
    A = np.array([[float(v) for v in row] for row in deq_exact("1x128", aq, as_)])
    B = np.array([[float(v) for v in row] for row in deq_exact("128x128", bq, bs)])
    want = A @ B.T
    got = orc.gemm_full(FMT["1x128"], aq, as_, FMT["128x128"], bq, bs)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows, cols = np.array([0, 63, 17]), np.array([159, 0, 128])
    assert np.array_equal(orc.gemm_entries(FMT["1x128"], aq, as_, FMT["128x128"], bq, bs, rows, cols),
                          got[rows, cols])


def test_gemm_nvfp4_entry(orc):
    rng = np.random.default_rng(4)
    x = workloads.as_u16(workloads.normal_bf16((8, 64), 0.02, seed=7))
    y = workloads.as_u16(workloads.normal_bf16((6, 64), 0.02, seed=8))
    aq, as_, ag = orc.quant_nvfp4(x)
    bq, bs, bg = orc.quant_nvfp4(y)
    got = orc.gemm_full(FMT["nvfp4"], aq, as_, FMT["nvfp4"], bq, bs, ag=ag, bg=bg)
    A, B = deq_exact("nvfp4", aq, as_, ag[0]), deq_exact("nvfp4", bq, bs, bg[0])
    for i in range(8):
        for j in range(6):
            exact = sum(A[i][t] * B[j][t] for t in range(64))
            assert abs(float(exact) - got[i, j]) <= 1e-12 * max(1e-30, sum(abs(float(A[i][t] * B[j][t])) for t in range(64)))


def test_grouped_entries_match_per_expert(orc):
    rng = np.random.default_rng(5)
    groups, n, k, total = 4, 48, 64, 50
    offsets = np.array([0, 7, 7, 30, 50], np.int32)          # includes an empty expert
    aq = rand_codes(rng, (total, k))
    as_ = rng.integers(115, 135, (total, k // 32)).astype(np.uint8)
    bq = rand_codes(rng, (groups, n, k))
    bs = rng.integers(115, 135, (groups, n, k // 32)).astype(np.uint8)
    rows = np.arange(total).repeat(3)
    cols = rng.integers(0, n, rows.size)
    got = orc.grouped_gemm_entries(FMT["mxfp8"], aq, as_, bq, bs, offsets, rows, cols)
    for i, (r, c) in enumerate(zip(rows, cols)):
        e = int(np.searchsorted(offsets, r, side="right") - 1)
        want = orc.gemm_entries(FMT["mxfp8"], aq, as_, FMT["mxfp8"], bq[e], bs[e], [r], [c])[0]
        assert got[i] == want


def test_tolerance_rule(orc):
    ref = np.array([1.0, -2.0, 0.0, 100.0])
    rms = float(np.sqrt(np.mean(ref ** 2)))
    ok, ratio = orc.gemm_tolerance_ok(ref + 8e-3 * np.abs(ref) + 0.99e-2 * rms, ref)
    assert ok and ratio < 1.0
    ok, ratio = orc.gemm_tolerance_ok(ref + np.array([0, 0, 0.011 * rms, 0]), ref)
    assert not ok and ratio > 1.0
