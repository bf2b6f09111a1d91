"""Worst-case accumulation at the workloads' contraction length (K = 7168).

"DeepSeek-V3 Blog 5: Low-Precision Training", Avoiding Numerical Drift with
Mixed-Precision Accumulation: a tensor-core accumulator narrower than fp32
loses the low bits of long sums, and the loss grows with K.  Random-sign data
hides it (errors cancel and partial sums stay small), so these tests use the
case that exposes it: every code positive and near the format's maximum,
every partial sum growing monotonically to ~1e9 at unit scales.  The block-
scaled MXFP8 and NVFP4 kernels keep the whole K loop in the TMEM accumulator
with no promotion, and the fp32-scale kernel promotes each 128-wide K block
into fp32 registers, so all three accumulation paths are covered, on one-CTA
tiles (M <= 128) and on CTA pairs (M > 128), dense and grouped.

Each case compares every output element with the oracle's fp64 product of
the dequantized operands under the GEMM acceptance
|gpu - ref| <= 8e-3 |ref| + 1e-2 rms(ref) (rms over the whole output), and,
for fp32 output, under the bound any fp32 accumulation meets on positive
terms: relative error <= K * 2^-22 (the any-order round-to-nearest bound is
(K - 1) 2^-24; the slack covers truncating adders and the scale products).
The second bound is the one that tells accumulators apart: simulated on the
CPU on these inputs, sums of 32-product partials truncated to 24 bits stay
near 5e-6, while truncation to 14 bits (the width the page describes for the
previous generation) gives 4e-3, over the bound, although still inside the
acceptance tolerance."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

F1x128, F128, FMX, FNV = 0, 1, 2, 3
K = 7168
FP32_ACCUM_REL = K * 2.0 ** -22


def dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.atleast_1d(a))).cuda()


def _threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def par_rows(fn, m):
    """fn(lo, hi) -> rows [lo, hi) of the reference, evaluated on all host
    cores (the oracle's C calls release the GIL) and stacked."""
    n = min(_threads(), m)
    cuts = np.linspace(0, m, n + 1).astype(int)
    with ThreadPoolExecutor(n) as ex:
        parts = list(ex.map(lambda i: fn(cuts[i], cuts[i + 1]), range(n)))
    return np.concatenate(parts)


def ref_full(orc, fa, aq, as_, fb, bq, bs, ag=None, bg=None):
    """The oracle's fp64 product, A's rows split over threads (A's scales are
    per row in every format used here, so a row slice is self-contained)."""
    orc.lib()
    return par_rows(lambda lo, hi: orc.gemm_full(fa, aq[lo:hi], as_[lo:hi], fb, bq, bs, ag=ag, bg=bg), aq.shape[0])


def check(got: torch.Tensor, ref: np.ndarray, orc, what: str, fp32_out: bool):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.all(ref > 0), "worst-case inputs are all positive"
    ok, ratio = orc.gemm_tolerance_ok(g, ref)
    rel = float(np.max(np.abs(g - ref) / ref))
    assert ok, f"{what}: worst |err|/bound = {ratio:.3f} (max rel err {rel:.3e})"
    if fp32_out:
        assert rel <= FP32_ACCUM_REL, f"{what}: max rel err {rel:.3e} above the fp32 accumulation bound " \
                                      f"{FP32_ACCUM_REL:.3e}"


def e4m3_near_max(rng, shape):
    """Positive E4M3 codes 0x70..0x7E: values 256 .. 448 (the format's max)."""
    return rng.integers(0x70, 0x7F, shape).astype(np.uint8)


def e2m1_near_max(rng, shape):
    """[rows, K] positive E2M1 codes 5..7 (3, 4, 6; 6 is the format's max)
    packed two per byte, element 2i in the low nibble."""
    c = rng.integers(5, 8, shape).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


OUTS = [(torch.float32, True), (torch.bfloat16, False)]


# ------------------------------------------------------------------ MXFP8, dense

@pytest.mark.parametrize("m", [128, 256])            # one-CTA tiles / CTA pairs
@pytest.mark.parametrize("scales", ["unit", "random"])
def test_mxfp8_accumulation_worst_case(fpq, orc, m, scales):
    rng = np.random.default_rng(71 + m + (scales == "random"))
    n = 256
    aq, bq = e4m3_near_max(rng, (m, K)), e4m3_near_max(rng, (n, K))
    if scales == "unit":
        as_, bs = np.full((m, K // 32), 127, np.uint8), np.full((n, K // 32), 127, np.uint8)
    else:
        as_ = rng.integers(120, 135, (m, K // 32)).astype(np.uint8)
        bs = rng.integers(120, 135, (n, K // 32)).astype(np.uint8)
    ref = ref_full(orc, FMX, aq, as_, FMX, bq, bs)
    for dt, f32 in OUTS:
        c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs), out_dtype=dt)
        check(c, ref, orc, f"mxfp8 {m}x{n}x{K} {scales} {dt}", f32)
    assert fpq.fpq_get_device_error() == 0


# ------------------------------------------------------------------ MXFP8, grouped

@pytest.mark.parametrize("scales", ["unit", "random"])
def test_grouped_mxfp8_accumulation_worst_case(fpq, orc, scales):
    """An empty expert, a 300-row expert (one full CTA-pair tile and a
    ragged one) and a 1-row expert, K = 7168."""
    rng = np.random.default_rng(81 + (scales == "random"))
    groups, n = 3, 256
    offsets = np.array([0, 0, 300, 301], np.int32)
    total = int(offsets[-1])
    aq, bq = e4m3_near_max(rng, (total, K)), e4m3_near_max(rng, (groups, n, K))
    if scales == "unit":
        as_, bs = np.full((total, K // 32), 127, np.uint8), np.full((groups, n, K // 32), 127, np.uint8)
    else:
        as_ = rng.integers(120, 135, (total, K // 32)).astype(np.uint8)
        bs = rng.integers(120, 135, (groups, n, K // 32)).astype(np.uint8)
    orc.lib()
    cols = np.arange(n)

    def rows(lo, hi):
        rr, cc = np.meshgrid(np.arange(lo, hi), cols, indexing="ij")
        return orc.grouped_gemm_entries(FMX, aq, as_, bq, bs, offsets, rr.ravel(), cc.ravel()).reshape(hi - lo, n)

    ref = par_rows(rows, total)
    for dt, f32 in OUTS:
        c = fpq.grouped_scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), dev(bq), dev(bs), dev(offsets), out_dtype=dt)
        check(c, ref, orc, f"grouped mxfp8 {scales} {dt}", f32)
    assert fpq.fpq_get_device_error() == 0


# ------------------------------------------------------------------ NVFP4

@pytest.mark.parametrize("m", [128, 256])            # one-CTA tiles / CTA pairs
@pytest.mark.parametrize("scales", ["unit", "random"])
def test_nvfp4_accumulation_worst_case(fpq, orc, m, scales):
    rng = np.random.default_rng(91 + m + (scales == "random"))
    n = 256
    aq, bq = e2m1_near_max(rng, (m, K)), e2m1_near_max(rng, (n, K))
    if scales == "unit":
        as_, bs = np.full((m, K // 16), 0x38, np.uint8), np.full((n, K // 16), 0x38, np.uint8)   # E4M3 1.0
        ag, bg = np.ones(1, np.float32), np.ones(1, np.float32)
    else:
        # E4M3 0x30..0x50: 0.5 .. 8 with every mantissa; fp32 tensor scales off powers of two
        as_ = rng.integers(0x30, 0x51, (m, K // 16)).astype(np.uint8)
        bs = rng.integers(0x30, 0x51, (n, K // 16)).astype(np.uint8)
        ag, bg = np.array([0.37], np.float32), np.array([1.9], np.float32)
    ref = ref_full(orc, FNV, aq, as_, FNV, bq, bs, ag=ag, bg=bg)
    for dt, f32 in OUTS:
        c = fpq.scaled_gemm_nvfp4(dev(aq), dev(as_), dev(ag), dev(bq), dev(bs), dev(bg), out_dtype=dt)
        check(c, ref, orc, f"nvfp4 {m}x{n}x{K} {scales} {dt}", f32)
    assert fpq.fpq_get_device_error() == 0


# ------------------------------------------------------------------ fp32 scales (1x128 x 128x128)

@pytest.mark.parametrize("scales", ["unit", "random"])
def test_fp8_f32scale_accumulation_worst_case(fpq, orc, scales):
    """Each 128-wide K block accumulates in TMEM and is promoted into fp32
    registers with its scale product; 56 promotions per output."""
    rng = np.random.default_rng(101 + (scales == "random"))
    m, n = 256, 256
    aq, bq = e4m3_near_max(rng, (m, K)), e4m3_near_max(rng, (n, K))
    if scales == "unit":
        as_, bs = np.ones((m, K // 128), np.float32), np.ones((n // 128, K // 128), np.float32)
    else:
        as_ = rng.uniform(0.25, 4.0, (m, K // 128)).astype(np.float32)
        bs = rng.uniform(0.25, 4.0, (n // 128, K // 128)).astype(np.float32)
    ref = ref_full(orc, F1x128, aq, as_, F128, bq, bs)
    for dt, f32 in OUTS:
        c = fpq.scaled_gemm(fpq.FP8_1x128, dev(aq), dev(as_), fpq.FP8_128x128, dev(bq), dev(bs), out_dtype=dt)
        check(c, ref, orc, f"fp8 f32-scale {m}x{n}x{K} {scales} {dt}", f32)
    assert fpq.fpq_get_device_error() == 0
