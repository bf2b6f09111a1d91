"""GPU parity of the quantize / dequantize / LoRA-merge kernels against the
CPU oracle: bit-exact codes, scales and bf16 outputs on the same seeded
inputs, at small sizes spanning several tiles with ragged tails, at the
workloads' full sizes, and on every finite bf16 bit pattern."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def dev(u16: np.ndarray) -> torch.Tensor:
    return workloads.from_u16(u16).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def assert_same(got, want, what):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}: " \
                          f"got {got[tuple(bad[0])]:#x} want {want[tuple(bad[0])]:#x}"


def rand(shape, seed, std=1.0, outliers=0.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed, outlier_frac=outliers))


def wide_range_bf16(shape, seed) -> np.ndarray:
    """Uniformly random finite bf16 bit patterns (all exponents, both signs)."""
    rng = np.random.default_rng(seed)
    return (rng.integers(0, 0x7F80, shape) | (rng.integers(0, 2, shape) << 15)).astype(np.uint16)


def all_finite_bf16(block: int, seed: int = 0) -> np.ndarray:
    """Every finite bf16 pattern once, shuffled, padded with zeros to whole
    rows of `block` elements."""
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    np.random.default_rng(seed).shuffle(pats)
    pad = (-pats.size) % (block * 4)
    pats = np.concatenate([pats, np.zeros(pad, np.uint16)])
    return pats.reshape(-1, block * 4)


def special_rows(cols: int) -> np.ndarray:
    """Rows of blocks the method treats specially: all zero, negative zero,
    one outlier among zeros, bf16 subnormals only, exact 448 * 2^e values."""
    rows = [np.zeros(cols, np.uint16), np.full(cols, 0x8000, np.uint16)]
    r = np.zeros(cols, np.uint16); r[3::32] = 0x3F80; rows.append(r)           # 1.0 outliers
    r = np.zeros(cols, np.uint16); r[::7] = 0x0008; r[1::7] = 0x8001; rows.append(r)   # subnormals
    r = np.full(cols, 0x3F00, np.uint16); r[::16] = 0x4160; rows.append(r)       # 0.5 and 14 = 448 * 2^-5
    r = np.full(cols, 0x4300, np.uint16); r[5::13] = 0xC3E0; rows.append(r)      # 128 and -448
    return np.stack(rows)


# ------------------------------------------------------------------ MXFP8

MX_CASES = {
    "b_256x512": lambda: workloads.as_u16(workloads.mxfp8_256x512()["b"]),
    "a_64x512": lambda: workloads.as_u16(workloads.mxfp8_256x512()["a"]),
    "ragged_333x1056": lambda: rand((333, 1056), 1, std=0.02, outliers=0.01),
    "one_block": lambda: rand((1, 32), 2),
    "special": lambda: special_rows(256),
    "all_finite_bf16": lambda: all_finite_bf16(32),
}


@pytest.mark.parametrize("case", sorted(MX_CASES))
def test_mxfp8_quant_and_dequant(fpq, orc, case):
    x = MX_CASES[case]()
    q, s = fpq.quantize(dev(x), fpq.MXFP8)
    oq, os_ = orc.quant_mxfp8(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), os_, "E8M0 scales")
    out = fpq.dequantize(fpq.MXFP8, q, s)
    assert_same(host(out), orc.dequant_mxfp8(oq, os_), "dequantized bf16")


def test_mxfp8_batched(fpq, orc):
    x = rand((3, 100, 256), 3, std=0.02, outliers=0.01)
    q, s = fpq.quantize(dev(x), fpq.MXFP8)
    oq, os_ = orc.quant_mxfp8(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), os_, "scales")


def test_mxfp8_full_size_activations(fpq, orc):
    """The grouped-GEMM workload's activation matrix, 16384 x 7168, sampled
    rows compared (the full oracle pass over 117 M elements is too slow)."""
    x = workloads.moe_grouped(with_weights=False)["x"]
    q, s = fpq.quantize(x.cuda(), fpq.MXFP8)
    rows = np.random.default_rng(0).choice(16384, 256, replace=False)
    rows.sort()
    xs = workloads.as_u16(x)[rows]
    oq, os_ = orc.quant_mxfp8(xs)
    assert_same(host(q)[rows], oq, "codes")
    assert_same(host(s)[rows], os_, "scales")


# ------------------------------------------------------------------ FP8 with fp32 scales

FP8_CASES = {
    "ragged_7x384": lambda: rand((7, 384), 11),
    "wide_range": lambda: wide_range_bf16((64, 1024), 12),
    "special": lambda: special_rows(512),
    "all_finite_bf16": lambda: all_finite_bf16(128),
    "subnormal_scales": lambda: rand((4, 256), 13) & 0x807F,        # bf16 subnormals only
}


@pytest.mark.parametrize("case", sorted(FP8_CASES))
def test_fp8_1x128_quant_and_dequant(fpq, orc, case):
    x = FP8_CASES[case]()
    q, s = fpq.quantize(dev(x), fpq.FP8_1x128)
    oq, os_ = orc.quant_fp8_1x128(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), f32_bits(os_), "fp32 scales")
    out = fpq.dequantize(fpq.FP8_1x128, q, s)
    assert_same(host(out), orc.dequant_fp8_1x128(oq, os_), "dequantized bf16")


@pytest.mark.parametrize("case", sorted(FP8_CASES) + ["ragged_rows_200"])
def test_fp8_128x128_quant_and_dequant(fpq, orc, case):
    x = rand((200, 384), 14, std=0.02) if case == "ragged_rows_200" else FP8_CASES[case]()
    q, s = fpq.quantize(dev(x), fpq.FP8_128x128)
    oq, os_ = orc.quant_fp8_128x128(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), f32_bits(os_), "fp32 scales")
    out = fpq.dequantize(fpq.FP8_128x128, q, s)
    assert_same(host(out), orc.dequant_fp8_128x128(oq, os_), "dequantized bf16")


def test_fp8_128x128_batched_ragged(fpq, orc):
    x = rand((3, 130, 256), 15, std=0.02)
    q, s = fpq.quantize(dev(x), fpq.FP8_128x128)
    oq, os_ = orc.quant_fp8_128x128(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), f32_bits(os_), "scales")
    assert_same(host(fpq.dequantize(fpq.FP8_128x128, q, s)), orc.dequant_fp8_128x128(oq, os_), "dequant")


def test_ds_fp8_full_size(fpq, orc):
    """The fine-grained FP8 GEMM workload at full size: A 4096x7168 per 1x128
    tile and B 2048x7168 per 128x128 block, compared in full."""
    wl = workloads.ds_fp8_gemm()
    a, b = workloads.as_u16(wl["a"]), workloads.as_u16(wl["b"])
    qa, sa = fpq.quantize(wl["a"].cuda(), fpq.FP8_1x128)
    qb, sb = fpq.quantize(wl["b"].cuda(), fpq.FP8_128x128)
    oqa, osa = orc.quant_fp8_1x128(a)
    oqb, osb = orc.quant_fp8_128x128(b)
    assert_same(host(qa), oqa, "A codes")
    assert_same(host(sa), f32_bits(osa), "A scales")
    assert_same(host(qb), oqb, "B codes")
    assert_same(host(sb), f32_bits(osb), "B scales")


def amax_sweep_blocks(exponents, block: int, seed: int) -> np.ndarray:
    """One block per (exponent field, mantissa field) pair: the block's
    largest magnitude is exactly that bf16 pattern (random sign), the other
    elements random patterns of no larger magnitude.  The quantizers derive
    a block scale from the amax through a per-mantissa table whenever the
    result is a normal fp32 number and by IEEE division otherwise, so the
    sweep covers every table entry on both sides of that boundary."""
    rng = np.random.default_rng(seed)
    pats = [(e << 7) | m for e in exponents for m in range(128)]
    out = np.empty((len(pats), block), np.uint16)
    for i, p in enumerate(pats):
        mags = rng.integers(0, p + 1, block)
        mags[rng.integers(0, block)] = p
        out[i] = (mags | (rng.integers(0, 2, block) << 15)).astype(np.uint16)
    return out


def test_fp8_1x128_every_amax_mantissa(fpq, orc):
    # amax / 448 is a normal fp32 number from exponent field 10 upwards
    x = amax_sweep_blocks(list(range(1, 14)) + list(range(120, 136)) + list(range(245, 255)), 128, 40)
    q, s = fpq.quantize(dev(x), fpq.FP8_1x128)
    oq, os_ = orc.quant_fp8_1x128(x)
    assert_same(host(q), oq, "codes")
    assert_same(host(s), f32_bits(os_), "fp32 scales")


def test_nvfp4_every_amax_mantissa(fpq, orc):
    # amax_b / 6 is a normal fp32 number from exponent field 4 upwards; one
    # matrix per exponent range, so that each has its own tensor scale
    groups = [range(2, 13), range(20, 31), range(100, 111), range(244, 255)]
    x = np.stack([amax_sweep_blocks(list(g), 16, 41 + i).reshape(88, 256) for i, g in enumerate(groups)])
    q, s, g = fpq.quantize(dev(x), fpq.NVFP4)
    oq, os_, og = orc.quant_nvfp4(x)
    assert_same(host(g), f32_bits(og), "tensor scales")
    assert_same(host(s), os_, "E4M3 block scales")
    assert_same(host(q), oq, "packed E2M1 codes")


# ------------------------------------------------------------------ NVFP4

NV_CASES = {
    "small_outliers": lambda: rand((5, 64), 21, std=0.02, outliers=0.05),
    "ragged_33x1056": lambda: rand((33, 1056), 22, std=0.02),
    "special": lambda: special_rows(256),
    "all_finite_bf16": lambda: all_finite_bf16(32)[:1000],
    "zero_tensor": lambda: np.zeros((4, 64), np.uint16),
}


@pytest.mark.parametrize("case", sorted(NV_CASES))
def test_nvfp4_quant_and_dequant(fpq, orc, case):
    x = NV_CASES[case]()
    q, s, g = fpq.quantize(dev(x), fpq.NVFP4)
    oq, os_, og = orc.quant_nvfp4(x)
    assert_same(host(g), f32_bits(og), "tensor scale")
    assert_same(host(s), os_, "E4M3 block scales")
    assert_same(host(q), oq, "packed E2M1 codes")
    out = fpq.dequantize(fpq.NVFP4, q, s, g)
    assert_same(host(out), orc.dequant_nvfp4(oq, os_, og), "dequantized bf16")


@pytest.mark.parametrize("second", ["scaled", "zero"])
def test_nvfp4_two_matrices(fpq, orc, second):
    """Two matrices take the two-launch path (amax pass, then encode); the
    second matrix has its own tensor scale (4x the first's spread, or an
    all-zero matrix whose tensor scale is 1)."""
    a = rand((96, 512), 35, std=0.02, outliers=0.01)
    b = rand((96, 512), 36, std=0.08) if second == "scaled" else np.zeros((96, 512), np.uint16)
    x = np.stack([a, b])
    q, s, g = fpq.quantize(dev(x), fpq.NVFP4)
    oq, os_, og = orc.quant_nvfp4(x)
    assert_same(host(g), f32_bits(og), "tensor scales")
    assert_same(host(s), os_, "E4M3 block scales")
    assert_same(host(q), oq, "packed E2M1 codes")


def test_nvfp4_batched_per_matrix_scale(fpq, orc):
    x = np.stack([rand((64, 128), 30 + i, std=0.02 * (i + 1)) for i in range(5)])
    q, s, g = fpq.quantize(dev(x), fpq.NVFP4)
    oq, os_, og = orc.quant_nvfp4(x)
    assert_same(host(g), f32_bits(og), "tensor scales")
    assert_same(host(s), os_, "block scales")
    assert_same(host(q), oq, "codes")


def test_moe_prequant_full_size_batch(fpq, orc):
    """64 down projections [7168, 2048] in one batched call per format (the
    expert-prequant workload's launch shape); two experts compared in full,
    every expert's NVFP4 tensor scale compared."""
    x = torch.stack([workloads.moe_prequant_matrix(3 * e + 2) for e in range(64)])
    xd = x.cuda()
    q8, s8 = fpq.quantize(xd, fpq.MXFP8)
    q4, s4, g4 = fpq.quantize(xd, fpq.NVFP4)
    xh = workloads.as_u16(x)
    og = np.array([orc.nvfp4_tensor_scale(xh[e]) for e in range(64)], np.float32)
    assert_same(host(g4), f32_bits(og), "tensor scales")
    for e in (0, 41):
        oq, os_ = orc.quant_mxfp8(xh[e])
        assert_same(host(q8[e]), oq, f"MXFP8 codes expert {e}")
        assert_same(host(s8[e]), os_, f"MXFP8 scales expert {e}")
        oq, os_, _ = orc.quant_nvfp4(xh[e])
        assert_same(host(q4[e]), oq, f"NVFP4 codes expert {e}")
        assert_same(host(s4[e]), os_, f"NVFP4 scales expert {e}")


# ------------------------------------------------------------------ LoRA merge + fake-quant

@pytest.mark.parametrize("n,k,r", [(256, 384, 16), (200, 256, 1), (130, 512, 64), (1, 128, 3), (133, 256, 3), (200, 384, 5),
                                   (384, 256, 8), (136, 384, 24), (256, 128, 32), (129, 256, 40)])
def test_lora_merge_fakequant_small(fpq, orc, n, k, r):
    """Every padded rank the kernel instantiates (8, 16, 32, 64) and ranks
    below them (zero-padded), ragged last block rows."""
    w = rand((n, k), 40, std=0.02)
    a = rand((r, k), 41, std=0.01)
    b = rand((n, r), 42, std=0.01)
    wq, ws, wfq = fpq.lora_merge_fakequant(dev(w), dev(a), dev(b), 2.0, want_fq=True)
    oq, os_, ofq = orc.lora_merge_fakequant(w, a, b, 2.0)
    assert_same(host(wq), oq, "codes")
    assert_same(host(ws), f32_bits(os_), "scales")
    assert_same(host(wfq), ofq, "fake-quantized bf16")


def test_lora_merge_fakequant_full_size(fpq, orc):
    wl = workloads.qat_forward()
    w, a, b = (workloads.as_u16(wl[t]) for t in ("w", "lora_a", "lora_b"))
    wq, ws = fpq.lora_merge_fakequant(wl["w"].cuda(), wl["lora_a"].cuda(), wl["lora_b"].cuda(), wl["alpha_over_r"])
    oq, os_ = orc.quant_fp8_128x128(orc.lora_merge(w, a, b, wl["alpha_over_r"]))
    assert_same(host(wq), oq, "codes")
    assert_same(host(ws), f32_bits(os_), "scales")


# ------------------------------------------------------------------ determinism

def test_bytes_identical_across_streams_and_splits(fpq):
    x = dev(rand((6, 128, 512), 50, std=0.02, outliers=0.01))
    for fmt in (fpq.MXFP8, fpq.FP8_1x128, fpq.FP8_128x128, fpq.NVFP4):
        ref = fpq.quantize(x, fmt)
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            again = fpq.quantize(x, fmt)
        side.synchronize()
        parts = [fpq.quantize(x[i:i + 2].contiguous(), fmt) for i in (0, 2, 4)]
        for j in range(len(ref)):
            assert torch.equal(ref[j], again[j])
            assert torch.equal(ref[j], torch.cat([p[j] for p in parts]))
    assert fpq.fpq_get_device_error() == 0
