"""GPU parity of the block-scaled GEMMs against the oracle's fp64 reference.

Small cases feed oracle-quantized operands to the GPU GEMM (isolating the
GEMM) and compare every output element.  Full-size cases run the whole GPU
path (quantize + GEMM) on the workload's seeded inputs while the oracle
quantizes and multiplies the sampled rows itself; the comparison covers a
sample of entries.  Acceptance (per element): |gpu - ref| <= 8e-3 |ref| +
1e-2 rms(ref), rms over the whole output (over the sample where the whole
output is not computed); bit-exact where the result is an exact integer."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

F1x128, F128, FMX = 0, 1, 2


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rand(shape, seed, std=1.0, outliers=0.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed, outlier_frac=outliers))


def check(got: torch.Tensor, ref: np.ndarray, orc, what: str, rms=None):
    g = got.float().cpu().numpy().astype(np.float64)
    ok, ratio = orc.gemm_tolerance_ok(g, ref, rms)
    assert ok, f"{what}: worst |err|/bound = {ratio:.3f}"
    return ratio


def rand_codes(rng, shape, lo=0x00, hi=0x7E):
    c = rng.integers(lo, hi + 1, shape).astype(np.uint8)
    return c | (rng.integers(0, 2, shape).astype(np.uint8) << 7)


# ------------------------------------------------------------------ MXFP8 dense

# M above 128 with K a multiple of 512 runs on CTA pairs (256 x 256 tiles,
# scale rows by TMA); the other shapes on one-CTA 128 x 256 tiles
@pytest.mark.parametrize("m,n,k", [(64, 256, 512), (300, 272, 640), (128, 256, 128), (1, 16, 128),
                                   (257, 512, 1024), (300, 272, 1024), (520, 512, 2048), (129, 16, 512)])
def test_mxfp8_gemm_random(fpq, orc, m, n, k):
    a = rand((m, k), 100 + m, std=0.02, outliers=0.01)
    b = rand((n, k), 200 + n, std=0.02, outliers=0.01)
    aq, as_ = orc.quant_mxfp8(a)
    bq, bs = orc.quant_mxfp8(b)
    ref = orc.gemm_full(FMX, aq, as_, FMX, bq, bs)
    for dt in (torch.float32, torch.bfloat16):
        c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs), out_dtype=dt)
        check(c, ref, orc, f"mxfp8 {m}x{n}x{k} {dt}")
    assert fpq.fpq_get_device_error() == 0


def test_mxfp8_gemm_workload_256x512(fpq, orc):
    """The small MXFP8 workload: B 256x512 (seed 0), A 64x512 (seed 1)."""
    wl = workloads.mxfp8_256x512()
    aq, as_ = orc.quant_mxfp8(workloads.as_u16(wl["a"]))
    bq, bs = orc.quant_mxfp8(workloads.as_u16(wl["b"]))
    ref = orc.gemm_full(FMX, aq, as_, FMX, bq, bs)
    c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs))
    check(c, ref, orc, "mxfp8 workload")
    # and the whole GPU path from bf16
    ga, gsa = fpq.quantize(wl["a"].cuda(), fpq.MXFP8)
    gb, gsb = fpq.quantize(wl["b"].cuda(), fpq.MXFP8)
    check(fpq.scaled_gemm(fpq.MXFP8, ga, gsa, fpq.MXFP8, gb, gsb), ref, orc, "mxfp8 workload, GPU quantize")


def test_mxfp8_gemm_integer_exact(fpq, orc):
    """Unit scales and codes for {-2..2}: an exact integer product, fp32 out."""
    rng = np.random.default_rng(0)
    code_of = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)       # -2, -1, 0, 1, 2
    m, n, k = 200, 512, 1024
    ia, ib = rng.integers(-2, 3, (m, k)), rng.integers(-2, 3, (n, k))
    aq, bq = code_of[ia + 2], code_of[ib + 2]
    as_, bs = np.full((m, k // 32), 127, np.uint8), np.full((n, k // 32), 127, np.uint8)
    c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs), out_dtype=torch.float32)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), (ia @ ib.T).astype(np.float64))


@pytest.mark.parametrize("side", ["a", "b"])
def test_mxfp8_gemm_one_hot_scales(fpq, orc, side):
    """Every scale 1 except one block at 2^5 per row: pins the scale-factor
    layout (row interleave, 32-wide K sub-block, 128-wide K tile) exactly."""
    rng = np.random.default_rng(1)
    m, n, k = 256, 512, 512
    code_of = np.array([0xB8, 0x00, 0x38], np.uint8)
    ia, ib = rng.integers(-1, 2, (m, k)), rng.integers(-1, 2, (n, k))
    aq, bq = code_of[ia + 1], code_of[ib + 1]
    as_, bs = np.full((m, k // 32), 127, np.uint8), np.full((n, k // 32), 127, np.uint8)
    sf = as_ if side == "a" else bs
    hot = rng.integers(0, k // 32, sf.shape[0])
    sf[np.arange(sf.shape[0]), hot] = 127 + 5
    ref = orc.gemm_full(FMX, aq, as_, FMX, bq, bs)
    c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs), out_dtype=torch.float32)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), ref)


def test_mxfp8_gemm_extreme_scales(fpq, orc):
    """Scales spanning the E8M0 range used by real blocks (2^-40 .. 2^20)."""
    rng = np.random.default_rng(2)
    m, n, k = 128, 256, 256
    aq, bq = rand_codes(rng, (m, k)), rand_codes(rng, (n, k))
    as_ = rng.integers(87, 147, (m, k // 32)).astype(np.uint8)
    bs = rng.integers(107, 128, (n, k // 32)).astype(np.uint8)
    ref = orc.gemm_full(FMX, aq, as_, FMX, bq, bs)
    c = fpq.scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), fpq.MXFP8, dev(bq), dev(bs), out_dtype=torch.float32)
    check(c, ref, orc, "extreme scales")


# ------------------------------------------------------------------ fp32-scale (1x128 x 128x128)

# ragged M and N, one and several 128 x 256 tiles
@pytest.mark.parametrize("m,n,k", [(128, 128, 128), (200, 144, 384), (333, 400, 1024), (1, 16, 256),
                                   (129, 16, 128), (520, 272, 768), (640, 1024, 2048)])
def test_fp8_blockscale_gemm_random(fpq, orc, m, n, k):
    a = rand((m, k), 300 + m)
    b = rand((n, k), 400 + n, std=0.02)
    aq, as_ = orc.quant_fp8_1x128(a)
    bq, bs = orc.quant_fp8_128x128(b)
    ref = orc.gemm_full(F1x128, aq, as_, F128, bq, bs)
    for dt in (torch.float32, torch.bfloat16):
        c = fpq.scaled_gemm(fpq.FP8_1x128, dev(aq), dev(as_), fpq.FP8_128x128, dev(bq), dev(bs), out_dtype=dt)
        check(c, ref, orc, f"fp8 blockscale {m}x{n}x{k} {dt}")


def test_fp8_blockscale_gemm_integer_exact(fpq, orc):
    rng = np.random.default_rng(3)
    code_of = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)
    m, n, k = 256, 256, 1024
    ia, ib = rng.integers(-2, 3, (m, k)), rng.integers(-2, 3, (n, k))
    c = fpq.scaled_gemm(fpq.FP8_1x128, dev(code_of[ia + 2]), dev(np.ones((m, k // 128), np.float32)),
                        fpq.FP8_128x128, dev(code_of[ib + 2]), dev(np.ones((n // 128, k // 128), np.float32)),
                        out_dtype=torch.float32)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), (ia @ ib.T).astype(np.float64))


def test_fp8_blockscale_gemm_one_hot_scales(fpq, orc):
    """Power-of-two block scales on both operands, one distinct block each:
    the promoted result must be exact (every partial sum is an integer)."""
    rng = np.random.default_rng(4)
    m, n, k = 256, 256, 512
    code_of = np.array([0xB8, 0x00, 0x38], np.uint8)
    ia, ib = rng.integers(-1, 2, (m, k)), rng.integers(-1, 2, (n, k))
    as_ = np.ones((m, k // 128), np.float32)
    bs = np.ones((n // 128, k // 128), np.float32)
    as_[np.arange(m), rng.integers(0, k // 128, m)] = 4.0
    bs[1, 2] = 0.5
    aq, bq = code_of[ia + 1], code_of[ib + 1]
    ref = orc.gemm_full(F1x128, aq, as_, F128, bq, bs)
    c = fpq.scaled_gemm(fpq.FP8_1x128, dev(aq), dev(as_), fpq.FP8_128x128, dev(bq), dev(bs), out_dtype=torch.float32)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), ref)


# More tiles than SMs (a second, partial wave; a ragged last row of tiles):
# 12 entries of every 128 x 256 tile and the ragged edges against the oracle.
@pytest.mark.parametrize("m,n,k", [(2560, 2048, 256), (3968 + 50, 2048, 384)])
def test_fp8_blockscale_gemm_many_tiles(fpq, orc, m, n, k):
    a = rand((m, k), 500 + m)
    b = rand((n, k), 600 + n, std=0.02)
    aq, as_ = orc.quant_fp8_1x128(a)
    bq, bs = orc.quant_fp8_128x128(b)
    c = fpq.scaled_gemm(fpq.FP8_1x128, dev(aq), dev(as_), fpq.FP8_128x128, dev(bq), dev(bs), out_dtype=torch.float32)
    assert fpq.fpq_get_device_error() == 0
    rng = np.random.default_rng(m)
    rows, cols = [], []
    for mt in range((m + 127) // 128):
        for nt in range((n + 255) // 256):
            rows += list(rng.integers(128 * mt, min(m, 128 * mt + 128), 12))
            cols += list(rng.integers(256 * nt, min(n, 256 * nt + 256), 12))
    rows += [m - 1] * 4 + list(rng.integers(0, m, 4))
    cols += list(rng.integers(0, n, 4)) + [n - 1] * 4
    rows, cols = np.array(rows), np.array(cols)
    ref = orc.gemm_entries(F1x128, aq, as_, F128, bq, bs, rows, cols)
    got = c[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()]
    check(got, ref, orc, f"fp8 blockscale {m}x{n}x{k}", rms=float(np.sqrt(np.mean(ref ** 2))))


def test_fp8_blockscale_gemm_repeatable(fpq):
    """Repeated launches give bit-identical C: the promotion warps and the MMA
    thread hand the two TMEM buffers back and forth through barriers, and a
    missing ordering would show up as run-to-run differences."""
    rng = np.random.default_rng(12)
    m, n, k = 4096, 1280, 4096          # 160 tiles: more than one wave
    aq = dev(rng.integers(0, 0x7F, (m, k), dtype=np.uint8) | (rng.integers(0, 2, (m, k), dtype=np.uint8) << 7))
    bq = dev(rng.integers(0, 0x7F, (n, k), dtype=np.uint8) | (rng.integers(0, 2, (n, k), dtype=np.uint8) << 7))
    as_ = dev(rng.uniform(0.5, 2.0, (m, k // 128)).astype(np.float32))
    bs = dev(rng.uniform(0.5, 2.0, (n // 128, k // 128)).astype(np.float32))
    first = fpq.scaled_gemm(fpq.FP8_1x128, aq, as_, fpq.FP8_128x128, bq, bs, out_dtype=torch.float32)
    for _ in range(8):
        assert torch.equal(fpq.scaled_gemm(fpq.FP8_1x128, aq, as_, fpq.FP8_128x128, bq, bs, out_dtype=torch.float32),
                           first)
    assert fpq.fpq_get_device_error() == 0


def _sampled_dense_check(orc, c_gpu, aq, as_, fa, bq, bs, fb, rows, cols, what):
    rr, cc = np.meshgrid(rows, cols, indexing="ij")
    ref = orc.gemm_entries(fa, aq, as_, fb, bq, bs, rr.ravel(), cc.ravel())
    got = c_gpu[torch.from_numpy(rr.ravel()).cuda(), torch.from_numpy(cc.ravel()).cuda()]
    return check(got, ref, orc, what, rms=float(np.sqrt(np.mean(ref ** 2))))


def test_ds_fp8_gemm_full_size(fpq, orc):
    """The fine-grained FP8 workload end to end at full size (A 4096x7168
    1x128, B 2048x7168 128x128, bf16 out), 256 rows x 64 columns sampled."""
    wl = workloads.ds_fp8_gemm()
    qa, sa = fpq.quantize(wl["a"].cuda(), fpq.FP8_1x128)
    qb, sb = fpq.quantize(wl["b"].cuda(), fpq.FP8_128x128)
    c = fpq.scaled_gemm(fpq.FP8_1x128, qa, sa, fpq.FP8_128x128, qb, sb)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(4096, 256, replace=False))
    cols = np.sort(rng.choice(2048, 64, replace=False))
    oqa, osa = orc.quant_fp8_1x128(workloads.as_u16(wl["a"])[rows])
    oqb, osb = orc.quant_fp8_128x128(workloads.as_u16(wl["b"]))
    rr, cc = np.meshgrid(np.arange(256), cols, indexing="ij")
    ref = orc.gemm_entries(F1x128, oqa, osa, F128, oqb, osb, rr.ravel(), cc.ravel())
    got = c[torch.from_numpy(np.repeat(rows, 64)).cuda(), torch.from_numpy(np.tile(cols, 256)).cuda()]
    check(got, ref, orc, "ds fp8 full size", rms=float(np.sqrt(np.mean(ref ** 2))))
    assert fpq.fpq_get_device_error() == 0


def test_qat_forward_full_size(fpq, orc):
    """QAT forward: merged + 128x128 fake-quantized W, 1x128 fake-quantized X
    (8192x7168), FP8 GEMM; 128 rows x 64 columns sampled."""
    wl = workloads.qat_forward()
    wq, ws = fpq.lora_merge_fakequant(wl["w"].cuda(), wl["lora_a"].cuda(), wl["lora_b"].cuda(), wl["alpha_over_r"])
    xq, xs = fpq.quantize(wl["x"].cuda(), fpq.FP8_1x128)
    c = fpq.scaled_gemm(fpq.FP8_1x128, xq, xs, fpq.FP8_128x128, wq, ws)
    rng = np.random.default_rng(6)
    rows = np.sort(rng.choice(8192, 128, replace=False))
    cols = np.sort(rng.choice(2048, 64, replace=False))
    w_eff = orc.lora_merge(*(workloads.as_u16(wl[t]) for t in ("w", "lora_a", "lora_b")), wl["alpha_over_r"])
    oqw, osw = orc.quant_fp8_128x128(w_eff)
    oqx, osx = orc.quant_fp8_1x128(workloads.as_u16(wl["x"])[rows])
    rr, cc = np.meshgrid(np.arange(128), cols, indexing="ij")
    ref = orc.gemm_entries(F1x128, oqx, osx, F128, oqw, osw, rr.ravel(), cc.ravel())
    got = c[torch.from_numpy(np.repeat(rows, 64)).cuda(), torch.from_numpy(np.tile(cols, 128)).cuda()]
    check(got, ref, orc, "qat forward", rms=float(np.sqrt(np.mean(ref ** 2))))


# ------------------------------------------------------------------ grouped MXFP8

def test_grouped_small_all_entries(fpq, orc):
    groups, n, k = 5, 256, 384
    offsets = np.array([0, 7, 7, 130, 300, 301], np.int32)          # empty, ragged, single-row experts
    total = int(offsets[-1])
    a = rand((total, k), 500, std=1.0)
    w = rand((groups * n, k), 501, std=0.02).reshape(groups, n, k)
    aq, as_ = orc.quant_mxfp8(a)
    bq, bs = orc.quant_mxfp8(w)
    rows, cols = np.meshgrid(np.arange(total), np.arange(n), indexing="ij")
    ref = orc.grouped_gemm_entries(FMX, aq, as_, bq, bs, offsets, rows.ravel(), cols.ravel()).reshape(total, n)
    for dt in (torch.float32, torch.bfloat16):
        c = fpq.grouped_scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), dev(bq), dev(bs), dev(offsets), out_dtype=dt)
        check(c, ref, orc, f"grouped small {dt}")
    assert fpq.fpq_get_device_error() == 0


@pytest.mark.parametrize("n", [256, 272])
def test_grouped_pair_all_entries(fpq, orc, n):
    """Grouped GEMM on CTA pairs (K a multiple of 512): an empty expert, one
    of 7 rows, a pair tile ending inside an expert (293 = 256 + 37 rows), one
    just over a pair tile (257) and a single row; with N = 272 the last
    column tile reaches into the next expert's weight rows, whose output
    columns must not be written."""
    groups, k = 5, 512
    offsets = np.array([0, 7, 7, 300, 557, 558], np.int32)
    total = int(offsets[-1])
    a = rand((total, k), 510, std=1.0)
    w = rand((groups * n, k), 511 + n, std=0.02).reshape(groups, n, k)
    aq, as_ = orc.quant_mxfp8(a)
    bq, bs = orc.quant_mxfp8(w)
    rows, cols = np.meshgrid(np.arange(total), np.arange(n), indexing="ij")
    ref = orc.grouped_gemm_entries(FMX, aq, as_, bq, bs, offsets, rows.ravel(), cols.ravel()).reshape(total, n)
    for dt in (torch.float32, torch.bfloat16):
        c = fpq.grouped_scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), dev(bq), dev(bs), dev(offsets), out_dtype=dt)
        check(c, ref, orc, f"grouped pair n={n} {dt}")
    assert fpq.fpq_get_device_error() == 0


def test_grouped_pair_repeatable(fpq):
    """Repeated grouped launches on CTA pairs give bit-identical C (the scale
    atoms are handed between the CTAs of a pair through barriers)."""
    rng = np.random.default_rng(13)
    groups, n, k = 8, 512, 2048
    offsets = np.array([0, 300, 300, 1100, 1357, 2000, 2001, 2600, 3072], np.int32)
    total = int(offsets[-1])
    aq = dev(rand_codes(rng, (total, k)))
    bq = dev(rand_codes(rng, (groups, n, k)))
    as_ = dev(rng.integers(120, 134, (total, k // 32)).astype(np.uint8))
    bs = dev(rng.integers(120, 134, (groups, n, k // 32)).astype(np.uint8))
    off = dev(offsets)
    first = fpq.grouped_scaled_gemm(fpq.MXFP8, aq, as_, bq, bs, off, out_dtype=torch.float32)
    for _ in range(6):
        assert torch.equal(fpq.grouped_scaled_gemm(fpq.MXFP8, aq, as_, bq, bs, off, out_dtype=torch.float32), first)
    assert fpq.fpq_get_device_error() == 0


def test_grouped_bad_offsets_reported(fpq, orc):
    """A decreasing offset list is malformed device input: the kernel
    reports FPQ_ERR_DEVICE_BAD_INPUT through the device error word."""
    rng = np.random.default_rng(7)
    groups, n, k, total = 3, 256, 128, 64
    aq, as_ = rand_codes(rng, (total, k)), np.full((total, k // 32), 127, np.uint8)
    bq, bs = rand_codes(rng, (groups, n, k)), np.full((groups, n, k // 32), 127, np.uint8)
    bad = np.array([0, 40, 20, 64], np.int32)
    fpq.grouped_scaled_gemm(fpq.MXFP8, dev(aq), dev(as_), dev(bq), dev(bs), dev(bad))
    assert fpq.fpq_get_device_error() == 6
    assert fpq.fpq_get_device_error() == 0          # reading clears it


def test_moe_grouped_full_size(fpq, orc):
    """The grouped workload at full size: 16384 tokens x top-8 of 64 experts
    (131072 permuted rows), up-projection 7168 -> 2048, MXFP8 on both sides.
    Sampled: 8 rows from each of the 4 smallest and 4 largest experts plus
    256 random rows, 48 random columns."""
    wl = workloads.moe_grouped()
    perm, offsets = wl["perm"].numpy(), wl["offsets"].numpy()
    x_perm = wl["x"][wl["perm"]]
    qa, sa = fpq.quantize(x_perm.cuda(), fpq.MXFP8)
    qb, sb = fpq.quantize(wl["w"].cuda(), fpq.MXFP8)
    c = fpq.grouped_scaled_gemm(fpq.MXFP8, qa, sa, qb, sb, torch.from_numpy(offsets).cuda())
    assert fpq.fpq_get_device_error() == 0
    rng = np.random.default_rng(8)
    counts = np.diff(offsets)
    order = np.argsort(counts)
    picks = [rng.integers(offsets[e], offsets[e + 1], 8) for e in list(order[:4]) + list(order[-4:]) if counts[e]]
    rows = np.unique(np.concatenate(picks + [rng.integers(0, 131072, 256)]))
    cols = np.sort(rng.choice(2048, 48, replace=False))
    xh = workloads.as_u16(x_perm)
    oqa, osa = orc.quant_mxfp8(xh[rows])
    experts = np.searchsorted(offsets, rows, side="right") - 1
    ref = np.empty((rows.size, cols.size))
    for e in np.unique(experts):
        oqb, osb = orc.quant_mxfp8(workloads.as_u16(wl["w"][int(e)])[cols])
        sel = np.nonzero(experts == e)[0]
        rr, cc = np.meshgrid(sel, np.arange(cols.size), indexing="ij")
        ref[sel] = orc.gemm_entries(FMX, oqa, osa, FMX, oqb, osb, rr.ravel(), cc.ravel()).reshape(sel.size, -1)
    got = c[torch.from_numpy(np.repeat(rows, cols.size)).cuda(), torch.from_numpy(np.tile(cols, rows.size)).cuda()]
    check(got, ref.ravel(), orc, "moe grouped", rms=float(np.sqrt(np.mean(ref ** 2))))
