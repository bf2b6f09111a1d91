"""GPU parity of the NVFP4 block-scaled GEMM ("fireworks-prequant 0.1.0",
Formats: packed FP4 + FP8 block scales) against the oracle's fp64 reference:
C = gA gB sum_k e2m1(A) sA e2m1(B) sB.  Same acceptance as the other GEMMs
(|gpu - ref| <= 8e-3 |ref| + 1e-2 rms(ref) per element); exact where every
product and partial sum is exact in fp32."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

FNV = 3
E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])   # OCP E2M1 by code


def dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.atleast_1d(a))).cuda()


def rand(shape, seed, std=1.0, outliers=0.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed, outlier_frac=outliers))


def check(got: torch.Tensor, ref: np.ndarray, orc, what: str, rms=None):
    g = got.float().cpu().numpy().astype(np.float64)
    ok, ratio = orc.gemm_tolerance_ok(g, ref, rms)
    assert ok, f"{what}: worst |err|/bound = {ratio:.3f}"


def pack(codes: np.ndarray) -> np.ndarray:
    """[r, k] 4-bit codes -> [r, k/2] bytes, element 2i in the low nibble."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


# K a multiple of 256 takes the paths whose scale rows arrive by TMA (rows of
# K/16 bytes on 16-byte boundaries), with CTA pairs (256 x 256 tiles) once M
# exceeds 128; other K read the scale rows directly.
@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (200, 272, 384), (1, 16, 128), (300, 512, 1024),
                                   (257, 256, 640), (160, 256, 896), (384, 512, 1152), (129, 16, 256),
                                   (520, 336, 512), (640, 1024, 2048)])
def test_nvfp4_gemm_random(fpq, orc, m, n, k):
    a = rand((m, k), 700 + m, std=0.02, outliers=0.01)
    b = rand((n, k), 800 + n, std=0.02, outliers=0.01)
    aq, as_, ag = orc.quant_nvfp4(a)
    bq, bs, bg = orc.quant_nvfp4(b)
    ref = orc.gemm_full(FNV, aq, as_, FNV, bq, bs, ag=ag, bg=bg)
    for dt in (torch.float32, torch.bfloat16):
        c = fpq.scaled_gemm_nvfp4(dev(aq), dev(as_), dev(ag), dev(bq), dev(bs), dev(bg), out_dtype=dt)
        check(c, ref, orc, f"nvfp4 {m}x{n}x{k} {dt}")
    assert fpq.fpq_get_device_error() == 0


def test_nvfp4_gemm_scale_layout_exact(fpq):
    """Random codes and random power-of-two block scales, unit tensor
    scales: every product is a multiple of 1/16 below 600 and every sum fits
    fp32 exactly, so C must equal the product of independently decoded
    operands bit for bit (any misplaced block scale changes it)."""
    rng = np.random.default_rng(3)
    m, n, k = 256, 512, 1024
    ca, cb = rng.integers(0, 16, (m, k)), rng.integers(0, 16, (n, k))
    pow2 = np.array([0x30, 0x38, 0x40, 0x48], np.uint8)                # E4M3 0.5, 1, 2, 4
    ia, ib = rng.integers(0, 4, (m, k // 16)), rng.integers(0, 4, (n, k // 16))
    A = E2M1[ca] * np.repeat(0.5 * 2.0 ** ia, 16, axis=1)
    B = E2M1[cb] * np.repeat(0.5 * 2.0 ** ib, 16, axis=1)
    one = np.ones(1, np.float32)
    c = fpq.scaled_gemm_nvfp4(dev(pack(ca)), dev(pow2[ia]), dev(one), dev(pack(cb)), dev(pow2[ib]), dev(one),
                              out_dtype=torch.float32)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), A @ B.T)


def test_nvfp4_gemm_tensor_scales(fpq, orc):
    """The per-operand tensor scales enter as a product in the epilogue."""
    a, b = rand((128, 512), 901, std=0.02), rand((256, 512), 902, std=0.02)
    aq, as_, ag = orc.quant_nvfp4(a)
    bq, bs, bg = orc.quant_nvfp4(b)
    for fa, fb in ((1.0, 1.0), (0.125, 3.0), (1e-3, 7e2)):
        ga, gb = np.float32(fa) * np.ones(1, np.float32), np.float32(fb) * np.ones(1, np.float32)
        ref = orc.gemm_full(FNV, aq, as_, FNV, bq, bs, ag=ga, bg=gb)
        c = fpq.scaled_gemm_nvfp4(dev(aq), dev(as_), dev(ga), dev(bq), dev(bs), dev(gb), out_dtype=torch.float32)
        check(c, ref, orc, f"tensor scales {fa} {fb}")


def test_nvfp4_gemm_gpu_quantized(fpq, orc):
    """The whole GPU path: bf16 -> NVFP4 (GPU quantizer) -> NVFP4 GEMM."""
    a, b = rand((192, 768), 903), rand((272, 768), 904, std=0.02)
    aq, as_, ag = orc.quant_nvfp4(a)
    bq, bs, bg = orc.quant_nvfp4(b)
    ref = orc.gemm_full(FNV, aq, as_, FNV, bq, bs, ag=ag, bg=bg)
    qa, sa, gga = fpq.quantize(workloads.from_u16(a).cuda(), fpq.NVFP4)
    qb, sb, ggb = fpq.quantize(workloads.from_u16(b).cuda(), fpq.NVFP4)
    check(fpq.scaled_gemm_nvfp4(qa, sa, gga, qb, sb, ggb), ref, orc, "nvfp4 GPU quantized")


def test_nvfp4_gemm_full_size_sampled(fpq, orc):
    """The fine-grained GEMM shape (A 4096x7168 N(0,1), B 2048x7168
    N(0,0.02)) in NVFP4, 128 rows x 64 columns sampled against the oracle."""
    wl = workloads.ds_fp8_gemm()
    qa, sa, ga = fpq.quantize(wl["a"].cuda(), fpq.NVFP4)
    qb, sb, gb = fpq.quantize(wl["b"].cuda(), fpq.NVFP4)
    c = fpq.scaled_gemm_nvfp4(qa, sa, ga, qb, sb, gb)
    rng = np.random.default_rng(6)
    rows = np.sort(rng.choice(4096, 128, replace=False))
    cols = np.sort(rng.choice(2048, 64, replace=False))
    A = workloads.as_u16(wl["a"])
    # the tensor scale depends on the whole matrix: quantize it whole, then sample rows
    oqa, osa, oga = orc.quant_nvfp4(A)
    oqb, osb, ogb = orc.quant_nvfp4(workloads.as_u16(wl["b"]))
    rr, cc = np.meshgrid(rows, cols, indexing="ij")
    ref = orc.gemm_entries(FNV, oqa, osa, FNV, oqb, osb, rr.ravel(), cc.ravel(), ag=oga, bg=ogb)
    got = c[torch.from_numpy(rr.ravel()).cuda(), torch.from_numpy(cc.ravel()).cuda()]
    check(got, ref, orc, "nvfp4 full size", rms=float(np.sqrt(np.mean(ref ** 2))))
    assert fpq.fpq_get_device_error() == 0



def test_nvfp4_gemm_repeatable(fpq):
    """Repeated launches on the same inputs give bit-identical results (the
    CTA-pair kernel hands scale atoms between CTAs through barriers; a
    missing ordering would show up as run-to-run differences)."""
    rng = np.random.default_rng(11)
    m, n, k = 2048, 1024, 4096
    aq = dev(rng.integers(0, 256, (m, k // 2), dtype=np.uint8))
    bq = dev(rng.integers(0, 256, (n, k // 2), dtype=np.uint8))
    # E4M3 scales in [2^-3, 2^3): exponent fields 4..9, random mantissas
    sa = dev((rng.integers(4, 10, (m, k // 16)) << 3 | rng.integers(0, 8, (m, k // 16))).astype(np.uint8))
    sb = dev((rng.integers(4, 10, (n, k // 16)) << 3 | rng.integers(0, 8, (n, k // 16))).astype(np.uint8))
    one = dev(np.ones(1, np.float32))
    first = fpq.scaled_gemm_nvfp4(aq, sa, one, bq, sb, one, out_dtype=torch.float32)
    for _ in range(8):
        again = fpq.scaled_gemm_nvfp4(aq, sa, one, bq, sb, one, out_dtype=torch.float32)
        assert torch.equal(again, first)
    assert fpq.fpq_get_device_error() == 0
