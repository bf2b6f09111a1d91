"""GPU parity of the strided quantize / dequantize entry points: each
logical matrix is a window of a larger padded buffer (row and batch strides
in elements), the codes land in a window of another padded buffer, and the
result must equal the oracle's on the dense logical matrices byte for byte,
with every padding byte left untouched."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

B, R, C = 2, 200, 256                  # 200 rows: a ragged last 128-row block
PAD = 0xEE


def _x_window(seed):
    """bf16 [B, 210, 384] buffer; the logical x is rows 3..202, columns 64..319."""
    big = workloads.normal_bf16((B, 210, 384), 1.0, seed=seed)
    view = big.cuda()
    return big[:, 3:3 + R, 64:64 + C].contiguous(), view, view[:, 3:3 + R, 64:64 + C], 384, 210 * 384


def _oracle(orc, fmt_name, x_u16):
    if fmt_name == "MXFP8":
        return orc.quant_mxfp8(x_u16)
    if fmt_name == "FP8_1x128":
        return orc.quant_fp8_1x128(x_u16)
    if fmt_name == "FP8_128x128":
        return orc.quant_fp8_128x128(x_u16)
    return orc.quant_nvfp4(x_u16)


def _dense_outputs(fpq, fmt):
    shape = (B, R, C)
    s = torch.empty(fpq.scale_shape(fmt, shape), dtype=fpq._scale_dtype(fmt), device="cuda")
    g = torch.empty((B,), dtype=torch.float32, device="cuda") if fmt == fpq.NVFP4 else None
    ws = None
    if fmt == fpq.NVFP4:
        ws = torch.empty((fpq.fpq_quantize_workspace_bytes(fmt, B) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    return s, g, ws


def _host_bits(t):
    t = t.detach().cpu().contiguous()
    return t.view(torch.int32).numpy().view(np.uint32) if t.dtype == torch.float32 else t.numpy()


@pytest.mark.parametrize("fmt_name", ["MXFP8", "FP8_1x128", "FP8_128x128", "NVFP4"])
def test_quantize_strided(fpq, orc, fmt_name):
    fmt = getattr(fpq, fmt_name)
    x_dense, _, xv, ld_x, bs_x = _x_window(900 + fmt)
    nv = fmt == fpq.NVFP4
    # codes: a window of a [B, 205, 288]-element padded buffer, rows 2.., columns 32..
    ld_q, rows_q = 288, 205
    qbig = torch.full((B, rows_q, ld_q // 2 if nv else ld_q), PAD, dtype=torch.uint8, device="cuda")
    qv = qbig[:, 2:2 + R, (16 if nv else 32):]
    s, g, ws = _dense_outputs(fpq, fmt)
    fpq.fpq_quantize_block_strided(fmt, xv, ld_x, bs_x, B, R, C, qv, ld_q, rows_q * ld_q, s, g, ws)
    want = _oracle(orc, fmt_name, workloads.as_u16(x_dense))
    cw = C // 2 if nv else C
    got_q = qbig[:, 2:2 + R, (16 if nv else 32):(16 if nv else 32) + cw].cpu().numpy()
    assert np.array_equal(got_q, want[0]), "codes"
    assert np.array_equal(_host_bits(s), want[1].view(np.uint32) if want[1].dtype == np.float32 else want[1]), \
        "scales"
    if nv:
        assert np.array_equal(_host_bits(g), np.ascontiguousarray(want[2], np.float32).view(np.uint32)), "g"
    mask = torch.ones_like(qbig, dtype=torch.bool)
    mask[:, 2:2 + R, (16 if nv else 32):(16 if nv else 32) + cw] = False
    assert (qbig[mask] == PAD).all(), "a byte outside the code window was written"
    assert fpq.fpq_get_device_error() == 0


@pytest.mark.parametrize("fmt_name", ["MXFP8", "FP8_1x128", "FP8_128x128", "NVFP4"])
def test_dequantize_strided(fpq, orc, fmt_name):
    fmt = getattr(fpq, fmt_name)
    nv = fmt == fpq.NVFP4
    x = workloads.as_u16(workloads.normal_bf16((B, R, C), 1.0, seed=950 + fmt))
    oq = _oracle(orc, fmt_name, x)
    deq = {"MXFP8": lambda: orc.dequant_mxfp8(oq[0], oq[1]), "FP8_1x128": lambda: orc.dequant_fp8_1x128(oq[0], oq[1]),
           "FP8_128x128": lambda: orc.dequant_fp8_128x128(oq[0], oq[1]),
           "NVFP4": lambda: orc.dequant_nvfp4(oq[0], oq[1], oq[2])}[fmt_name]()
    # codes placed in a window of a padded buffer: ld 320 elements, rows 1..
    ld_q, rows_q = 320, 204
    qbig = torch.full((B, rows_q, ld_q // 2 if nv else ld_q), PAD, dtype=torch.uint8, device="cuda")
    cw = C // 2 if nv else C
    qbig[:, 1:1 + R, :cw] = torch.from_numpy(oq[0]).cuda()
    s = torch.from_numpy(np.ascontiguousarray(oq[1])).cuda()
    g = torch.from_numpy(np.ascontiguousarray(oq[2], np.float32)).cuda() if nv else None
    # output: a window of a padded bf16 buffer [B, 203, 272], rows 2.., columns 16..
    obig = torch.full((B, 203, 272), -7.0, dtype=torch.bfloat16, device="cuda")
    ov = obig[:, 2:2 + R, 16:16 + C]
    fpq.fpq_dequantize_strided(fmt, qbig[:, 1:], ld_q, rows_q * ld_q, s, g, B, R, C, ov, 272, 203 * 272)
    got = workloads.as_u16(obig[:, 2:2 + R, 16:16 + C].contiguous())
    assert np.array_equal(got, deq), "dequantized bf16"
    mask = torch.ones(obig.shape, dtype=torch.bool, device="cuda")
    mask[:, 2:2 + R, 16:16 + C] = False
    assert (obig[mask] == -7.0).all(), "an element outside the output window was written"
    assert fpq.fpq_get_device_error() == 0


def test_strided_single_matrix_ignores_batch_stride(fpq, orc):
    x = workloads.normal_bf16((R, 384), 1.0, seed=960)
    xv = x.cuda()[:, :C]
    qbig = torch.full((R, 272), PAD, dtype=torch.uint8, device="cuda")
    s = torch.empty((R, C // 32), dtype=torch.uint8, device="cuda")
    fpq.fpq_quantize_block_strided(fpq.MXFP8, xv, 384, 0, 1, R, C, qbig, 272, 0, s)
    oq, os_ = orc.quant_mxfp8(workloads.as_u16(x[:, :C].contiguous()))
    assert np.array_equal(qbig[:, :C].cpu().numpy(), oq) and np.array_equal(s.cpu().numpy(), os_)
    assert (qbig[:, C:] == PAD).all()


def test_strided_rejects_bad_strides(fpq):
    x = torch.zeros((2, 64, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((2, 64, 256), dtype=torch.uint8, device="cuda")
    s = torch.zeros((2, 64, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(fpq.FpqError):        # ld below cols
        fpq.fpq_quantize_block_strided(fpq.MXFP8, x, 128, 64 * 256, 2, 64, 256, q, 256, 64 * 256, s)
    with pytest.raises(fpq.FpqError):        # ld not a multiple of 16
        fpq.fpq_quantize_block_strided(fpq.MXFP8, x, 264, 64 * 264, 2, 64, 256, q, 256, 64 * 256, s)
    with pytest.raises(fpq.FpqError):        # batch stride overlapping the previous matrix
        fpq.fpq_quantize_block_strided(fpq.MXFP8, x, 256, 32 * 256, 2, 64, 256, q, 256, 64 * 256, s)
