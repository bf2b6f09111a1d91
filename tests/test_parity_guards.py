"""Guard canaries around every dense output (a stand-in for a memory checker,
which this setup does not run): each output buffer of a quantize,
dequantize, LoRA-merge and GEMM call is carved out of a larger allocation
whose bytes before and after it hold a poison pattern; after the call the
result must equal the oracle's and every poison byte must be intact.  The
shapes are ragged (rows not a multiple of any tile, several column tiles) so
that the kernels' edge handling is what stands next to the guards."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

POISON = 0xA5
GUARD = 4096                      # bytes on each side (keeps 16-byte alignment)


class Guarded:
    """A tensor of `shape`/`dtype` inside a poisoned byte buffer."""

    def __init__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + nbytes + GUARD,), POISON, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool(torch.all(self.buf[:GUARD] == POISON)) and bool(torch.all(self.buf[-GUARD:] == POISON))


def host_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def rand(shape, seed, std=1.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed, outlier_frac=0.01))


SHAPE = (2, 200, 640)             # batch 2, ragged rows, 5 blocks of 128 / 20 of 32 / 40 of 16


@pytest.mark.parametrize("fmt", ["FP8_1x128", "FP8_128x128", "MXFP8", "NVFP4"])
def test_quantize_and_dequantize_guarded(fpq, orc, fmt):
    f = getattr(fpq, fmt)
    x = rand(SHAPE, 31)
    b, r, c = SHAPE
    q = Guarded(fpq.code_shape(f, SHAPE), torch.uint8)
    s = Guarded(fpq.scale_shape(f, SHAPE), torch.float32 if f in (fpq.FP8_1x128, fpq.FP8_128x128) else torch.uint8)
    g = ws = None
    if f == fpq.NVFP4:
        g = Guarded((b,), torch.float32)
        ws = Guarded(((fpq.fpq_quantize_workspace_bytes(f, b) + 15) // 16 * 16,), torch.uint8)
    fpq.fpq_quantize_block(f, workloads.from_u16(x).cuda(), b, r, c, q.t, s.t, g and g.t, ws and ws.t)
    torch.cuda.synchronize()
    want = {"FP8_1x128": orc.quant_fp8_1x128, "FP8_128x128": orc.quant_fp8_128x128, "MXFP8": orc.quant_mxfp8,
            "NVFP4": orc.quant_nvfp4}[fmt](x)
    assert np.array_equal(host_bits(q.t), want[0]) and np.array_equal(host_bits(s.t), bits(want[1]))
    if g is not None:
        assert np.array_equal(host_bits(g.t), bits(np.asarray(want[2], np.float32)))
    for gd in (q, s, g, ws):
        assert gd is None or gd.intact()

    out = Guarded(SHAPE, torch.bfloat16)
    fpq.fpq_dequantize(f, q.t, s.t, g and g.t, b, r, c, out.t)
    torch.cuda.synchronize()
    deq = {"FP8_1x128": orc.dequant_fp8_1x128, "FP8_128x128": orc.dequant_fp8_128x128,
           "MXFP8": orc.dequant_mxfp8}
    ref = orc.dequant_nvfp4(*want) if fmt == "NVFP4" else deq[fmt](*want)
    assert np.array_equal(host_bits(out.t), ref)
    assert out.intact() and q.intact() and s.intact()
    assert fpq.fpq_get_device_error() == 0


def test_lora_merge_guarded(fpq, orc):
    n, k, r = 200, 640, 16
    w, a, bm = rand((n, k), 32, 0.02), rand((r, k), 33, 0.01), rand((n, r), 34, 0.01)
    wq = Guarded((n, k), torch.uint8)
    ws = Guarded(((n + 127) // 128, k // 128), torch.float32)
    wfq = Guarded((n, k), torch.bfloat16)
    fpq.fpq_lora_merge_fakequant(*(workloads.from_u16(t).cuda() for t in (w, a, bm)), n, k, r, 2.0, wq.t, ws.t, wfq.t)
    torch.cuda.synchronize()
    oq, os_, ofq = orc.lora_merge_fakequant(w, a, bm, 2.0)
    assert np.array_equal(host_bits(wq.t), oq) and np.array_equal(host_bits(ws.t), bits(os_))
    assert np.array_equal(host_bits(wfq.t), ofq)
    assert wq.intact() and ws.intact() and wfq.intact()


@pytest.mark.parametrize("m,n,k", [(200, 272, 384), (300, 272, 1024)])   # one-CTA tiles / CTA pairs
def test_gemm_outputs_guarded(fpq, orc, m, n, k):
    """The C of the MXFP8 and fp32-scale GEMMs (ragged M and N: the last row
    tile and column tile are partial) leaves its neighbours untouched."""
    a, b = rand((m, k), 35), rand((n, k), 36, 0.02)
    for fa, fb, qa_fn, qb_fn in ((fpq.MXFP8, fpq.MXFP8, orc.quant_mxfp8, orc.quant_mxfp8),
                                 (fpq.FP8_1x128, fpq.FP8_128x128, orc.quant_fp8_1x128, orc.quant_fp8_128x128)):
        aq, as_ = qa_fn(a)
        bq, bs = qb_fn(b)
        ref = orc.gemm_full(fa, aq, as_, fb, bq, bs)
        for dt, code in ((torch.float32, fpq.OUT_F32), (torch.bfloat16, fpq.OUT_BF16)):
            c = Guarded((m, n), dt)
            d = [torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (aq, as_, bq, bs)]
            fpq.fpq_scaled_gemm(fa, d[0], d[1], fb, d[2], d[3], m, n, k, c.t, code)
            torch.cuda.synchronize()
            ok, ratio = orc.gemm_tolerance_ok(c.t.float().cpu().numpy().astype(np.float64), ref)
            assert ok, ratio
            assert c.intact()
    assert fpq.fpq_get_device_error() == 0
