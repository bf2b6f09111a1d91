"""Failure detection without faulting the GPU.

Every mbarrier wait in the GEMMs is bounded by wall time; when a wait runs
out the kernel records FPQ_ERR_DEVICE_TIMEOUT in the device error word,
skips its stores, frees its TMEM and returns, so the context stays usable.
The test makes the waits run out on purpose: FPQ_DEBUG_GEMM_STALL=1 makes the
MXFP8 GEMM's producer declare 16 more TMA bytes per stage than it loads (the
stage barriers can never complete, while every issued load still lands), and
FPQ_WAIT_TIMEOUT_MS shortens the limit.  Malformed device input (decreasing
group offsets) is covered in test_parity_gemm.py; host-side validation in
test_abi.py."""
import os
import time

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _mx_operands(fpq, m):
    wl = workloads.mxfp8_256x512()
    a = wl["a"] if m == wl["a"].shape[0] else workloads.normal_bf16((m, 512), 0.02, 7)
    qa, sa = fpq.quantize(a.cuda(), fpq.MXFP8)
    qb, sb = fpq.quantize(wl["b"].cuda(), fpq.MXFP8)
    return qa, sa, qb, sb


# m = 64: one-CTA kernel; m = 256: CTA pair (the leader's stage barrier
# never completes; the peer, the scale loaders and the epilogue time out too)
@pytest.mark.parametrize("m", [64, 256])
def test_gemm_wait_timeout_is_reported_and_context_survives(fpq, orc, m):
    qa, sa, qb, sb = _mx_operands(fpq, m)
    torch.cuda.synchronize()
    assert fpq.fpq_get_device_error() == 0
    good = fpq.scaled_gemm(fpq.MXFP8, qa, sa, fpq.MXFP8, qb, sb, out_dtype=torch.float32)
    torch.cuda.synchronize()

    os.environ["FPQ_DEBUG_GEMM_STALL"] = "1"
    os.environ["FPQ_WAIT_TIMEOUT_MS"] = "50"
    try:
        t0 = time.time()
        stalled = torch.full_like(good, -7.0)
        fpq.fpq_scaled_gemm(fpq.MXFP8, qa, sa, fpq.MXFP8, qb, sb, m, 256, 512, stalled, fpq.OUT_F32)
        code = fpq.fpq_get_device_error()
        elapsed = time.time() - t0
    finally:
        del os.environ["FPQ_DEBUG_GEMM_STALL"]
        del os.environ["FPQ_WAIT_TIMEOUT_MS"]
    assert code == 5, code                       # FPQ_ERR_DEVICE_TIMEOUT
    assert elapsed < 10.0
    assert torch.all(stalled == -7.0)            # the timed-out kernel stored nothing
    assert fpq.fpq_get_device_error() == 0       # reading cleared the word

    again = fpq.scaled_gemm(fpq.MXFP8, qa, sa, fpq.MXFP8, qb, sb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(again, good)              # the context is still usable
    assert fpq.fpq_get_device_error() == 0
