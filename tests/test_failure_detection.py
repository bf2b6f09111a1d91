"""Failure detection without faulting the GPU.

Every mbarrier wait in the GEMMs is bounded by wall time; when a wait runs
out the kernel records FPQ_ERR_DEVICE_TIMEOUT in the device error word,
skips its stores, frees its TMEM and returns, so the context stays usable.
The test makes the waits run out on purpose: FPQ_DEBUG_GEMM_STALL=1 makes the
MXFP8 GEMM's producer declare 16 more TMA bytes per stage than it loads (the
stage barriers can never complete, while every issued load still lands), and
FPQ_WAIT_TIMEOUT_MS shortens the limit.  The library reads both once per
process, so the stalled launches run in a child process started with them
set.  Malformed device input (decreasing group offsets) is covered in
test_parity_gemm.py; host-side validation in test_abi.py."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The child: an MXFP8 GEMM whose waits run out (m = 64: one-CTA kernel;
# m = 256: CTA pair, where the leader's stage barrier never completes and
# the peer, the scale loaders and the epilogue time out too), then work that
# shows the context still runs kernels correctly: a quantize, and an fp32-
# scale GEMM on integer operands whose exact product is known.
CHILD = r'''
import json, sys, time
sys.path.insert(0, ROOT)
import numpy as np, torch
import mxfp8_block_scaled_warp_b200 as fpq
import workloads
fpq.load()
out = {}
wl = workloads.mxfp8_256x512()
qb, sb = fpq.quantize(wl["b"].cuda(), fpq.MXFP8)
for m in (64, 256):
    a = wl["a"] if m == wl["a"].shape[0] else workloads.normal_bf16((m, 512), 0.02, 7)
    qa, sa = fpq.quantize(a.cuda(), fpq.MXFP8)
    torch.cuda.synchronize()
    first = fpq.fpq_get_device_error()
    stalled = torch.full((m, 256), -7.0, device="cuda")
    t0 = time.time()
    fpq.fpq_scaled_gemm(fpq.MXFP8, qa, sa, fpq.MXFP8, qb, sb, m, 256, 512, stalled, fpq.OUT_F32)
    code = fpq.fpq_get_device_error()
    out[m] = {"before": first, "code": code, "elapsed": time.time() - t0,
              "untouched": bool(torch.all(stalled == -7.0)), "after_read": fpq.fpq_get_device_error()}
rng = np.random.default_rng(3)
code_of = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)
ia, ib = rng.integers(-2, 3, (256, 512)), rng.integers(-2, 3, (256, 512))
dev = lambda t: torch.from_numpy(np.ascontiguousarray(t)).cuda()
c = fpq.scaled_gemm(fpq.FP8_1x128, dev(code_of[ia + 2]), dev(np.ones((256, 4), np.float32)),
                    fpq.FP8_128x128, dev(code_of[ib + 2]), dev(np.ones((2, 4), np.float32)), out_dtype=torch.float32)
out["exact_after"] = bool(np.array_equal(c.cpu().numpy().astype(np.float64), (ia @ ib.T).astype(np.float64)))
q2, s2 = fpq.quantize(wl["b"].cuda(), fpq.MXFP8)
out["quantize_after"] = bool(torch.equal(q2, qb) and torch.equal(s2, sb))
out["final_error"] = fpq.fpq_get_device_error()
print("RESULT " + json.dumps(out))
'''


def test_gemm_wait_timeout_is_reported_and_context_survives(fpq):
    env = dict(os.environ, FPQ_DEBUG_GEMM_STALL="1", FPQ_WAIT_TIMEOUT_MS="50")
    p = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    res = json.loads([ln for ln in p.stdout.splitlines() if ln.startswith("RESULT ")][-1][7:])
    for m in ("64", "256"):
        r = res[m]
        assert r["before"] == 0
        assert r["code"] == 5, r                    # FPQ_ERR_DEVICE_TIMEOUT
        assert r["elapsed"] < 10.0
        assert r["untouched"]                       # the timed-out kernel stored nothing
        assert r["after_read"] == 0                 # reading cleared the word
    assert res["exact_after"] and res["quantize_after"]   # the context is still usable
    assert res["final_error"] == 0
