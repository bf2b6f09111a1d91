"""The non-allocating NVFP4 entry point.

Some callers cannot allocate device memory -- for example a plugin running
inside a serving runtime that owns the whole device memory pool -- and so
cannot supply the amax workspace the regular NVFP4 quantize call needs.
fpq_quantize_nvfp4_noalloc keeps that scratch in a static device array
inside the library instead.  This test calls it through the C ABI twice in a
row and checks both results against the regular (workspace-taking) entry
point on the same inputs; the second call's input has a much smaller
magnitude than the first, so scratch left over from the first call would
show up in its tensor scales.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _noalloc(fpq, x):
    b, r, c = x.shape
    q = torch.empty((b, r, c // 2), dtype=torch.uint8, device=x.device)
    s = torch.empty((b, r, c // 16), dtype=torch.uint8, device=x.device)
    g = torch.empty((b,), dtype=torch.float32, device=x.device)
    fpq.fpq_quantize_nvfp4_noalloc(x, b, r, c, q, s, g)
    return q, s, g


def test_noalloc_nvfp4_matches_workspace_entry_point_twice(fpq):
    first = workloads.normal_bf16((6, 256, 512), 1.0, seed=901, outlier_frac=0.01).cuda()
    second = workloads.normal_bf16((3, 128, 1024), 0.001, seed=902).cuda()
    for x in (first, second):
        want = fpq.quantize(x, fpq.NVFP4)            # the regular entry point, caller workspace
        got = _noalloc(fpq, x)
        torch.cuda.synchronize()
        for w, g in zip(want, got):
            assert torch.equal(w, g)
    assert fpq.fpq_get_device_error() == 0


def test_noalloc_rejects_batch_over_limit(fpq):
    n = fpq.NOALLOC_NVFP4_MAX_BATCH + 1
    x = torch.zeros((n, 1, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpq.FpqError) as e:
        _noalloc(fpq, x)
    assert e.value.status == 1
