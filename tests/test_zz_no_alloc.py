"""The non-allocating NVFP4 entry point.

Some callers cannot allocate device memory -- for example a plugin running
inside a serving runtime that owns the whole device memory pool -- and so
cannot supply the amax workspace the regular NVFP4 quantize call needs.
fpq_quantize_nvfp4_noalloc keeps that scratch in a static device array
inside the library instead.  These tests call it through the C ABI twice in
a row and check both results against the regular (workspace-taking) entry
point on the same inputs; the second call's input has a much smaller
magnitude than the first, so scratch left over from the first call would
show up in its tensor scales.  They also check that repeated calls change
neither the device's free memory nor torch's allocation count.

The file name sorts last so that pytest collects it after every other test:
a run that stops at the first failure has then already run the rest of the
suite if this file fails."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _outputs(x):
    b, r, c = x.shape
    return (torch.empty((b, r, c // 2), dtype=torch.uint8, device=x.device),
            torch.empty((b, r, c // 16), dtype=torch.uint8, device=x.device),
            torch.empty((b,), dtype=torch.float32, device=x.device))


def _noalloc(fpq, x, out=None):
    b, r, c = x.shape
    q, s, g = out if out is not None else _outputs(x)
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


def test_noalloc_allocates_nothing(fpq):
    """After a warm-up call (which looks up the scratch address), further
    calls leave the device's free memory and torch's allocations as they
    were: the outputs are the caller's, the scratch is the static array."""
    x = workloads.normal_bf16((4, 256, 1024), 1.0, seed=903).cuda()
    out = _outputs(x)
    _noalloc(fpq, x, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(5):
        _noalloc(fpq, x, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    assert fpq.fpq_get_device_error() == 0


def test_noalloc_rejects_batch_over_limit(fpq):
    n = fpq.NOALLOC_NVFP4_MAX_BATCH + 1
    x = torch.zeros((n, 1, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpq.FpqError) as e:
        _noalloc(fpq, x)
    assert e.value.status == 1
