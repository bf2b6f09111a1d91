"""The C ABI library loads, exports every entry point include/fpq.h declares,
and validates arguments on the host (no kernel launches, no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fpq.h")


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FPQ_API\s+[\w\s\*]+?\b(fpq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from mxfp8_block_scaled_warp_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_five_operations():
    names = declared_entry_points()
    for op in ("fpq_quantize_block", "fpq_dequantize", "fpq_lora_merge_fakequant", "fpq_scaled_gemm",
               "fpq_grouped_scaled_gemm"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    _, path = lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(fpq_\w+)", out))
    missing = [n for n in declared_entry_points() if n not in exported]
    assert not missing, missing
    # nothing beyond the header leaks out
    assert exported == set(declared_entry_points())


def test_host_side_validation(lib):
    L, _ = lib
    import mxfp8_block_scaled_warp_b200 as f
    P = ctypes.c_void_p
    L.fpq_quantize_block.restype = ctypes.c_int32
    L.fpq_quantize_block.argtypes = [ctypes.c_int32, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                     P, P, P, P, ctypes.c_size_t, P]
    ok_ptr = 1 << 20                         # aligned, never dereferenced: validation fails first
    # null input
    assert L.fpq_quantize_block(f.MXFP8, None, 1, 1, 32, ok_ptr, ok_ptr, None, None, 0, None) == 1
    # cols not a multiple of the block
    assert L.fpq_quantize_block(f.MXFP8, ok_ptr, 1, 1, 48, ok_ptr, ok_ptr, None, None, 0, None) == 1
    assert L.fpq_quantize_block(f.FP8_1x128, ok_ptr, 1, 1, 96, ok_ptr, ok_ptr, None, None, 0, None) == 1
    # misaligned pointer
    assert L.fpq_quantize_block(f.MXFP8, ok_ptr + 2, 1, 1, 32, ok_ptr, ok_ptr, None, None, 0, None) == 2
    # NVFP4 without workspace
    assert L.fpq_quantize_block(f.NVFP4, ok_ptr, 1, 1, 32, ok_ptr, ok_ptr, ok_ptr, None, 0, None) == 7
    # unknown format
    assert L.fpq_quantize_block(9, ok_ptr, 1, 1, 32, ok_ptr, ok_ptr, None, None, 0, None) == 1
    assert L.fpq_last_error_detail
    L.fpq_scaled_gemm.restype = ctypes.c_int32
    L.fpq_scaled_gemm.argtypes = [ctypes.c_int32, P, P, ctypes.c_int32, P, P, ctypes.c_int64, ctypes.c_int64,
                                  ctypes.c_int64, P, ctypes.c_int32, P]
    assert L.fpq_scaled_gemm(f.MXFP8, ok_ptr, ok_ptr, f.MXFP8, ok_ptr, ok_ptr, 64, 256, 100, ok_ptr, 0, None) == 1
    assert L.fpq_scaled_gemm(f.MXFP8, ok_ptr, ok_ptr, f.MXFP8, ok_ptr, ok_ptr, 64, 250, 128, ok_ptr, 0, None) == 1


def test_moe_dispatch_host_side_validation(lib):
    L, _ = lib
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.fpq_moe_route.restype = I32
    L.fpq_moe_route.argtypes = [P, I64, I32, I32, P, P, ctypes.c_size_t, P]
    L.fpq_moe_dispatch_layout.restype = I32
    L.fpq_moe_dispatch_layout.argtypes = [P, I32, I32, I32, I32, P, P, P]
    L.fpq_moe_dispatch_mxfp8.restype = I32
    L.fpq_moe_dispatch_mxfp8.argtypes = [P, I64, I64, P, I32, I32, P, ctypes.c_size_t, P, I32, P, P, P, P]
    ok = 1 << 20
    assert L.fpq_moe_route(ok, 16, 33, 8, ok, ok, 1 << 20, None) == 1            # topk above 32
    assert L.fpq_moe_route(ok, 1 << 27, 32, 8, ok, ok, 1 << 30, None) == 1       # 2^32 pairs: int32 counts overflow
    assert L.fpq_moe_route(ok, 16, 2, 2048, ok, ok, 1 << 20, None) == 1          # too many experts
    assert L.fpq_moe_route(ok, 16, 2, 8, ok, None, 0, None) == 7                 # no workspace
    assert L.fpq_moe_dispatch_layout(ok, 3, 8, 0, 0, ok, ok, None) == 1          # world does not divide E
    assert L.fpq_moe_dispatch_layout(ok, 2, 8, 2, 0, ok, ok, None) == 1          # rank out of range
    assert L.fpq_moe_dispatch_layout(ok, 2, 8, 0, 5, ok, ok, None) == 1          # unknown mode
    assert L.fpq_moe_dispatch_mxfp8(ok, 16, 48, ok, 2, 8, ok, 1 << 20, ok, 1, ok, ok, ok, None) == 1  # hidden % 32
    assert L.fpq_moe_dispatch_mxfp8(ok, 16, 64, ok, 2, 8, ok, 1 << 20, ok, 3, ok, ok, ok, None) == 1  # n_dest ∤ E
    assert L.fpq_moe_dispatch_mxfp8(ok + 4, 16, 64, ok, 2, 8, ok, 1 << 20, ok, 1, ok, ok, ok, None) == 2


def test_no_device_is_unsupported_not_fallback(lib):
    """Valid arguments on a machine without a GPU: the call refuses with
    FPQ_ERR_UNSUPPORTED instead of computing anything on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; this checks the no-device path")
    L, _ = lib
    import mxfp8_block_scaled_warp_b200 as f
    P = ctypes.c_void_p
    ok_ptr = 1 << 20
    st = L.fpq_quantize_block(f.MXFP8, P(ok_ptr), ctypes.c_int64(1), ctypes.c_int64(1), ctypes.c_int64(32),
                              P(ok_ptr), P(ok_ptr), None, None, ctypes.c_size_t(0), None)
    assert st == 3


def test_status_strings(lib):
    L, _ = lib
    L.fpq_status_string.restype = ctypes.c_char_p
    for code in range(8):
        assert L.fpq_status_string(code)
    L.fpq_version.restype = ctypes.c_int32
    assert L.fpq_version() >= 10000


def test_nvfp4_workspace_size(lib):
    """NVFP4 needs a 64-bit work counter (16 bytes with padding) plus an amax
    word and a progress counter per matrix; the other formats need none."""
    L, _ = lib
    import mxfp8_block_scaled_warp_b200 as f
    L.fpq_quantize_workspace_bytes.restype = ctypes.c_size_t
    L.fpq_quantize_workspace_bytes.argtypes = [ctypes.c_int32, ctypes.c_int64]
    for b in (1, 2, 64, 4096):
        assert L.fpq_quantize_workspace_bytes(f.NVFP4, b) == 16 + 8 * b
    assert L.fpq_quantize_workspace_bytes(f.NVFP4, 0) == 0
    for fmt in (f.MXFP8, f.FP8_1x128, f.FP8_128x128):
        assert L.fpq_quantize_workspace_bytes(fmt, 8) == 0
