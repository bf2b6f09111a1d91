"""Block-scaled FP8/FP4 quantization and block-scaled GEMM for B200 (sm_100a).

A thin ctypes binding over ``libfpq.so`` (C ABI: ``include/fpq.h``).  Every
step of the computation runs in the library's CUDA kernels; this module only
checks and marshals torch tensors (device memory, streams) into the C calls.
There is no CPU fallback: the first call (or ``load()``) raises ImportError
when ``libfpq.so`` is missing (build it with ``python -m
mxfp8_block_scaled_warp_b200.build``), and every call fails with
FPQ_ERR_UNSUPPORTED on a device that is not sm_100.

The ``fpq_*`` functions mirror the C entry points one to one (tensors in
place of pointers, the current torch stream by default).  ``quantize``,
``dequantize``, ``lora_merge_fakequant``, ``scaled_gemm`` and
``grouped_scaled_gemm`` are conveniences that allocate the outputs with
torch and call them.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "FP8_1x128", "FP8_128x128", "MXFP8", "NVFP4", "OUT_BF16", "OUT_F32", "FpqError", "lib_path", "load",
    "fpq_version", "fpq_quantize_workspace_bytes", "fpq_quantize_block", "fpq_dequantize",
    "fpq_lora_merge_fakequant", "fpq_scaled_gemm", "fpq_scaled_gemm_nvfp4", "fpq_grouped_scaled_gemm",
    "fpq_get_device_error", "fpq_gemm_bf16", "fpq_gemm_bf16_layout", "fpq_transpose_bf16",
    "fpq_gemm_bf16_splitk_workspace_bytes", "fpq_gemm_bf16_splitk", "fpq_qat_backward_workspace_bytes",
    "fpq_moe_route_workspace_bytes", "fpq_moe_route", "fpq_moe_dispatch_layout", "fpq_moe_dispatch_mxfp8",
    "fpq_moe_regroup",
    "fpq_quantize_block_strided", "fpq_dequantize_strided",
    "MOE_DIRECT", "MOE_PACK",
    "fpq_qat_backward", "fpq_qat_lora_grads", "fpq_qat_lora_grads_workspace_bytes",
    "fpq_quantize_nvfp4_noalloc", "NOALLOC_NVFP4_MAX_BATCH",
    "quantize", "dequantize", "lora_merge_fakequant", "scaled_gemm", "scaled_gemm_nvfp4", "grouped_scaled_gemm",
    "scale_shape", "code_shape", "gemm_bf16", "qat_backward",
]

FP8_1x128, FP8_128x128, MXFP8, NVFP4 = 0, 1, 2, 3
OUT_BF16, OUT_F32 = 0, 1
STATUS = {0: "FPQ_OK", 1: "FPQ_ERR_INVALID_ARG", 2: "FPQ_ERR_ALIGNMENT", 3: "FPQ_ERR_UNSUPPORTED",
          4: "FPQ_ERR_CUDA", 5: "FPQ_ERR_DEVICE_TIMEOUT", 6: "FPQ_ERR_DEVICE_BAD_INPUT",
          7: "FPQ_ERR_WORKSPACE"}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libfpq.so")


class FpqError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({detail})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libfpq.so (once); ImportError if it has not been built."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _load() -> ctypes.CDLL:
    if not os.path.exists(lib_path):
        raise ImportError(f"{lib_path} is not built; run `python -m mxfp8_block_scaled_warp_b200.build`")
    L = ctypes.CDLL(lib_path)
    P, I64, I32, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    sig = {
        "fpq_version": (I32, []),
        "fpq_status_string": (ctypes.c_char_p, [I32]),
        "fpq_last_error_detail": (ctypes.c_char_p, []),
        "fpq_last_cuda_error": (ctypes.c_char_p, []),
        "fpq_quantize_workspace_bytes": (SZ, [I32, I64]),
        "fpq_quantize_block": (I32, [I32, P, I64, I64, I64, P, P, P, P, SZ, P]),
        "fpq_dequantize": (I32, [I32, P, P, P, I64, I64, I64, P, P]),
        "fpq_lora_merge_fakequant": (I32, [P, P, P, I64, I64, I32, F, P, P, P, P]),
        "fpq_scaled_gemm": (I32, [I32, P, P, I32, P, P, I64, I64, I64, P, I32, P]),
        "fpq_scaled_gemm_nvfp4": (I32, [P, P, P, P, P, P, I64, I64, I64, P, I32, P]),
        "fpq_grouped_scaled_gemm": (I32, [I32, P, P, P, P, P, I32, I64, I64, I64, P, I32, P]),
        "fpq_get_device_error": (I32, [P, ctypes.POINTER(I32)]),
        "fpq_gemm_bf16": (I32, [P, P, I64, I64, I64, F, P, P]),
        "fpq_transpose_bf16": (I32, [P, P, I64, I64, P]),
        "fpq_gemm_bf16_layout": (I32, [P, I32, P, I32, I64, I64, I64, F, P, P]),
        "fpq_gemm_bf16_splitk_workspace_bytes": (SZ, [I64, I64, I64]),
        "fpq_gemm_bf16_splitk": (I32, [P, I32, P, I32, I64, I64, I64, F, P, P, SZ, P]),
        "fpq_qat_backward_workspace_bytes": (SZ, [I64, I64, I64, I32]),
        "fpq_qat_lora_grads_workspace_bytes": (SZ, [I64, I64, I32]),
        "fpq_qat_lora_grads": (I32, [P, P, P, I64, I64, I32, F, P, P, P, SZ, P]),
        "fpq_moe_route_workspace_bytes": (SZ, [I64, I32]),
        "fpq_quantize_block_strided": (I32, [I32, P, I64, I64, I64, I64, I64, P, I64, I64, P, P, P, SZ, P]),
        "fpq_dequantize_strided": (I32, [I32, P, I64, I64, P, P, I64, I64, I64, P, I64, I64, P]),
        "fpq_moe_route": (I32, [P, I64, I32, I32, P, P, SZ, P]),
        "fpq_moe_dispatch_layout": (I32, [P, I32, I32, I32, I32, P, P, P]),
        "fpq_moe_dispatch_mxfp8": (I32, [P, I64, I64, P, I32, I32, P, SZ, P, I32, P, P, P, P]),
        "fpq_moe_regroup": (I32, [P, P, P, I32, I32, I32, I64, I64, P, P, P]),
        "fpq_qat_backward": (I32, [P, P, P, P, P, I64, I64, I64, I32, F, P, P, P, P, P, SZ, P]),
        "fpq_quantize_nvfp4_noalloc": (I32, [P, I64, I64, I64, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise FpqError(status, where, load().fpq_last_error_detail().decode(errors="replace"))


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ---------------------------------------------------------------- raw C entry points

def fpq_version() -> int:
    return load().fpq_version()


def fpq_quantize_workspace_bytes(fmt: int, batch: int) -> int:
    return load().fpq_quantize_workspace_bytes(fmt, batch)


def fpq_quantize_block(fmt, x, batch, rows, cols, q, scales, tensor_scale=None, workspace=None, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_quantize_block(fmt, _ptr(x), batch, rows, cols, _ptr(q), _ptr(scales), _ptr(tensor_scale),
                                   _ptr(workspace), wsb, _stream(stream)), "fpq_quantize_block")


def fpq_dequantize(fmt, q, scales, tensor_scale, batch, rows, cols, out, stream=None):
    _check(load().fpq_dequantize(fmt, _ptr(q), _ptr(scales), _ptr(tensor_scale), batch, rows, cols, _ptr(out),
                               _stream(stream)), "fpq_dequantize")


def fpq_lora_merge_fakequant(w, lora_a, lora_b, n, k, r, alpha_over_r, wq, ws, w_fq=None, stream=None):
    _check(load().fpq_lora_merge_fakequant(_ptr(w), _ptr(lora_a), _ptr(lora_b), n, k, r, float(alpha_over_r),
                                         _ptr(wq), _ptr(ws), _ptr(w_fq), _stream(stream)),
           "fpq_lora_merge_fakequant")


def fpq_scaled_gemm(fmt_a, aq, as_, fmt_b, bq, bs, m, n, k, c, c_dtype, stream=None):
    _check(load().fpq_scaled_gemm(fmt_a, _ptr(aq), _ptr(as_), fmt_b, _ptr(bq), _ptr(bs), m, n, k, _ptr(c), c_dtype,
                                _stream(stream)), "fpq_scaled_gemm")


def fpq_scaled_gemm_nvfp4(aq, as_, ag, bq, bs, bg, m, n, k, c, c_dtype, stream=None):
    _check(load().fpq_scaled_gemm_nvfp4(_ptr(aq), _ptr(as_), _ptr(ag), _ptr(bq), _ptr(bs), _ptr(bg), m, n, k,
                                      _ptr(c), c_dtype, _stream(stream)), "fpq_scaled_gemm_nvfp4")


def fpq_gemm_bf16(p, q, m, n, k, alpha, c, stream=None):
    _check(load().fpq_gemm_bf16(_ptr(p), _ptr(q), m, n, k, float(alpha), _ptr(c), _stream(stream)), "fpq_gemm_bf16")


def fpq_gemm_bf16_layout(p, p_mn, q, q_mn, m, n, k, alpha, c, stream=None):
    _check(load().fpq_gemm_bf16_layout(_ptr(p), int(p_mn), _ptr(q), int(q_mn), m, n, k, float(alpha), _ptr(c),
                                       _stream(stream)), "fpq_gemm_bf16_layout")


def fpq_gemm_bf16_splitk_workspace_bytes(m: int, n: int, k: int) -> int:
    return load().fpq_gemm_bf16_splitk_workspace_bytes(m, n, k)


def fpq_gemm_bf16_splitk(p, p_mn, q, q_mn, m, n, k, alpha, c, workspace, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_gemm_bf16_splitk(_ptr(p), int(p_mn), _ptr(q), int(q_mn), m, n, k, float(alpha), _ptr(c),
                                       _ptr(workspace) if workspace is not None else None, wsb, _stream(stream)),
           "fpq_gemm_bf16_splitk")


def _ptr_rows(t: torch.Tensor | None):
    """Address of a row-strided view (rows may be apart; each row contiguous)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if t.stride(-1) != 1:
        raise ValueError("the last dimension must be contiguous")
    return t.data_ptr()


def fpq_quantize_block_strided(fmt, x, ld_x, bs_x, batch, rows, cols, q, ld_q, bs_q, scales, tensor_scale=None,
                               workspace=None, stream=None):
    """x, q: views whose first element is (0, 0, 0); strides in elements
    (NVFP4 codes: two per byte).  Scales dense."""
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_quantize_block_strided(fmt, _ptr_rows(x), ld_x, bs_x, batch, rows, cols, _ptr_rows(q), ld_q,
                                             bs_q, _ptr(scales), _ptr(tensor_scale), _ptr(workspace), wsb,
                                             _stream(stream)), "fpq_quantize_block_strided")


def fpq_dequantize_strided(fmt, q, ld_q, bs_q, scales, tensor_scale, batch, rows, cols, out, ld_out, bs_out,
                           stream=None):
    _check(load().fpq_dequantize_strided(fmt, _ptr_rows(q), ld_q, bs_q, _ptr(scales), _ptr(tensor_scale), batch,
                                         rows, cols, _ptr_rows(out), ld_out, bs_out, _stream(stream)),
           "fpq_dequantize_strided")


MOE_DIRECT, MOE_PACK = 0, 1


def fpq_moe_route_workspace_bytes(tokens: int, num_experts: int) -> int:
    return load().fpq_moe_route_workspace_bytes(tokens, num_experts)


def fpq_moe_route(topk_ids, tokens, topk, num_experts, counts, workspace, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_moe_route(_ptr(topk_ids) if tokens else None, tokens, topk, num_experts, _ptr(counts),
                                _ptr(workspace) if workspace is not None else None, wsb, _stream(stream)),
           "fpq_moe_route")


def fpq_moe_dispatch_layout(counts_all, world, num_experts, rank, mode, dst_row0, recv_offsets, stream=None):
    _check(load().fpq_moe_dispatch_layout(_ptr(counts_all), world, num_experts, rank, mode, _ptr(dst_row0),
                                          _ptr(recv_offsets), _stream(stream)), "fpq_moe_dispatch_layout")


def fpq_moe_dispatch_mxfp8(x, tokens, hidden, topk_ids, topk, num_experts, workspace, dst_row0, n_dest, dst_codes,
                           dst_scales, dst_capacity, stream=None):
    """dst_codes, dst_scales, dst_capacity: device int64 tensors of n_dest
    entries (buffer addresses, and rows per buffer)."""
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_moe_dispatch_mxfp8(_ptr(x), tokens, hidden, _ptr(topk_ids), topk, num_experts,
                                         _ptr(workspace) if workspace is not None else None, wsb, _ptr(dst_row0),
                                         n_dest, _ptr(dst_codes), _ptr(dst_scales), _ptr(dst_capacity),
                                         _stream(stream)), "fpq_moe_dispatch_mxfp8")


def fpq_moe_regroup(recv_codes, recv_scales, counts_all, world, num_experts, rank, hidden, rows, codes, scales,
                    stream=None):
    """Source-major received rows -> the expert-grouped receive layout."""
    if rows == 0:
        return
    _check(load().fpq_moe_regroup(_ptr(recv_codes), _ptr(recv_scales), _ptr(counts_all), world, num_experts, rank,
                                  hidden, rows, _ptr(codes), _ptr(scales), _stream(stream)), "fpq_moe_regroup")


def fpq_transpose_bf16(x, out, rows, cols, stream=None):
    _check(load().fpq_transpose_bf16(_ptr(x), _ptr(out), rows, cols, _stream(stream)), "fpq_transpose_bf16")


def fpq_qat_lora_grads_workspace_bytes(n: int, k: int, r: int) -> int:
    return load().fpq_qat_lora_grads_workspace_bytes(n, k, r)


def fpq_qat_lora_grads(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_qat_lora_grads(_ptr(dw), _ptr(lora_a), _ptr(lora_b), n, k, r, alpha_over_r, _ptr(da), _ptr(db),
                                     _ptr(workspace) if workspace is not None else None, wsb, _stream(stream)),
           "fpq_qat_lora_grads")


def fpq_qat_backward_workspace_bytes(m: int, n: int, k: int, r: int) -> int:
    return load().fpq_qat_backward_workspace_bytes(m, n, k, r)


def fpq_qat_backward(dy, x_fq, w_fq, lora_a, lora_b, m, n, k, r, alpha_over_r, dx, dw, da, db, workspace,
                     stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().fpq_qat_backward(_ptr(dy), _ptr(x_fq), _ptr(w_fq), _ptr(lora_a), _ptr(lora_b), m, n, k, r,
                                   float(alpha_over_r), _ptr(dx), _ptr(dw), _ptr(da), _ptr(db),
                                   _ptr(workspace) if workspace is not None else None, wsb, _stream(stream)),
           "fpq_qat_backward")


def fpq_grouped_scaled_gemm(fmt, aq, as_, bq, bs, group_offsets, groups, total_m, n, k, c, c_dtype, stream=None):
    _check(load().fpq_grouped_scaled_gemm(fmt, _ptr(aq), _ptr(as_), _ptr(bq), _ptr(bs), _ptr(group_offsets), groups,
                                        total_m, n, k, _ptr(c), c_dtype, _stream(stream)),
           "fpq_grouped_scaled_gemm")


def fpq_quantize_nvfp4_noalloc(x, batch, rows, cols, q, scales, tensor_scale, stream=None):
    """NVFP4 quantize without a workspace argument, for callers that cannot
    allocate: the library keeps the scratch in a static device array (at most
    NOALLOC_NVFP4_MAX_BATCH batch items; calls that overlap on the GPU race)."""
    _check(load().fpq_quantize_nvfp4_noalloc(_ptr(x), batch, rows, cols, _ptr(q), _ptr(scales), _ptr(tensor_scale),
                                           _stream(stream)), "fpq_quantize_nvfp4_noalloc")


NOALLOC_NVFP4_MAX_BATCH = 4096


def fpq_get_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load().fpq_get_device_error(_stream(stream), ctypes.byref(code)), "fpq_get_device_error")
    return code.value


# ---------------------------------------------------------------- allocating conveniences

def code_shape(fmt: int, shape) -> tuple:
    *lead, cols = shape
    return tuple(lead) + ((cols // 2,) if fmt == NVFP4 else (cols,))


def scale_shape(fmt: int, shape) -> tuple:
    *lead, rows, cols = shape
    if fmt == FP8_1x128:
        return tuple(lead) + (rows, cols // 128)
    if fmt == FP8_128x128:
        return tuple(lead) + ((rows + 127) // 128, cols // 128)
    if fmt == MXFP8:
        return tuple(lead) + (rows, cols // 32)
    if fmt == NVFP4:
        return tuple(lead) + (rows, cols // 16)
    raise ValueError(f"unknown format {fmt}")


def _scale_dtype(fmt):
    return torch.float32 if fmt in (FP8_1x128, FP8_128x128) else torch.uint8


def _brc(shape):
    if len(shape) == 2:
        return 1, shape[0], shape[1]
    if len(shape) == 3:
        return shape
    raise ValueError("expected a 2-D or 3-D tensor")


def quantize(x: torch.Tensor, fmt: int, stream=None):
    """bf16 [(B,) R, C] -> (codes, scales[, tensor_scale]) in the layouts of include/fpq.h."""
    if x.dtype != torch.bfloat16:
        raise TypeError("quantize expects bf16 input")
    b, r, c = _brc(x.shape)
    q = torch.empty(code_shape(fmt, x.shape), dtype=torch.uint8, device=x.device)
    s = torch.empty(scale_shape(fmt, x.shape), dtype=_scale_dtype(fmt), device=x.device)
    if fmt == NVFP4:
        g = torch.empty((b,), dtype=torch.float32, device=x.device)
        ws = torch.empty((max(1, fpq_quantize_workspace_bytes(fmt, b)) + 15) // 16 * 16, dtype=torch.uint8,
                         device=x.device)
        fpq_quantize_block(fmt, x, b, r, c, q, s, g, ws, stream)
        return q, s, g
    fpq_quantize_block(fmt, x, b, r, c, q, s, None, None, stream)
    return q, s


def dequantize(fmt: int, q: torch.Tensor, s: torch.Tensor, tensor_scale: torch.Tensor | None = None, stream=None):
    shape = tuple(q.shape[:-1]) + ((q.shape[-1] * 2,) if fmt == NVFP4 else (q.shape[-1],))
    b, r, c = _brc(shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
    fpq_dequantize(fmt, q, s, tensor_scale, b, r, c, out, stream)
    return out


def lora_merge_fakequant(w, lora_a, lora_b, alpha_over_r: float, want_fq: bool = False, stream=None):
    n, k = w.shape
    r = lora_a.shape[0]
    wq = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    ws = torch.empty(((n + 127) // 128, k // 128), dtype=torch.float32, device=w.device)
    w_fq = torch.empty((n, k), dtype=torch.bfloat16, device=w.device) if want_fq else None
    fpq_lora_merge_fakequant(w, lora_a, lora_b, n, k, r, alpha_over_r, wq, ws, w_fq, stream)
    return (wq, ws, w_fq) if want_fq else (wq, ws)


def scaled_gemm(fmt_a, aq, as_, fmt_b, bq, bs, out_dtype=torch.bfloat16, stream=None):
    m, k = aq.shape
    n = bq.shape[0]
    c = torch.empty((m, n), dtype=out_dtype, device=aq.device)
    fpq_scaled_gemm(fmt_a, aq, as_, fmt_b, bq, bs, m, n, k, c, OUT_F32 if out_dtype == torch.float32 else OUT_BF16,
                    stream)
    return c


def scaled_gemm_nvfp4(aq, as_, ag, bq, bs, bg, out_dtype=torch.bfloat16, stream=None):
    """C = ag bg (A B^T) for NVFP4 operands as returned by quantize(x, NVFP4):
    aq [m, k/2] packed codes, as_ [m, k/16] E4M3 scales, ag a one-element
    fp32 tensor (likewise for B [n, k])."""
    m, k = aq.shape[0], aq.shape[1] * 2
    n = bq.shape[0]
    c = torch.empty((m, n), dtype=out_dtype, device=aq.device)
    fpq_scaled_gemm_nvfp4(aq, as_, ag, bq, bs, bg, m, n, k, c, OUT_F32 if out_dtype == torch.float32 else OUT_BF16,
                          stream)
    return c


def gemm_bf16(p, q, alpha: float = 1.0, stream=None):
    """C = alpha (P Q^T) for bf16 P [m, k] and Q [n, k]; C bf16 [m, n]."""
    m, k = p.shape
    n = q.shape[0]
    c = torch.empty((m, n), dtype=torch.bfloat16, device=p.device)
    fpq_gemm_bf16(p, q, m, n, k, alpha, c, stream)
    return c


def qat_backward(dy, x_fq, w_fq, lora_a, lora_b, alpha_over_r: float, stream=None):
    """Gradients of the QAT linear layer (straight-through estimator) for the
    output gradient dy [m, n]: returns (dx [m, k], dw [n, k], da [r, k],
    db [n, r]), all bf16."""
    m, n = dy.shape
    k = x_fq.shape[1]
    r = lora_a.shape[0]
    dev = dy.device
    dx = torch.empty((m, k), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((n, k), dtype=torch.bfloat16, device=dev)
    da = torch.empty((r, k), dtype=torch.bfloat16, device=dev)
    db = torch.empty((n, r), dtype=torch.bfloat16, device=dev)
    wsb = fpq_qat_backward_workspace_bytes(m, n, k, r)
    ws = torch.empty((wsb + 15) // 16 * 16, dtype=torch.uint8, device=dev) if wsb else None
    fpq_qat_backward(dy, x_fq, w_fq, lora_a, lora_b, m, n, k, r, alpha_over_r, dx, dw, da, db, ws, stream)
    return dx, dw, da, db


def grouped_scaled_gemm(fmt, aq, as_, bq, bs, group_offsets, out_dtype=torch.bfloat16, stream=None):
    total_m, k = aq.shape
    groups, n, _ = bq.shape
    c = torch.empty((total_m, n), dtype=out_dtype, device=aq.device)
    fpq_grouped_scaled_gemm(fmt, aq, as_, bq, bs, group_offsets, groups, total_m, n, k, c,
                            OUT_F32 if out_dtype == torch.float32 else OUT_BF16, stream)
    return c
