"""Oracle: plain, slow CPU reference for block-scaled FP8/FP4 quantization
and the block-scaled GEMM.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library (``mxfp8_block_scaled_warp_b200``) and never imports it; the
CUDA library never imports this package.

All floating-point arithmetic lives in ``oracle.c`` (plain C, no fast-math,
no FMA contraction); this module marshals numpy arrays into it, and holds
the integer bookkeeping of the MoE dispatch (which rows go where).  What each
function computes, and which page passage it follows, is stated in
``oracle.c``.

Formats (``FMT_*``) and layouts:

=============  =========================  ===================================
format         codes                      scales
=============  =========================  ===================================
FMT_1x128      uint8 e4m3 [B, R, C]       fp32 [B, R, C/128]
FMT_128x128    uint8 e4m3 [B, R, C]       fp32 [B, ceil(R/128), C/128]
FMT_MXFP8      uint8 e4m3 [B, R, C]       uint8 E8M0 [B, R, C/32]
FMT_NVFP4      uint8 e2m1x2 [B, R, C/2]   uint8 e4m3 [B, R, C/16] + fp32 g[B]
=============  =========================  ===================================
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

FMT_1x128, FMT_128x128, FMT_MXFP8, FMT_NVFP4 = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Flags that keep every fp32 step a single IEEE binary32 operation.
CFLAGS = ["-O2", "-std=c11", "-Wall", "-Wextra", "-fno-fast-math", "-ffp-contract=off",
          "-fexcess-precision=standard", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I32, U8, U16, F, D, I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                          ctypes.c_uint8, ctypes.c_uint16, ctypes.c_float,
                                          ctypes.c_double, ctypes.c_int)
        sig = {
            "orc_bf16_decode": (D, [U16]),
            "orc_bf16_encode": (U16, [F]),
            "orc_e4m3_decode": (D, [U8]),
            "orc_e4m3_encode": (U8, [D]),
            "orc_e2m1_decode": (D, [U8]),
            "orc_e2m1_encode": (U8, [D]),
            "orc_e8m0_decode": (D, [U8]),
            "orc_mx_block_exponent": (I, [D]),
            "orc_nvfp4_tensor_scale": (F, [P, I64]),
            "orc_quant_mxfp8": (None, [P, I64, I64, I64, P, P]),
            "orc_quant_fp8_1x128": (None, [P, I64, I64, I64, P, P]),
            "orc_quant_fp8_128x128": (None, [P, I64, I64, I64, P, P]),
            "orc_quant_nvfp4": (None, [P, I64, I64, I64, P, P, P]),
            "orc_dequant_mxfp8": (None, [P, P, I64, I64, I64, P]),
            "orc_dequant_fp8_1x128": (None, [P, P, I64, I64, I64, P]),
            "orc_dequant_fp8_128x128": (None, [P, P, I64, I64, I64, P]),
            "orc_dequant_nvfp4": (None, [P, P, P, I64, I64, I64, P]),
            "orc_lora_merge": (None, [P, P, P, I64, I64, I32, F, P]),
            "orc_gemm_entry": (D, [I, P, P, P, I, P, P, P, I64, I64, I64, I64, I64]),
            "orc_gemm_entries": (None, [I, P, P, P, I, P, P, P, I64, I64, I64, P, P, I64, P]),
            "orc_gemm_full": (None, [I, P, P, P, I, P, P, P, I64, I64, I64, P]),
            "orc_grouped_gemm_entries": (None, [I, P, P, P, P, P, I32, I64, I64, I64, P, P, I64, P]),
            "orc_gemm_bf16_entries": (None, [P, P, I64, D, P, P, I64, P]),
            "orc_gemm_bf16_full": (None, [P, P, I64, I64, I64, D, P]),
            "orc_bf16_encode_f64": (U16, [D]),
            "orc_bf16_encode_f64_array": (None, [P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _bf16(x: np.ndarray) -> np.ndarray:
    """Accept bf16 bit patterns as uint16 (the oracle's input type)."""
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return x


def _brc(x: np.ndarray):
    if x.ndim == 2:
        return 1, x.shape[0], x.shape[1]
    assert x.ndim == 3
    return x.shape


# ---------------------------------------------------------------- element codecs

def bf16_decode(b: int) -> float:
    return lib().orc_bf16_decode(int(b))


def bf16_encode(v: float) -> int:
    return lib().orc_bf16_encode(float(v))


def e4m3_decode(c: int) -> float:
    return lib().orc_e4m3_decode(int(c))


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(v))


def e2m1_decode(c: int) -> float:
    return lib().orc_e2m1_decode(int(c))


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def e8m0_decode(c: int) -> float:
    return lib().orc_e8m0_decode(int(c))


def mx_block_exponent(amax: float) -> int:
    return lib().orc_mx_block_exponent(float(amax))


# ---------------------------------------------------------------- block quantizers

def quant_mxfp8(x: np.ndarray):
    """bf16 [.., R, C] -> (e4m3 codes [.., R, C], E8M0 scales [.., R, C/32])."""
    x = _bf16(x)
    b, r, c = _brc(x)
    assert c % 32 == 0
    q = np.empty(x.shape, np.uint8)
    s = np.empty(x.shape[:-1] + (c // 32,), np.uint8)
    lib().orc_quant_mxfp8(_p(x), b, r, c, _p(q), _p(s))
    return q, s


def quant_fp8_1x128(x: np.ndarray):
    """bf16 [.., R, C] -> (e4m3 codes [.., R, C], fp32 scales [.., R, C/128])."""
    x = _bf16(x)
    b, r, c = _brc(x)
    assert c % 128 == 0
    q = np.empty(x.shape, np.uint8)
    s = np.empty(x.shape[:-1] + (c // 128,), np.float32)
    lib().orc_quant_fp8_1x128(_p(x), b, r, c, _p(q), _p(s))
    return q, s


def quant_fp8_128x128(x: np.ndarray):
    """bf16 [.., R, C] -> (e4m3 codes [.., R, C], fp32 scales [.., ceil(R/128), C/128])."""
    x = _bf16(x)
    b, r, c = _brc(x)
    assert c % 128 == 0
    q = np.empty(x.shape, np.uint8)
    s = np.empty(x.shape[:-2] + ((r + 127) // 128, c // 128), np.float32)
    lib().orc_quant_fp8_128x128(_p(x), b, r, c, _p(q), _p(s))
    return q, s


def quant_nvfp4(x: np.ndarray):
    """bf16 [.., R, C] -> (packed e2m1 [.., R, C/2], e4m3 scales [.., R, C/16], fp32 g [B])."""
    x = _bf16(x)
    b, r, c = _brc(x)
    assert c % 16 == 0
    q = np.empty(x.shape[:-1] + (c // 2,), np.uint8)
    s = np.empty(x.shape[:-1] + (c // 16,), np.uint8)
    g = np.empty((b,), np.float32)
    lib().orc_quant_nvfp4(_p(x), b, r, c, _p(q), _p(s), _p(g))
    return q, s, g


def nvfp4_tensor_scale(x: np.ndarray) -> float:
    x = _bf16(x)
    return lib().orc_nvfp4_tensor_scale(_p(x), x.size)


# ---------------------------------------------------------------- dequantizers

def dequant_mxfp8(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    b, r, c = _brc(q)
    out = np.empty(q.shape, np.uint16)
    lib().orc_dequant_mxfp8(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(s)), b, r, c, _p(out))
    return out


def dequant_fp8_1x128(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    b, r, c = _brc(q)
    out = np.empty(q.shape, np.uint16)
    lib().orc_dequant_fp8_1x128(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(s, np.float32)),
                                b, r, c, _p(out))
    return out


def dequant_fp8_128x128(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    b, r, c = _brc(q)
    out = np.empty(q.shape, np.uint16)
    lib().orc_dequant_fp8_128x128(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(s, np.float32)),
                                  b, r, c, _p(out))
    return out


def dequant_nvfp4(q: np.ndarray, s: np.ndarray, g: np.ndarray) -> np.ndarray:
    b, r, half = _brc(q)
    c = 2 * half
    out = np.empty(q.shape[:-1] + (c,), np.uint16)
    lib().orc_dequant_nvfp4(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(s)),
                            _p(np.ascontiguousarray(g, np.float32)), b, r, c, _p(out))
    return out


# ---------------------------------------------------------------- LoRA merge (QAT forward)

def lora_merge(w: np.ndarray, lora_a: np.ndarray, lora_b: np.ndarray, alpha_over_r: float) -> np.ndarray:
    """W [N, K], A [r, K], B [N, r] (bf16 as uint16) -> merged bf16 W_eff [N, K]."""
    w, lora_a, lora_b = _bf16(w), _bf16(lora_a), _bf16(lora_b)
    n, k = w.shape
    r = lora_a.shape[0]
    assert lora_a.shape == (r, k) and lora_b.shape == (n, r)
    out = np.empty_like(w)
    lib().orc_lora_merge(_p(w), _p(lora_a), _p(lora_b), n, k, r, float(np.float32(alpha_over_r)), _p(out))
    return out


def lora_merge_fakequant(w, lora_a, lora_b, alpha_over_r):
    """Merge, then 128x128 quantize; returns (q, s, fake-quantized bf16 W)."""
    w_eff = lora_merge(w, lora_a, lora_b, alpha_over_r)
    q, s = quant_fp8_128x128(w_eff)
    return q, s, dequant_fp8_128x128(q, s)


# ---------------------------------------------------------------- GEMM reference

def _gemm_args(fmt, q, s, g):
    s = np.ascontiguousarray(s)
    g = None if g is None else np.ascontiguousarray(np.atleast_1d(g), np.float32)
    return fmt, _p(np.ascontiguousarray(q)), _p(s), _p(g), (q, s, g)


def _cols(fmt, q):
    return q.shape[-1] * (2 if fmt == FMT_NVFP4 else 1)


def gemm_full(fmt_a, aq, as_, fmt_b, bq, bs, ag=None, bg=None) -> np.ndarray:
    """fp64 C = deq(A) @ deq(B)^T, A [M, K], B [N, K]."""
    m, n, k = aq.shape[0], bq.shape[0], _cols(fmt_a, aq)
    fa, pa, psa, pga, keep_a = _gemm_args(fmt_a, aq, as_, ag)
    fb, pb, psb, pgb, keep_b = _gemm_args(fmt_b, bq, bs, bg)
    out = np.empty((m, n), np.float64)
    lib().orc_gemm_full(fa, pa, psa, pga, fb, pb, psb, pgb, m, n, k, _p(out))
    return out


def gemm_entries(fmt_a, aq, as_, fmt_b, bq, bs, rows, cols, ag=None, bg=None) -> np.ndarray:
    """fp64 entries C[rows[i], cols[i]] of deq(A) @ deq(B)^T."""
    m, n, k = aq.shape[0], bq.shape[0], _cols(fmt_a, aq)
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    fa, pa, psa, pga, keep_a = _gemm_args(fmt_a, aq, as_, ag)
    fb, pb, psb, pgb, keep_b = _gemm_args(fmt_b, bq, bs, bg)
    out = np.empty(rows.shape, np.float64)
    lib().orc_gemm_entries(fa, pa, psa, pga, fb, pb, psb, pgb, m, n, k,
                           _p(rows), _p(cols), rows.size, _p(out))
    return out


def grouped_gemm_entries(fmt, aq, as_, bq, bs, offsets, rows, cols) -> np.ndarray:
    """fp64 entries of the per-expert product: row r in [off[e], off[e+1]) uses B[e]."""
    aq, as_ = np.ascontiguousarray(aq), np.ascontiguousarray(as_)
    bq, bs = np.ascontiguousarray(bq), np.ascontiguousarray(bs)
    offsets = np.ascontiguousarray(offsets, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    groups, n, k = bq.shape
    out = np.empty(rows.shape, np.float64)
    lib().orc_grouped_gemm_entries(fmt, _p(aq), _p(as_), _p(bq), _p(bs), _p(offsets), groups,
                                   aq.shape[0], n, k, _p(rows), _p(cols), rows.size, _p(out))
    return out


def gemm_tolerance_ok(got: np.ndarray, ref: np.ndarray, rms_ref: float | None = None):
    """The GEMM acceptance test: |got - ref| <= 8e-3 |ref| + 1e-2 rms(ref),
    element-wise, rms taken over the whole reference output (or given).
    Returns (ok, worst ratio of error to bound)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if rms_ref is None else float(rms_ref)
    bound = 8e-3 * np.abs(ref) + 1e-2 * rms
    err = np.abs(got - ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
    return bool(np.all(err <= bound)), ratio


# ---------------------------------------------------------------- QAT backward (oracle.c, "QAT backward")

def gemm_bf16_full(p: np.ndarray, q: np.ndarray, alpha: float = 1.0) -> np.ndarray:
    """fp64 C = alpha * P Q^T, P [m, k], Q [n, k] bf16 (uint16)."""
    p, q = _bf16(p), _bf16(q)
    m, k = p.shape
    n = q.shape[0]
    assert q.shape[1] == k
    out = np.empty((m, n), np.float64)
    lib().orc_gemm_bf16_full(_p(p), _p(q), m, n, k, float(alpha), _p(out))
    return out


def gemm_bf16_entries(p: np.ndarray, q: np.ndarray, rows, cols, alpha: float = 1.0) -> np.ndarray:
    """fp64 entries alpha * (P Q^T)[rows[i], cols[i]]."""
    p, q = _bf16(p), _bf16(q)
    k = p.shape[1]
    assert q.shape[1] == k
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    out = np.empty(rows.shape[0], np.float64)
    lib().orc_gemm_bf16_entries(_p(p), _p(q), k, float(alpha), _p(rows), _p(cols), rows.shape[0], _p(out))
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 (ties to even) of fp64 values, as uint16 patterns."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_encode_f64_array(_p(x), x.size, _p(out))
    return out


def qat_backward(dy, x_fq, w_fq, lora_a, lora_b, alpha_over_r: float):
    """(dx, dw, da, db) in fp64 for the straight-through-estimator backward:
    dx = dy Wfq, dw = dy^T Xfq, da = (alpha/r) B^T bf16(dw),
    db = (alpha/r) bf16(dw) A^T.  Inputs bf16 as uint16; the transposes here
    only move data."""
    dy, x_fq, w_fq, lora_a, lora_b = (_bf16(t) for t in (dy, x_fq, w_fq, lora_a, lora_b))
    dx = gemm_bf16_full(dy, np.ascontiguousarray(w_fq.T))
    dw = gemm_bf16_full(np.ascontiguousarray(dy.T), np.ascontiguousarray(x_fq.T))
    dw16 = bf16_round(dw)
    da = gemm_bf16_full(np.ascontiguousarray(lora_b.T), np.ascontiguousarray(dw16.T), alpha_over_r)
    db = gemm_bf16_full(dw16, lora_a, alpha_over_r)
    return dx, dw, da, db


# ------------------------------------------------------------- MoE FP8 dispatch
#
# "DeepSeek-V3 Blog 5: Low-Precision Training", Reducing Communication
# Overhead in MoE with FP8: token activations are quantized to FP8 before
# they are sent to the GPUs that hold their experts.  The format is MXFP8
# (E4M3 codes, E8M0 scale per 32 elements), the input format of the grouped
# expert GEMM.  Only the bookkeeping below is written in Python (integers and
# data movement); every code and scale comes from quant_mxfp8 above.
#
# Reading of the order (the page fixes none): rank r of `world` owns experts
# [r L, (r + 1) L), L = E / world; its receive buffer holds the rows of its
# local experts in expert order, each expert's rows from source rank 0, 1, ...
# in turn, and within one source the pairs (token t, choice j) routed to that
# expert in token order, then choice order.


def moe_route_plan(topk_ids: np.ndarray, num_experts: int):
    """counts[e] = number of (token, choice) pairs routed to expert e, and
    slot[t, j] = the index of pair (t, j) among them, pairs numbered in token
    order, then choice order."""
    ids = np.asarray(topk_ids)
    tokens, k = ids.shape
    counts = np.zeros(num_experts, np.int64)
    slot = np.zeros((tokens, k), np.int64)
    for t in range(tokens):
        for j in range(k):
            e = int(ids[t, j])
            slot[t, j] = counts[e]
            counts[e] += 1
    return counts, slot


def moe_dispatch(xs, topk_ids_list, num_experts: int):
    """The FP8 dispatch over len(xs) ranks: xs[s] bf16 [T_s, K] (uint16) and
    topk_ids_list[s] int [T_s, k] are source rank s's activations and routing.
    Returns, per receiving rank r, (codes uint8 [rows_r, K], scales uint8 E8M0
    [rows_r, K/32], group_offsets int64 [L + 1]) with rows ordered as stated
    above; group_offsets[l] is the first row of local expert l."""
    world = len(xs)
    assert num_experts % world == 0
    L = num_experts // world
    quant = [quant_mxfp8(_bf16(x)) for x in xs]
    plans = [moe_route_plan(ids, num_experts) for ids in topk_ids_list]
    out = []
    for r in range(world):
        rows_q, rows_s, offsets = [], [], [0]
        for l in range(L):
            e = r * L + l
            for s in range(world):
                ids = np.asarray(topk_ids_list[s])
                _, slot = plans[s]
                # pairs of source s routed to e, placed by their slot
                seg = [None] * int(plans[s][0][e])
                for t in range(ids.shape[0]):
                    for j in range(ids.shape[1]):
                        if int(ids[t, j]) == e:
                            seg[int(slot[t, j])] = t
                for t in seg:
                    rows_q.append(quant[s][0][t])
                    rows_s.append(quant[s][1][t])
            offsets.append(len(rows_q))
        k_cols = quant[0][0].shape[1]
        codes = np.array(rows_q, np.uint8).reshape(-1, k_cols)
        scales = np.array(rows_s, np.uint8).reshape(-1, k_cols // 32)
        out.append((codes, scales, np.array(offsets, np.int64)))
    return out
