"""Seeded synthetic inputs for the five workloads.

This module holds no quantization or GEMM arithmetic: it only draws seeded
random tensors (torch CPU generators, fp32 normals cast to bf16 with
round-to-nearest-even) and the MoE routing of the grouped-GEMM workload.
Both the CUDA path's tests/benchmark and the CPU oracle take their inputs
from here, so the two sides see the same bytes.

Recipe (seed = 1000 * workload + tensor index unless stated):

  mxfp8_256x512   B [256, 512] ~ N(0, 0.02) with 1 % of entries (rand < 0.01,
                  drawn after the normals) multiplied by 50, seed 0; A [64, 512]
                  same law, seed 1.  MXFP8 quant/dequant of B; 64x256x512 GEMM.
  ds_fp8_gemm     A [4096, 7168] ~ N(0, 1) (1x128 tiles); B [2048, 7168] ~ N(0, 0.02)
                  (128x128 blocks), B stored [N, K].
  qat_forward     W [2048, 7168] ~ N(0, 0.02); LoRA A [16, 7168] ~ N(0, 0.01),
                  LoRA B [2048, 16] ~ N(0, 0.01), alpha = 32, r = 16;
                  X [8192, 7168] ~ N(0, 1).
  moe_prequant    64 experts x {gate [2048, 7168], up [2048, 7168],
                  down [7168, 2048]} ~ N(0, 0.02); matrix i has seed 4000 + i,
                  i = 3 * expert + {0: gate, 1: up, 2: down}.
  moe_grouped     X [16384, 7168] ~ N(0, 1) (seed 5000); each token picks 8
                  distinct experts of 64 by Gumbel-top-8 on log((e+1)^-1.1)
                  (seed 5001); rows are gathered by expert, then by token;
                  W [64, 2048, 7168] ~ N(0, 0.02), expert e with seed 5100 + e.
  moe_dispatch    per source rank s: X_s [16384, 7168] ~ N(0, 1) (seed 5000 + 10 s)
                  and its top-8 of 64 experts as above (seed 5001 + 10 s), kept as
                  the [tokens, 8] choice matrix, highest score first.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "normal_bf16", "as_u16", "from_u16", "route_choices", "route_topk", "WORKLOADS",
    "mxfp8_256x512", "ds_fp8_gemm", "qat_forward", "moe_prequant_matrix", "moe_grouped", "moe_dispatch",
]


def normal_bf16(shape, std: float, seed: int, outlier_frac: float = 0.0,
                outlier_mult: float = 50.0) -> torch.Tensor:
    """N(0, std^2) in fp32 from a seeded CPU generator, optional outliers
    (entries with U(0,1) < outlier_frac, drawn after the normals, scaled by
    outlier_mult), cast to bf16 (round-to-nearest-even)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32) * std
    if outlier_frac > 0.0:
        u = torch.rand(*shape, generator=g, dtype=torch.float32)
        x = torch.where(u < outlier_frac, x * outlier_mult, x)
    return x.to(torch.bfloat16)


def as_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns (copy on host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_u16(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


# ---------------------------------------------------------------- workloads

def mxfp8_256x512():
    return {
        "b": normal_bf16((256, 512), 0.02, seed=0, outlier_frac=0.01),
        "a": normal_bf16((64, 512), 0.02, seed=1, outlier_frac=0.01),
    }


def ds_fp8_gemm(m: int = 4096, n: int = 2048, k: int = 7168):
    return {
        "a": normal_bf16((m, k), 1.0, seed=2000),
        "b": normal_bf16((n, k), 0.02, seed=2001),
    }


def qat_forward(m: int = 8192, n: int = 2048, k: int = 7168, r: int = 16, alpha: float = 32.0):
    return {
        "w": normal_bf16((n, k), 0.02, seed=3000),
        "lora_a": normal_bf16((r, k), 0.01, seed=3001),
        "lora_b": normal_bf16((n, r), 0.01, seed=3002),
        "x": normal_bf16((m, k), 1.0, seed=3003),
        "alpha_over_r": alpha / r,
    }


MOE_EXPERTS = 64
MOE_HIDDEN = 7168
MOE_INTER = 2048


def moe_prequant_matrix(i: int) -> torch.Tensor:
    """Matrix i of the expert prequant workload (3 per expert: gate, up, down)."""
    kind = i % 3
    shape = (MOE_INTER, MOE_HIDDEN) if kind < 2 else (MOE_HIDDEN, MOE_INTER)
    return normal_bf16(shape, 0.02, seed=4000 + i)


def route_choices(tokens: int, experts: int = MOE_EXPERTS, topk: int = 8, zipf_s: float = 1.1,
                  seed: int = 5001) -> torch.Tensor:
    """[tokens, topk] int32: each token's `topk` distinct experts, drawn by
    Gumbel-top-k with expert popularity (e+1)^-s, highest score first."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    logw = -zipf_s * torch.log(torch.arange(1, experts + 1, dtype=torch.float64))
    u = torch.rand(tokens, experts, generator=g, dtype=torch.float64).clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    return torch.topk(logw[None, :] + gumbel, topk, dim=1).indices.to(torch.int32).contiguous()


def route_topk(tokens: int, experts: int = MOE_EXPERTS, topk: int = 8, zipf_s: float = 1.1,
               seed: int = 5001):
    """Gumbel-top-k routing with expert popularity (e+1)^-s: each token draws
    `topk` distinct experts (sampling without replacement, weights (e+1)^-s).
    Returns (perm_token [tokens*topk] int64: the token of each permuted row,
    offsets [experts+1] int32: expert e owns permuted rows [off[e], off[e+1]))."""
    choice = route_choices(tokens, experts, topk, zipf_s, seed).to(torch.int64)
    expert_of = choice.reshape(-1)
    token_of = torch.arange(tokens).repeat_interleave(topk)
    order = torch.argsort(expert_of * tokens + token_of)                        # by expert, then token
    counts = torch.bincount(expert_of, minlength=experts)
    offsets = torch.zeros(experts + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    return token_of[order].contiguous(), offsets.to(torch.int32)


def moe_grouped(tokens: int = 16384, experts: int = MOE_EXPERTS, n: int = MOE_INTER,
                k: int = MOE_HIDDEN, with_weights: bool = True):
    x = normal_bf16((tokens, k), 1.0, seed=5000)
    perm, offsets = route_topk(tokens, experts)
    out = {"x": x, "perm": perm, "offsets": offsets}
    if with_weights:
        out["w"] = torch.stack([normal_bf16((n, k), 0.02, seed=5100 + e) for e in range(experts)])
    return out


def moe_dispatch(tokens: int = 16384, experts: int = MOE_EXPERTS, k: int = MOE_HIDDEN, topk: int = 8,
                 world: int = 1):
    """Per source rank s: activations x_s bf16 [tokens, k] N(0,1) and its
    routing [tokens, topk] (Gumbel-top-k as route_choices); rank 0 of one
    rank is the moe_grouped tokens and routing."""
    xs = [normal_bf16((tokens, k), 1.0, seed=5000 + 10 * s) for s in range(world)]
    ids = [route_choices(tokens, experts, topk, seed=5001 + 10 * s) for s in range(world)]
    return {"x": xs, "topk_ids": ids}


WORKLOADS = {
    "mxfp8_256x512": "MXFP8 quantize+dequantize of bf16 256x512 + 64x256x512 MXFP8 GEMM",
    "ds_fp8_gemm": "1x128/128x128 FP8 quantize of A 4096x7168, B 2048x7168 + fp32-scaled GEMM",
    "qat_forward": "LoRA merge + 128x128 fake-quant of W 2048x7168, 1x128 of X 8192x7168 + GEMM",
    "moe_prequant": "64 experts x {gate, up 2048x7168; down 7168x2048} -> MXFP8 and NVFP4",
    "moe_grouped": "16384 tokens x 7168, top-8 of 64 experts, grouped MXFP8 GEMM N=2048",
    "moe_dispatch": "16384 tokens x 7168, top-8 of 64 experts: MXFP8 quantize + scatter by expert",
}
