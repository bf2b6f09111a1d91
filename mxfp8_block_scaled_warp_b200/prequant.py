"""In-memory prequantization of a model state dict's routed MoE expert
projections to MXFP8 or NVFP4 ("fireworks-prequant 0.1.0", Quick start:
the in-memory hook; Formats).

Only the routed expert projections are quantized; every other tensor
(attention, dense MLP, router, shared experts, norms) passes through
unchanged, as the Formats section states for the serving precision policy.
Expert matrices of the same shape are stacked and quantized by one batched
call of the library's quantize kernel (the batch dimension carries one
E8M0/E4M3 scale grid, and for NVFP4 one tensor scale, per matrix).

Output names and dtypes per quantized ``<name>.weight``:

  MXFP8  ``<name>.weight``           float8_e4m3fn [N, K]
         ``<name>.weight_scale_inv`` uint8 (E8M0) [N, K/32]
  NVFP4  ``<name>.weight``           uint8 [N, K/2] (two E2M1 codes per byte, element 2i low nibble)
         ``<name>.weight_scale_inv`` float8_e4m3fn [N, K/16]
         ``<name>.weight_scale_2``   float32 scalar (the per-matrix tensor scale g)

All arithmetic runs in the CUDA library; this module only selects, stacks
and names tensors.
"""
from __future__ import annotations

import re
from collections import OrderedDict

import torch

from . import MXFP8, NVFP4, quantize

# model.layers.<l>.mlp.experts.<e>.{gate,up,down}_proj.weight, with any prefix
EXPERT_WEIGHT = re.compile(r"(?:^|\.)layers\.\d+\.mlp\.experts\.\d+\.(?:gate|up|down)_proj\.weight$")

FORMATS = {"mxfp8": MXFP8, "nvfp4": NVFP4}


def is_expert_weight(name: str) -> bool:
    """Whether `name` is a routed expert projection weight (quantized)."""
    return EXPERT_WEIGHT.search(name) is not None


def quantize_state_dict(state: "dict[str, torch.Tensor]", fmt: str = "mxfp8", device="cuda",
                        stream=None) -> "OrderedDict[str, torch.Tensor]":
    """Quantize the routed expert projections of `state` (bf16, any device)
    to `fmt` ("mxfp8" or "nvfp4") on `device`; return a new dict in the
    input's key order with the quantized tensors (on `device`) in place of
    the expert weights and every other tensor passed through unchanged."""
    if fmt not in FORMATS:
        raise ValueError(f"fmt must be one of {sorted(FORMATS)}, got {fmt!r}")
    code = FORMATS[fmt]
    groups: "OrderedDict[tuple, list[str]]" = OrderedDict()
    for name, t in state.items():
        if not is_expert_weight(name):
            continue
        if t.dtype != torch.bfloat16 or t.dim() != 2:
            raise TypeError(f"{name}: expert weights must be 2-D bf16, got {t.dtype} {tuple(t.shape)}")
        groups.setdefault(tuple(t.shape), []).append(name)

    done: "dict[str, dict[str, torch.Tensor]]" = {}
    for shape, names in groups.items():
        x = torch.stack([state[n] for n in names]).to(device, non_blocking=True)
        if code == MXFP8:
            q, s = quantize(x, code, stream)
            for i, n in enumerate(names):
                done[n] = {"weight": q[i].view(torch.float8_e4m3fn), "weight_scale_inv": s[i]}
        else:
            q, s, g = quantize(x, code, stream)
            for i, n in enumerate(names):
                done[n] = {"weight": q[i], "weight_scale_inv": s[i].view(torch.float8_e4m3fn),
                           "weight_scale_2": g[i]}
        del x

    out: "OrderedDict[str, torch.Tensor]" = OrderedDict()
    for name, t in state.items():
        if name in done:
            base = name[: -len("weight")]
            for suffix, v in done[name].items():
                out[base + suffix] = v
        else:
            out[name] = t
    return out
