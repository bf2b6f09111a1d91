"""MoE FP8 dispatch ("DeepSeek-V3 Blog 5: Low-Precision Training", Reducing
Communication Overhead in MoE with FP8: token activations are quantized to
FP8 before they are sent to the GPUs that hold their experts).

``dispatch`` quantizes every token row once to MXFP8 (E4M3 codes, E8M0 scale
per 32) and places one copy per chosen expert in the receive buffer of the
expert's rank, grouped by local expert: the ``aq``/``as`` operands of
``grouped_scaled_gemm(MXFP8, ...)`` with ``group_offsets``.  Row order: a
rank's local experts in order; each expert's rows from source rank 0, 1, ...;
from one source, its (token, choice) pairs in token order, then choice order.

One rank (or no process group): the fused kernel writes the rows straight
into the grouped buffer.  Several ranks: the per-expert counts are
all-gathered, the kernel writes an expert-major send buffer, and one
point-to-point transfer per (expert, peer) segment (NCCL over NVLink; no TMA
of any kind touches a peer's memory) lands each segment at its row in the
receiver's buffer.  Every step of the computation runs in the library's
kernels; this module allocates buffers and moves segments.
"""
from __future__ import annotations

from typing import NamedTuple

import torch
import torch.distributed as dist

from . import (MOE_DIRECT, MOE_PACK, fpq_moe_dispatch_layout, fpq_moe_dispatch_mxfp8, fpq_moe_route,
               fpq_moe_route_workspace_bytes)

__all__ = ["Dispatched", "route", "dispatch", "segment_plan", "exchange_rows"]


class Dispatched(NamedTuple):
    codes: torch.Tensor          # uint8 [rows, hidden] E4M3
    scales: torch.Tensor         # uint8 [rows, hidden / 32] E8M0
    group_offsets: torch.Tensor  # int32 [L + 1] on the device: local expert l owns rows [off[l], off[l + 1])
    counts_all: torch.Tensor     # int32 [world, E] on the device: pairs of source s routed to expert e


def route(topk_ids: torch.Tensor, num_experts: int, stream=None):
    """Per-expert pair counts of this rank (int32 [E], device) and the
    workspace holding the slot bases that ``fpq_moe_dispatch_mxfp8`` reads."""
    tokens, topk = topk_ids.shape
    dev = topk_ids.device
    counts = torch.empty((num_experts,), dtype=torch.int32, device=dev)
    wsb = fpq_moe_route_workspace_bytes(tokens, num_experts)
    ws = torch.empty(((wsb + 15) // 16 * 16,), dtype=torch.uint8, device=dev)
    fpq_moe_route(topk_ids, tokens, topk, num_experts, counts, ws, stream)
    return counts, ws


def _dispatch_into(x, topk_ids, num_experts, ws, dst_row0, buffers, stream=None):
    """Quantize + write every pair's row into `buffers` [(codes, scales)],
    expert e to buffers[e // (E / len(buffers))]."""
    tokens, topk = topk_ids.shape
    dev = x.device
    codes_p = torch.tensor([c.data_ptr() for c, _ in buffers], dtype=torch.int64, device=dev)
    scales_p = torch.tensor([s.data_ptr() for _, s in buffers], dtype=torch.int64, device=dev)
    cap = torch.tensor([c.shape[0] for c, _ in buffers], dtype=torch.int64, device=dev)
    fpq_moe_dispatch_mxfp8(x, tokens, x.shape[1], topk_ids, topk, num_experts, ws, dst_row0, len(buffers),
                           codes_p, scales_p, cap, stream)


def dispatch(x: torch.Tensor, topk_ids: torch.Tensor, num_experts: int, group=None, stream=None) -> Dispatched:
    """x bf16 [tokens, hidden] (hidden a multiple of 32) and topk_ids int32
    [tokens, k] on this rank's GPU; returns this rank's expert-grouped MXFP8
    rows.  With a process group of several ranks the call is collective."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or topk_ids.dtype != torch.int32 or topk_ids.dim() != 2:
        raise ValueError("need x bf16 [tokens, hidden] and topk_ids int32 [tokens, k]")
    tokens, hidden = x.shape
    world = 1 if group is None else dist.get_world_size(group)
    rank = 0 if group is None else dist.get_rank(group)
    if num_experts % world:
        raise ValueError("the number of experts must be a multiple of the number of ranks")
    dev = x.device
    L = num_experts // world
    counts, ws = route(topk_ids, num_experts, stream)
    dst_row0 = torch.empty((num_experts,), dtype=torch.int64, device=dev)
    offsets = torch.empty((L + 1,), dtype=torch.int32, device=dev)
    u8 = dict(dtype=torch.uint8, device=dev)
    if world == 1:
        counts_all = counts.view(1, num_experts)
        fpq_moe_dispatch_layout(counts_all, 1, num_experts, 0, MOE_DIRECT, dst_row0, offsets, stream)
        rows = tokens * topk_ids.shape[1]
        codes, scales = torch.empty((rows, hidden), **u8), torch.empty((rows, hidden // 32), **u8)
        _dispatch_into(x, topk_ids, num_experts, ws, dst_row0, [(codes, scales)], stream)
        return Dispatched(codes, scales, offsets, counts_all)
    counts_flat = torch.empty((world * num_experts,), dtype=torch.int32, device=dev)
    dist.all_gather_into_tensor(counts_flat, counts, group=group)     # flat output: every backend takes it
    counts_all = counts_flat.view(world, num_experts)
    fpq_moe_dispatch_layout(counts_all, world, num_experts, rank, MOE_PACK, dst_row0, offsets, stream)
    rows = tokens * topk_ids.shape[1]
    send_q, send_s = torch.empty((rows, hidden), **u8), torch.empty((rows, hidden // 32), **u8)
    _dispatch_into(x, topk_ids, num_experts, ws, dst_row0, [(send_q, send_s)], stream)
    counts_host = counts_all.cpu()           # segment sizes for the transfers (waits for the counts)
    codes, scales = exchange_rows(send_q, send_s, counts_host, rank, world, num_experts, group)
    return Dispatched(codes, scales, offsets, counts_all)


def segment_plan(counts_all, rank: int, world: int, num_experts: int):
    """Host-side row arithmetic of the exchange, from the all-gathered counts
    (int [world, E]): the send segments of this rank ([(peer, expert, first
    row in the expert-major send buffer, rows)]), the receive segments
    ([(source, expert, first row in this rank's grouped buffer, rows)]) and
    this rank's receive row count."""
    c = [[int(v) for v in row] for row in counts_all.tolist()] if hasattr(counts_all, "tolist") else counts_all
    L = num_experts // world
    sends, row = [], 0
    for e in range(num_experts):
        if c[rank][e]:
            sends.append((e // L, e, row, c[rank][e]))
        row += c[rank][e]
    recvs, row = [], 0
    for e in range(rank * L, (rank + 1) * L):
        for s in range(world):
            if c[s][e]:
                recvs.append((s, e, row, c[s][e]))
            row += c[s][e]
    return sends, recvs, row


def exchange_rows(send_codes, send_scales, counts_all, rank: int, world: int, num_experts: int, group=None):
    """Move every (expert, source) segment of the expert-major send buffers to
    the expert's rank, at its row in that rank's grouped buffer.  Segments
    for this rank are copied locally; the others go as one send and one
    receive per segment and tensor, matched by (source, expert) order on both
    sides.  Works on any backend with point-to-point support (NCCL on GPUs,
    gloo on CPU tensors)."""
    sends, recvs, rows = segment_plan(counts_all, rank, world, num_experts)
    hidden = send_codes.shape[1]
    codes = torch.empty((rows, hidden), dtype=torch.uint8, device=send_codes.device)
    scales = torch.empty((rows, send_scales.shape[1]), dtype=torch.uint8, device=send_codes.device)
    ops = []
    local = {}
    for peer, e, r0, n in sends:
        if peer == rank:
            local[e] = (r0, n)
            continue
        ops.append(dist.P2POp(dist.isend, send_codes[r0:r0 + n], dist.get_global_rank(group, peer)
                              if group is not None else peer, group))
        ops.append(dist.P2POp(dist.isend, send_scales[r0:r0 + n], dist.get_global_rank(group, peer)
                              if group is not None else peer, group))
    for src, e, r0, n in recvs:
        if src == rank:
            s0, _ = local[e]
            codes[r0:r0 + n].copy_(send_codes[s0:s0 + n])
            scales[r0:r0 + n].copy_(send_scales[s0:s0 + n])
            continue
        ops.append(dist.P2POp(dist.irecv, codes[r0:r0 + n], dist.get_global_rank(group, src)
                              if group is not None else src, group))
        ops.append(dist.P2POp(dist.irecv, scales[r0:r0 + n], dist.get_global_rank(group, src)
                              if group is not None else src, group))
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()
    return codes, scales
