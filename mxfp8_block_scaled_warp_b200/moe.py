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
all-gathered, the kernel writes an expert-major send buffer (the rows bound
for rank p, experts [p L, (p + 1) L), are one contiguous run), one
all-to-all per tensor (codes, scales) with per-rank row counts moves every
run to its rank (NCCL over NVLink; no TMA of any kind touches a peer's
memory), and a kernel regroups the rows that arrived source-major into the
expert-then-source order.  Every step of the computation runs in the
library's kernels; this module allocates buffers and issues the collectives.
"""
from __future__ import annotations

from typing import NamedTuple

import torch
import torch.distributed as dist

from . import (MOE_DIRECT, MOE_PACK, fpq_moe_dispatch_layout, fpq_moe_dispatch_mxfp8, fpq_moe_regroup,
               fpq_moe_route, fpq_moe_route_workspace_bytes)

__all__ = ["Dispatched", "route", "dispatch", "split_sizes", "exchange_rows"]


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


_PTR_TABLES: dict = {}        # device pointer tables of destination buffer sets, by address


def _ptr_tables(buffers, dev):
    """Device arrays of the buffers' code and scale addresses and row
    capacities, built once per buffer set (a fresh set of addresses makes a
    new entry; a few recent sets are kept)."""
    key = (dev.index, tuple((c.data_ptr(), s.data_ptr(), c.shape[0]) for c, s in buffers))
    t = _PTR_TABLES.get(key)
    if t is None:
        if len(_PTR_TABLES) >= 16:
            _PTR_TABLES.pop(next(iter(_PTR_TABLES)))
        t = (torch.tensor([c.data_ptr() for c, _ in buffers], dtype=torch.int64, device=dev),
             torch.tensor([s.data_ptr() for _, s in buffers], dtype=torch.int64, device=dev),
             torch.tensor([c.shape[0] for c, _ in buffers], dtype=torch.int64, device=dev))
        _PTR_TABLES[key] = t
    return t


def _dispatch_into(x, topk_ids, num_experts, ws, dst_row0, buffers, stream=None):
    """Quantize + write every pair's row into `buffers` [(codes, scales)],
    expert e to buffers[e // (E / len(buffers))]."""
    tokens, topk = topk_ids.shape
    codes_p, scales_p, cap = _ptr_tables(buffers, x.device)
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
    counts_host = counts_all.cpu()           # row counts of the all-to-all (waits for the counts)
    codes, scales = exchange_rows(send_q, send_s, counts_host, rank, world, num_experts, group,
                                  counts_dev=counts_all, stream=stream)
    return Dispatched(codes, scales, offsets, counts_all)


def split_sizes(counts_all, rank: int, world: int, num_experts: int):
    """Host-side row counts of the all-to-all, from the all-gathered counts
    (int [world, E]): rows this rank sends to each rank (its experts' runs
    of the expert-major send buffer) and rows it receives from each rank."""
    c = [[int(v) for v in row] for row in counts_all.tolist()] if hasattr(counts_all, "tolist") else counts_all
    L = num_experts // world
    send = [sum(c[rank][p * L:(p + 1) * L]) for p in range(world)]
    recv = [sum(c[s][rank * L:(rank + 1) * L]) for s in range(world)]
    return send, recv


def exchange_rows(send_codes, send_scales, counts_all, rank: int, world: int, num_experts: int, group=None,
                  counts_dev=None, regroup=None, stream=None):
    """Move this rank's expert-major send rows to the experts' ranks: one
    all-to-all per tensor (each rank's run of rows to that rank), then the
    regroup of the rows received source-major into this rank's grouped
    buffer (expert-major; within an expert, source 0, 1, ...).
    `counts_all` (host, int [world, E]) gives the row counts; `counts_dev`
    is the same table on the device, read by the regroup kernel.  `regroup`
    replaces the device regroup step (same arguments as fpq_moe_regroup;
    used by CPU tests of the collective plumbing).  Works on any backend
    with all-to-all support (NCCL on GPUs, gloo on CPU tensors)."""
    send, recv = split_sizes(counts_all, rank, world, num_experts)
    hidden = send_codes.shape[1]
    rows = sum(recv)
    dev = send_codes.device
    recv_q = torch.empty((rows, hidden), dtype=torch.uint8, device=dev)
    recv_s = torch.empty((rows, send_scales.shape[1]), dtype=torch.uint8, device=dev)
    sent = sum(send)
    dist.all_to_all_single(recv_q, send_codes[:sent], recv, send, group=group)
    dist.all_to_all_single(recv_s, send_scales[:sent], recv, send, group=group)
    codes = torch.empty_like(recv_q)
    scales = torch.empty_like(recv_s)
    (regroup or fpq_moe_regroup)(recv_q, recv_s, counts_dev, world, num_experts, rank, hidden, rows, codes, scales,
                                 stream)
    return codes, scales
