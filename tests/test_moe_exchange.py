"""Multi-rank plumbing of the MoE FP8 dispatch on CPU (gloo, world sizes 2
and 3): the counts all-gather, the all-to-all row counts and the all-to-all
exchange of ``mxfp8_block_scaled_warp_b200.moe``, with each rank's
expert-major send buffer built by the oracle and the device regroup step
stood in for by its definition (``regroup_standin``; the CUDA kernels that
do both on a GPU are checked against the oracle in the GPU tests).  The
received buffers must equal the oracle's dispatch over all ranks, byte for
byte."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
EXPERTS, TOKENS, HIDDEN, TOPK = 12, 10, 64, 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world):
    sys.path.insert(0, ROOT)
    import workloads
    xs, ids = [], []
    for s in range(world):
        t = TOKENS + 3 * s                                # unequal token counts per rank
        xs.append(workloads.as_u16(workloads.normal_bf16((t, HIDDEN), 1.0, seed=700 + s)))
        ids.append(workloads.route_choices(t, EXPERTS, TOPK, seed=710 + s).numpy())
    return xs, ids


def regroup_standin(recv_q, recv_s, counts_dev, world, experts, rank, hidden, rows, codes, scales, stream=None):
    """fpq_moe_regroup by its definition: rows that arrived source-major
    (source 0's rows for this rank's experts, expert-major, then source 1's,
    ...) into expert-major order, sources in order within an expert."""
    c = np.asarray(counts_dev, np.int64)
    L = experts // world
    start, a = {}, 0
    for s in range(world):
        for l in range(L):
            start[(l, s)] = a
            a += int(c[s][rank * L + l])
    d = 0
    for l in range(L):
        for s in range(world):
            n = int(c[s][rank * L + l])
            codes[d:d + n] = recv_q[start[(l, s)]:start[(l, s)] + n]
            scales[d:d + n] = recv_s[start[(l, s)]:start[(l, s)] + n]
            d += n
    assert d == rows


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from mxfp8_block_scaled_warp_b200 import moe
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        xs, ids = _inputs(world)
        counts, _ = oracle.moe_route_plan(ids[rank], EXPERTS)
        parts = [torch.zeros(EXPERTS, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(counts.astype(np.int32)))
        counts_all = torch.stack(parts)
        send_q, send_s, _ = oracle.moe_dispatch([xs[rank]], [ids[rank]], EXPERTS)[0]   # expert-major pack
        codes, scales = moe.exchange_rows(torch.from_numpy(send_q), torch.from_numpy(send_s), counts_all, rank,
                                          world, EXPERTS, None, counts_dev=counts_all, regroup=regroup_standin)
        q.put((rank, codes.numpy(), scales.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_matches_oracle_dispatch(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, codes, scales = q.get(timeout=180)
        got[rank] = (codes, scales)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    xs, ids = _inputs(world)
    want = oracle.moe_dispatch(xs, ids, EXPERTS)
    for r in range(world):
        codes, scales = got[r]
        wq, ws, woff = want[r]
        assert codes.shape[0] == woff[-1]
        assert np.array_equal(codes, wq) and np.array_equal(scales, ws)


def _dispatch_worker(rank, world, port, q):
    """moe.dispatch on gloo ranks with its four device steps (route, layout,
    the quantize + pack kernel, the regroup) stood in for by their
    definitions; the counts all-gather, the row counts and the all-to-all
    transfers run as written."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    import workloads
    from mxfp8_block_scaled_warp_b200 import moe

    def fake_route(topk_ids, num_experts, stream=None):
        counts, _ = oracle.moe_route_plan(topk_ids.numpy(), num_experts)
        return torch.from_numpy(counts.astype(np.int32)), None

    def fake_layout(counts_all, world_, num_experts, rank_, mode, dst_row0, offsets, stream=None):
        c = counts_all.numpy().astype(np.int64)
        L = num_experts // world_
        assert mode == moe.MOE_PACK
        dst_row0.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(c[rank_])[:-1]])))
        tot = c.sum(axis=0)[rank_ * L:(rank_ + 1) * L]
        offsets.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(tot)]).astype(np.int32)))

    def fake_pack(x, topk_ids, num_experts, ws, dst_row0, buffers, stream=None):
        q, s, _ = oracle.moe_dispatch([workloads.as_u16(x)], [topk_ids.numpy()], num_experts)[0]
        buffers[0][0].copy_(torch.from_numpy(q))
        buffers[0][1].copy_(torch.from_numpy(s))

    moe.route, moe.fpq_moe_dispatch_layout, moe._dispatch_into = fake_route, fake_layout, fake_pack
    moe.fpq_moe_regroup = regroup_standin
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        xs, ids = _inputs(world)
        d = moe.dispatch(workloads.from_u16(xs[rank]), torch.from_numpy(ids[rank].astype(np.int32)), EXPERTS,
                         group=dist.group.WORLD)
        q.put((rank, d.codes.numpy(), d.scales.numpy(), d.group_offsets.numpy(), d.counts_all.numpy()))
    finally:
        dist.destroy_process_group()


def test_dispatch_orchestration_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dispatch_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, rest) for r, *rest in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    xs, ids = _inputs(world)
    want = oracle.moe_dispatch(xs, ids, EXPERTS)
    counts = np.stack([oracle.moe_route_plan(i, EXPERTS)[0] for i in ids])
    for r in range(world):
        codes, scales, offs, counts_all = got[r]
        assert np.array_equal(codes, want[r][0]) and np.array_equal(scales, want[r][1])
        assert np.array_equal(offs, want[r][2])
        assert np.array_equal(counts_all, counts)
