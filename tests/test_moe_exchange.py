"""Multi-rank plumbing of the MoE FP8 dispatch on CPU (gloo, world sizes 2
and 3): the counts all-gather, the segment arithmetic and the point-to-point
exchange of ``mxfp8_block_scaled_warp_b200.moe``, with each rank's
expert-major send buffer built by the oracle (the CUDA kernels that build it
on a GPU are checked against the same oracle in the GPU tests).  The
received buffers must equal the oracle's dispatch over all ranks, byte for
byte, and the segment plan must give the oracle's group offsets."""
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
                                          world, EXPERTS, None)
        _, recvs, rows = moe.segment_plan(counts_all, rank, world, EXPERTS)
        q.put((rank, codes.numpy(), scales.numpy(), rows, recvs))
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
        rank, codes, scales, rows, recvs = q.get(timeout=180)
        got[rank] = (codes, scales, rows, recvs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    xs, ids = _inputs(world)
    want = oracle.moe_dispatch(xs, ids, EXPERTS)
    L = EXPERTS // world
    for r in range(world):
        codes, scales, rows, recvs = got[r]
        wq, ws, woff = want[r]
        assert rows == woff[-1]
        assert np.array_equal(codes, wq) and np.array_equal(scales, ws)
        # the first receive segment of each local expert starts at its group offset
        for l in range(L):
            segs = [seg for seg in recvs if seg[1] == r * L + l]
            if segs:
                assert segs[0][2] == woff[l]


def test_segment_plan_single_rank():
    sys.path.insert(0, ROOT)
    from mxfp8_block_scaled_warp_b200 import moe
    counts_all = torch.tensor([[2, 0, 3]], dtype=torch.int32)
    sends, recvs, rows = moe.segment_plan(counts_all, 0, 1, 3)
    assert sends == [(0, 0, 0, 2), (0, 2, 2, 3)]
    assert recvs == [(0, 0, 0, 2), (0, 2, 2, 3)]
    assert rows == 5


def _dispatch_worker(rank, world, port, q):
    """moe.dispatch on gloo ranks with its three device steps (route, layout,
    the quantize + pack kernel) stood in for by the oracle's definitions; the
    counts all-gather, the segment plan and the transfers run as written."""
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
