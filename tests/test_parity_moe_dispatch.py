"""GPU parity of the MoE FP8 dispatch ("DeepSeek-V3 Blog 5: Low-Precision
Training", Reducing Communication Overhead in MoE with FP8) against the
oracle, byte for byte: codes, E8M0 scales, row placement, group offsets and
counts.  Several source ranks are run on one GPU as one launch sequence each,
writing into every receiver's buffer (all buffers local); no kernel waits on
another."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

BAD_INPUT = 6          # FPQ_ERR_DEVICE_BAD_INPUT, read from the device error word


def _ids(tokens, experts, k, seed):
    return workloads.route_choices(tokens, experts, k, seed=seed)


def _x(tokens, hidden, seed):
    return workloads.normal_bf16((tokens, hidden), 1.0, seed=seed)


class Source:
    """One source rank's inputs on the GPU, routed."""

    def __init__(self, fpq, x, ids, experts):
        self.f, self.experts = fpq, experts
        self.x, self.ids = x.cuda(), ids.cuda()
        self.tokens, self.topk = ids.shape
        self.counts = torch.empty((experts,), dtype=torch.int32, device="cuda")
        wsb = fpq.fpq_moe_route_workspace_bytes(self.tokens, experts)
        self.ws = torch.empty(((wsb + 15) // 16 * 16,), dtype=torch.uint8, device="cuda")
        fpq.fpq_moe_route(self.ids, self.tokens, self.topk, experts, self.counts, self.ws)

    def dispatch(self, counts_all, world, rank, mode, buffers):
        f, E = self.f, self.experts
        dst_row0 = torch.empty((E,), dtype=torch.int64, device="cuda")
        offs = torch.empty((E // world + 1,), dtype=torch.int32, device="cuda")
        f.fpq_moe_dispatch_layout(counts_all, world, E, rank, mode, dst_row0, offs)
        qp = torch.tensor([q.data_ptr() for q, _ in buffers], dtype=torch.int64, device="cuda")
        sp = torch.tensor([s.data_ptr() for _, s in buffers], dtype=torch.int64, device="cuda")
        cap = torch.tensor([q.shape[0] for q, _ in buffers], dtype=torch.int64, device="cuda")
        f.fpq_moe_dispatch_mxfp8(self.x, self.tokens, self.x.shape[1], self.ids, self.topk, E, self.ws, dst_row0,
                                 len(buffers), qp, sp, cap)
        return offs


def _buffers(rows, hidden):
    return (torch.full((rows, hidden), 0xEE, dtype=torch.uint8, device="cuda"),
            torch.full((rows, hidden // 32), 0xEE, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("tokens,hidden,experts,k", [(1, 32, 1, 1), (7, 64, 8, 3), (100, 7168, 64, 8),
                                                     (5000, 512, 16, 4), (9500, 96, 64, 8), (300, 2048, 256, 6),
                                                     (50, 128, 64, 32), (200, 64, 1024, 4)])
def test_single_rank(fpq, orc, tokens, hidden, experts, k):
    x, ids = _x(tokens, hidden, 800 + tokens), _ids(tokens, experts, k, 801 + tokens)
    src = Source(fpq, x, ids, experts)
    buf = _buffers(tokens * k, hidden)
    offs = src.dispatch(src.counts.view(1, experts), 1, 0, fpq.MOE_DIRECT, [buf])
    wq, ws, woff = orc.moe_dispatch([workloads.as_u16(x)], [ids.numpy()], experts)[0]
    counts, _ = orc.moe_route_plan(ids.numpy(), experts)
    assert np.array_equal(src.counts.cpu().numpy(), counts)
    assert np.array_equal(offs.cpu().numpy(), woff)
    assert np.array_equal(buf[0].cpu().numpy(), wq)
    assert np.array_equal(buf[1].cpu().numpy(), ws)
    assert fpq.fpq_get_device_error() == 0


@pytest.mark.parametrize("world,experts,k", [(2, 8, 2), (4, 16, 4), (8, 64, 8)])
def test_virtual_ranks_direct(fpq, orc, world, experts, k):
    """Every source writes straight into every receiver's grouped buffer."""
    hidden = 256
    xs = [_x(40 + 17 * s, hidden, 820 + s) for s in range(world)]
    ids = [_ids(40 + 17 * s, experts, k, 830 + s) for s in range(world)]
    srcs = [Source(fpq, xs[s], ids[s], experts) for s in range(world)]
    counts_all = torch.stack([s.counts for s in srcs]).contiguous()
    want = orc.moe_dispatch([workloads.as_u16(x) for x in xs], [i.numpy() for i in ids], experts)
    bufs = [_buffers(int(want[r][2][-1]), hidden) for r in range(world)]
    for s in range(world):
        offs = srcs[s].dispatch(counts_all, world, s, fpq.MOE_DIRECT, bufs)
        assert np.array_equal(offs.cpu().numpy(), want[s][2])          # rank s's own group offsets
    for r in range(world):
        assert np.array_equal(bufs[r][0].cpu().numpy(), want[r][0])
        assert np.array_equal(bufs[r][1].cpu().numpy(), want[r][1])
    assert fpq.fpq_get_device_error() == 0


def test_pack_mode_is_expert_major(fpq, orc):
    """PACK: the send buffer is this rank's pairs expert-major in slot order
    (the oracle's single-rank layout), whatever the other ranks hold."""
    world, experts, k, hidden = 4, 16, 3, 128
    xs = [_x(30 + 11 * s, hidden, 850 + s) for s in range(world)]
    ids = [_ids(30 + 11 * s, experts, k, 860 + s) for s in range(world)]
    srcs = [Source(fpq, xs[s], ids[s], experts) for s in range(world)]
    counts_all = torch.stack([s.counts for s in srcs]).contiguous()
    want_recv = orc.moe_dispatch([workloads.as_u16(x) for x in xs], [i.numpy() for i in ids], experts)
    for s in range(world):
        buf = _buffers(ids[s].shape[0] * k, hidden)
        offs = srcs[s].dispatch(counts_all, world, s, fpq.MOE_PACK, [buf])
        wq, ws, _ = orc.moe_dispatch([workloads.as_u16(xs[s])], [ids[s].numpy()], experts)[0]
        assert np.array_equal(buf[0].cpu().numpy(), wq) and np.array_equal(buf[1].cpu().numpy(), ws)
        assert np.array_equal(offs.cpu().numpy(), want_recv[s][2])


def test_full_size_sampled(fpq, orc):
    """16384 tokens x 7168, top-8 of 64 experts (the bench workload): counts
    and group offsets in full, 512 sampled pairs' rows byte for byte."""
    wl = workloads.moe_dispatch()
    x, ids = wl["x"][0], wl["topk_ids"][0]
    tokens, k = ids.shape
    src = Source(fpq, x, ids, 64)
    buf = _buffers(tokens * k, x.shape[1])
    offs = src.dispatch(src.counts.view(1, 64), 1, 0, fpq.MOE_DIRECT, [buf])
    counts, slot = orc.moe_route_plan(ids.numpy(), 64)
    assert np.array_equal(src.counts.cpu().numpy(), counts)
    woff = np.concatenate([[0], np.cumsum(counts)])
    assert np.array_equal(offs.cpu().numpy(), woff)
    rng = np.random.default_rng(40)
    ts, js = rng.integers(0, tokens, 512), rng.integers(0, k, 512)
    xu = workloads.as_u16(x)
    idn = ids.numpy()
    q_all, s_all = buf[0].cpu().numpy(), buf[1].cpu().numpy()
    for t, j in zip(ts, js):
        row = woff[idn[t, j]] + slot[t, j]
        q, s = orc.quant_mxfp8(xu[t][None])
        assert np.array_equal(q_all[row], q[0]) and np.array_equal(s_all[row], s[0])
    assert fpq.fpq_get_device_error() == 0


def test_convenience_dispatch_single_rank(fpq, orc):
    from mxfp8_block_scaled_warp_b200 import moe
    x, ids = _x(64, 256, 870), _ids(64, 8, 2, 871)
    d = moe.dispatch(x.cuda(), ids.cuda(), 8)
    wq, ws, woff = orc.moe_dispatch([workloads.as_u16(x)], [ids.numpy()], 8)[0]
    assert np.array_equal(d.codes.cpu().numpy(), wq) and np.array_equal(d.scales.cpu().numpy(), ws)
    assert np.array_equal(d.group_offsets.cpu().numpy(), woff)


def test_empty_tokens(fpq):
    ids = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    counts = torch.full((8,), 7, dtype=torch.int32, device="cuda")
    wsb = fpq.fpq_moe_route_workspace_bytes(0, 8)
    ws = torch.empty(((wsb + 15) // 16 * 16,), dtype=torch.uint8, device="cuda")
    fpq.fpq_moe_route(ids, 0, 4, 8, counts, ws)
    assert counts.cpu().tolist() == [0] * 8


def test_bad_expert_id_reported(fpq, orc):
    """An id outside [0, E) raises FPQ_ERR_DEVICE_BAD_INPUT; its pair is
    dropped (never written) and every other pair lands where the oracle puts
    it for the routing without that pair."""
    x, ids = _x(20, 64, 880), _ids(20, 8, 2, 881)
    bad = ids.clone()
    bad[5, 1] = 8
    src = Source(fpq, x, bad, 8)
    assert fpq.fpq_get_device_error() == BAD_INPUT
    buf = _buffers(40, 64)
    src.dispatch(src.counts.view(1, 8), 1, 0, fpq.MOE_DIRECT, [buf])
    assert fpq.fpq_get_device_error() == 0           # the dispatch itself saw only valid ids
    # the same routing without pair (5, 1), as one pair per row in pair order
    pair_ids = np.delete(ids.numpy().reshape(-1), 11).reshape(-1, 1)
    pair_x = np.delete(np.repeat(workloads.as_u16(x), 2, axis=0), 11, axis=0)
    counts, _ = orc.moe_route_plan(pair_ids, 8)
    assert np.array_equal(src.counts.cpu().numpy(), counts)
    wq, ws, _ = orc.moe_dispatch([pair_x], [pair_ids], 8)[0]
    assert np.array_equal(buf[0][:39].cpu().numpy(), wq) and np.array_equal(buf[1][:39].cpu().numpy(), ws)
    assert (buf[0][39:] == 0xEE).all()                # the dropped pair's row is never written


def test_capacity_overflow_reported(fpq):
    """A destination buffer with fewer rows than the layout needs: rows past
    its end are not written and FPQ_ERR_DEVICE_BAD_INPUT is raised."""
    x, ids = _x(30, 64, 890), _ids(30, 4, 2, 891)
    src = Source(fpq, x, ids, 4)
    big = _buffers(60, 64)
    small = (big[0][:50], big[1][:50])
    src.dispatch(src.counts.view(1, 4), 1, 0, fpq.MOE_DIRECT, [small])
    assert fpq.fpq_get_device_error() == BAD_INPUT
    assert (big[0][50:] == 0xEE).all() and (big[1][50:] == 0xEE).all()


def test_rejects_bad_args(fpq):
    t = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    c = torch.zeros((8,), dtype=torch.int32, device="cuda")
    ws = torch.empty((4096,), dtype=torch.uint8, device="cuda")
    with pytest.raises(fpq.FpqError):           # topk out of range
        fpq.fpq_moe_route(t, 4, 33, 8, c, ws)
    with pytest.raises(fpq.FpqError):           # world does not divide the experts
        fpq.fpq_moe_dispatch_layout(c.view(1, 8), 3, 8, 0, fpq.MOE_DIRECT, torch.empty(8, dtype=torch.int64,
                                    device="cuda"), c)
    with pytest.raises(fpq.FpqError):           # hidden not a multiple of 32
        x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
        p = torch.zeros(1, dtype=torch.int64, device="cuda")
        fpq.fpq_moe_dispatch_mxfp8(x, 4, 48, t, 2, 8, ws, torch.zeros(8, dtype=torch.int64, device="cuda"), 1, p, p,
                                   p)


@pytest.mark.parametrize("world,experts,k,hidden", [(2, 8, 2, 256), (3, 12, 3, 96), (8, 64, 8, 7168),
                                                    (4, 16, 4, 2048)])
def test_pack_exchange_regroup(fpq, orc, world, experts, k, hidden):
    """The several-rank path end to end on one GPU: every source's PACK send
    buffer (the kernels), the all-to-all stood in for by moving each
    source's run of rows for rank r into r's receive buffer in source order,
    then fpq_moe_regroup: each rank's grouped buffer equals the oracle's
    dispatch over all ranks byte for byte.  Some sources hold no tokens."""
    L = experts // world
    tokens = [0 if s == 1 else 20 + 13 * s for s in range(world)]
    xs = [_x(t, hidden, 900 + s) for s, t in enumerate(tokens)]
    ids = [_ids(t, experts, k, 910 + s) for s, t in enumerate(tokens)]
    srcs = [Source(fpq, xs[s], ids[s], experts) for s in range(world)]
    counts_all = torch.stack([s.counts for s in srcs]).contiguous()
    c = counts_all.cpu().numpy().astype(np.int64)
    packs = []
    for s in range(world):
        buf = _buffers(max(1, tokens[s] * k), hidden)
        srcs[s].dispatch(counts_all, world, s, fpq.MOE_PACK, [buf])
        packs.append(buf)
    want = orc.moe_dispatch([workloads.as_u16(x) for x in xs], [i.numpy() for i in ids], experts)
    for r in range(world):
        runs_q, runs_s = [], []
        for s in range(world):
            a = int(c[s][:r * L].sum())
            n = int(c[s][r * L:(r + 1) * L].sum())
            runs_q.append(packs[s][0][a:a + n])
            runs_s.append(packs[s][1][a:a + n])
        recv_q, recv_s = torch.cat(runs_q).contiguous(), torch.cat(runs_s).contiguous()
        rows = recv_q.shape[0]
        assert rows == want[r][2][-1]
        out = _buffers(max(1, rows), hidden)
        fpq.fpq_moe_regroup(recv_q, recv_s, counts_all, world, experts, r, hidden, rows, out[0], out[1])
        assert np.array_equal(out[0][:rows].cpu().numpy(), want[r][0])
        assert np.array_equal(out[1][:rows].cpu().numpy(), want[r][1])
    assert fpq.fpq_get_device_error() == 0


def test_regroup_malformed_counts_reported(fpq):
    """Counts that place a segment past the buffer: FPQ_ERR_DEVICE_BAD_INPUT,
    and the segment is not copied."""
    counts = torch.tensor([[3, 2], [4, 50]], dtype=torch.int32, device="cuda")      # world 2, E 2, rank 1: 52 rows
    recv_q, recv_s = _buffers(10, 64)
    out_q, out_s = _buffers(10, 64)
    fpq.fpq_moe_regroup(recv_q, recv_s, counts, 2, 2, 1, 64, 10, out_q, out_s)
    assert fpq.fpq_get_device_error() == BAD_INPUT
    assert (out_q[2:] == 0xEE).all()                 # rows of the oversize segment untouched
