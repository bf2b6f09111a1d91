"""Host logic of the MoE FP8 dispatch without a GPU: argument checks that
fire before any device work, and the segment arithmetic of the exchange
against the oracle's group offsets (every receive segment starts where the
oracle's grouped buffer puts that source's rows of that expert)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from mxfp8_block_scaled_warp_b200 import moe


def test_dispatch_rejects_bad_inputs_before_device_work():
    x = torch.zeros((4, 64), dtype=torch.float32)
    ids = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError):
        moe.dispatch(x, ids, 8)                                   # x not bf16
    with pytest.raises(ValueError):
        moe.dispatch(x.to(torch.bfloat16), ids.to(torch.int64), 8)  # ids not int32
    with pytest.raises(ValueError):
        moe.dispatch(x.to(torch.bfloat16), ids[:, 0], 8)         # ids not 2-D


@pytest.mark.parametrize("world,experts", [(1, 5), (2, 8), (4, 8), (4, 16)])
def test_segment_plan_matches_oracle_layout(world, experts):
    rng = np.random.default_rng(world * 100 + experts)
    k, hidden = 2, 32
    xs, ids = [], []
    for s in range(world):
        t = int(rng.integers(0, 9))                               # some sources may hold no tokens
        xs.append(workloads.as_u16(workloads.normal_bf16((t, hidden), 1.0, seed=1200 + s)))
        ids.append(np.array([rng.choice(experts, k, replace=False) for _ in range(t)],
                            np.int64).reshape(t, k))
    counts_all = np.stack([oracle.moe_route_plan(i, experts)[0] for i in ids])
    want = oracle.moe_dispatch(xs, ids, experts)
    L = experts // world
    for r in range(world):
        sends, recvs, rows = moe.segment_plan(torch.from_numpy(counts_all), r, world, experts)
        assert rows == want[r][2][-1]
        # receive segments tile [0, rows) in (local expert, source) order
        pos = 0
        for src, e, r0, n in recvs:
            assert r0 == pos and n == counts_all[src][e] and e // L == r
            pos += n
        assert pos == rows
        # the first segment of each local expert starts at its group offset
        for l in range(L):
            segs = [seg for seg in recvs if seg[1] == r * L + l]
            if segs:
                assert segs[0][2] == want[r][2][l]
        # send segments tile this rank's expert-major pack
        pos = 0
        for peer, e, r0, n in sends:
            assert r0 == sum(counts_all[r][:e]) and n == counts_all[r][e] and peer == e // L
        assert sum(n for *_, n in sends) == counts_all[r].sum()


def test_segment_plan_accepts_nested_lists():
    sends, recvs, rows = moe.segment_plan([[1, 0, 2, 3], [0, 4, 0, 1]], 1, 2, 4)
    assert rows == 2 + 0 + 3 + 1                                  # experts 2 and 3, both sources
    assert sends == [(0, 1, 0, 4), (1, 3, 4, 1)]
    assert recvs == [(0, 2, 0, 2), (0, 3, 2, 3), (1, 3, 5, 1)]
