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
def test_split_sizes_match_oracle_layout(world, experts):
    """The all-to-all's row counts: what rank r sends to rank p is the run of
    p's experts in r's expert-major pack, and what r receives from all
    sources adds up to the oracle's grouped buffer."""
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
    sends = {}
    for r in range(world):
        send, recv = moe.split_sizes(torch.from_numpy(counts_all), r, world, experts)
        sends[r] = send
        assert sum(recv) == want[r][2][-1]
        assert sum(send) == counts_all[r].sum()
        for p in range(world):
            assert send[p] == counts_all[r][p * L:(p + 1) * L].sum()
    for r in range(world):                                        # the two sides of every transfer agree
        _, recv = moe.split_sizes(torch.from_numpy(counts_all), r, world, experts)
        assert recv == [sends[s][r] for s in range(world)]


def test_split_sizes_accept_nested_lists():
    send, recv = moe.split_sizes([[1, 0, 2, 3], [0, 4, 0, 1]], 1, 2, 4)
    assert send == [4, 1] and recv == [5, 1]
