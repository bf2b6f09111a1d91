"""Pins of the oracle's MoE FP8 dispatch ("DeepSeek-V3 Blog 5: Low-Precision
Training", Reducing Communication Overhead in MoE with FP8: activations are
quantized to FP8 before they are sent to the GPUs of their experts).

The placement is checked against a hand-worked example and against an
independent construction (numpy's stable lexsort on the keys expert, source
rank, token, choice); row contents against the oracle's MXFP8 quantizer of
the source row (the quantizer has its own pins)."""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _routing(rng, tokens, k, experts):
    return np.array([rng.choice(experts, k, replace=False) for _ in range(tokens)], np.int32).reshape(tokens, k)


def test_route_plan_hand_worked():
    # token 0 -> experts 1, 0; token 1 -> 0, 2; token 2 -> 1, 2
    ids = np.array([[1, 0], [0, 2], [1, 2]])
    counts, slot = oracle.moe_route_plan(ids, 4)
    assert list(counts) == [2, 2, 2, 0]
    # expert 0: (0,1) then (1,0); expert 1: (0,0) then (2,0); expert 2: (1,1) then (2,1)
    assert slot.tolist() == [[0, 0], [1, 0], [1, 1]]


def test_dispatch_hand_worked_two_ranks():
    """Two ranks, four experts (rank 0 owns 0-1, rank 1 owns 2-3), one
    choice per token; rows of 32 elements whose quantization is checked by
    value: row t of rank s holds the constant 2^(s*4 + t), so its E8M0 scale
    identifies it."""
    xs, ids = [], []
    for s, route in enumerate(([2, 0, 2], [1, 2])):
        rows = np.stack([np.full(32, 2.0 ** (4 * s + t), np.float32) for t in range(len(route))])
        xs.append(workloads.as_u16(torch.from_numpy(rows).to(torch.bfloat16)))
        ids.append(np.array(route).reshape(-1, 1))
    out = oracle.moe_dispatch(xs, ids, 4)
    # the scale of a constant block 2^p is 2^(p - 8) (2^p / 448 rounded up to a power of two)
    tags = [[int(sc[0]) - 127 + 8 for sc in out[r][1]] for r in range(2)]
    # rank 0: expert 0 <- (s0,t1); expert 1 <- (s1,t0)
    assert tags[0] == [1, 4] and out[0][2].tolist() == [0, 1, 2]
    # rank 1: expert 2 <- (s0,t0), (s0,t2), (s1,t1); expert 3 <- none
    assert tags[1] == [0, 2, 5] and out[1][2].tolist() == [0, 3, 3]


@pytest.mark.parametrize("world,experts,k", [(1, 8, 2), (2, 8, 3), (4, 8, 1), (4, 16, 4)])
def test_dispatch_matches_lexsort(world, experts, k):
    rng = np.random.default_rng(100 + world * experts + k)
    K = 64
    xs, ids = [], []
    for s in range(world):
        t = int(rng.integers(0, 12)) if s else 9          # rank 0 non-empty, others may be empty
        xs.append(workloads.as_u16(workloads.normal_bf16((t, K), 1.0, seed=200 + s)))
        ids.append(_routing(rng, t, k, experts))
    out = oracle.moe_dispatch(xs, ids, experts)
    L = experts // world
    # all pairs, with keys (expert, source, token, choice)
    e_all, s_all, t_all, j_all = [], [], [], []
    for s in range(world):
        for t in range(ids[s].shape[0]):
            for j in range(k):
                e_all.append(ids[s][t, j]), s_all.append(s), t_all.append(t), j_all.append(j)
    e_all, s_all, t_all, j_all = map(np.array, (e_all, s_all, t_all, j_all))
    order = np.lexsort((j_all, t_all, s_all, e_all))
    total = 0
    for r in range(world):
        codes, scales, offs = out[r]
        sel = order[(e_all[order] // L) == r]
        assert codes.shape[0] == len(sel) == offs[-1]
        for i, p in enumerate(sel):
            q, sc = oracle.quant_mxfp8(xs[s_all[p]][t_all[p]][None])
            assert np.array_equal(codes[i], q[0]) and np.array_equal(scales[i], sc[0])
        for l in range(L):
            assert offs[l + 1] - offs[l] == int(np.sum(e_all == r * L + l))
        total += codes.shape[0]
    assert total == len(e_all)


def test_single_rank_is_expert_major_slot_order():
    """With one rank the buffer is every expert's pairs in slot order: row
    offs[e] + slot[t, j] holds token t."""
    rng = np.random.default_rng(7)
    x = workloads.as_u16(workloads.normal_bf16((20, 64), 1.0, seed=300))
    ids = _routing(rng, 20, 3, 6)
    codes, scales, offs = oracle.moe_dispatch([x], [ids], 6)[0]
    counts, slot = oracle.moe_route_plan(ids, 6)
    assert np.array_equal(np.diff(offs), counts)
    q, sc = oracle.quant_mxfp8(x)
    for t in range(20):
        for j in range(3):
            row = offs[ids[t, j]] + slot[t, j]
            assert np.array_equal(codes[row], q[t]) and np.array_equal(scales[row], sc[t])
