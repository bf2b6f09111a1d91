"""Pins of the oracle's QAT backward (straight-through estimator; "DeepSeek
R1 and V3 get quantization-aware fine-tuning on Fireworks", Synopsis and
Interpretation): against float64 autograd of the forward
y = fq(x) fq(W_eff)^T, W_eff = W + (alpha/r) B A, written with the
straight-through trick (the fake-quantized value with the gradient of the
unquantized one), and the bf16 product against brute force."""
import numpy as np
import torch

import oracle


def _bf16(rng, shape, scale=1.0):
    x = torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16).copy()


def _dec(u16):
    return torch.from_numpy(u16.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64)


def test_gemm_bf16_brute_force():
    rng = np.random.default_rng(20)
    p, q = _bf16(rng, (5, 7)), _bf16(rng, (3, 7))
    got = oracle.gemm_bf16_full(p, q, 0.75)
    ref = np.zeros((5, 3))
    for i in range(5):
        for j in range(3):
            for t in range(7):
                ref[i, j] += oracle.bf16_decode(p[i, t]) * oracle.bf16_decode(q[j, t])
    assert np.array_equal(got, 0.75 * ref)
    rows, cols = np.array([0, 4, 2]), np.array([2, 0, 1])
    assert np.array_equal(oracle.gemm_bf16_entries(p, q, rows, cols, 0.75), got[rows, cols])


def test_bf16_round_ties_and_neighbours():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties go to the even pattern
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, 1.0 + 2 ** -8 + 2 ** -40, -2.5, 0.0])
    got = oracle.bf16_round(vals)
    assert list(got) == [0x3F80, 0x3F80, 0x3F81, 0x3F81, 0xC020, 0x0000]
    # every value is within half an ulp of its rounding
    rng = np.random.default_rng(21)
    x = rng.standard_normal(4096) * 10.0 ** rng.integers(-3, 4, 4096)
    r = _dec(oracle.bf16_round(x)).numpy()
    ulp = 2.0 ** (np.floor(np.log2(np.abs(r))) - 7)
    assert np.all(np.abs(r - x) <= ulp / 2)


def test_qat_backward_matches_autograd():
    rng = np.random.default_rng(22)
    m, n, k, r, alpha_over_r = 24, 40, 56, 8, 2.0
    dy, x_fq, w_fq = _bf16(rng, (m, n)), _bf16(rng, (m, k)), _bf16(rng, (n, k), 0.05)
    a, b, w0 = _bf16(rng, (r, k), 0.1), _bf16(rng, (n, r), 0.1), _bf16(rng, (n, k), 0.05)
    dx, dw, da, db = oracle.qat_backward(dy, x_fq, w_fq, a, b, alpha_over_r)

    # autograd in float64 with the straight-through estimator
    X = _dec(x_fq).requires_grad_(True)
    A, B = _dec(a).requires_grad_(True), _dec(b).requires_grad_(True)
    W_eff = _dec(w0) + alpha_over_r * (B @ A)
    W_eff.retain_grad()
    Wq = W_eff + (_dec(w_fq) - W_eff).detach()              # value fq(W_eff), gradient of W_eff
    y = X @ Wq.T
    (y * _dec(dy)).sum().backward()
    assert np.allclose(dx, X.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dw, W_eff.grad.numpy(), rtol=1e-12, atol=1e-12)
    # da, db use the bf16-rounded dw: within alpha/r * sum |.| * 2^-8 of autograd
    bound_a = alpha_over_r * (np.abs(_dec(b).numpy()).T @ np.abs(dw)) * 2.0 ** -8 + 1e-12
    bound_b = alpha_over_r * (np.abs(dw) @ np.abs(_dec(a).numpy()).T) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(da - A.grad.numpy()) <= bound_a)
    assert np.all(np.abs(db - B.grad.numpy()) <= bound_b)
    # and exactly the formulas on the rounded dw
    dw16 = _dec(oracle.bf16_round(dw)).numpy()
    assert np.allclose(da, alpha_over_r * _dec(b).numpy().T @ dw16, rtol=1e-12, atol=1e-12)
    assert np.allclose(db, alpha_over_r * dw16 @ _dec(a).numpy().T, rtol=1e-12, atol=1e-12)
