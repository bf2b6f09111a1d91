"""GPU parity of the bf16 tensor-core GEMM and the QAT backward
(straight-through estimator; "DeepSeek R1 and V3 get quantization-aware
fine-tuning on Fireworks", Synopsis and Interpretation) against the oracle's
fp64 sums: |gpu - ref| <= 8e-3 |ref| + 1e-2 rms(ref) per element, the same
acceptance as the other GEMMs; bit-exact where every product and partial sum
is exact in fp32 and the result is a bf16 value."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda() if a.dtype == np.uint16 else \
        torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rand(shape, seed, std=1.0):
    return workloads.as_u16(workloads.normal_bf16(shape, std, seed))


def check(got: torch.Tensor, ref: np.ndarray, orc, what: str, rms=None):
    g = got.float().cpu().numpy().astype(np.float64)
    ok, ratio = orc.gemm_tolerance_ok(g, ref, rms)
    assert ok, f"{what}: worst |err|/bound = {ratio:.3f}"


@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (200, 272, 136), (1, 8, 8), (300, 512, 1000), (16, 7168, 2048),
                                   (2048, 16, 7168)])
def test_gemm_bf16_random(fpq, orc, m, n, k):
    p, q = rand((m, k), 900 + m), rand((n, k), 901 + n, std=0.05)
    for alpha in (1.0, 2.0):
        ref = orc.gemm_bf16_full(p, q, alpha)
        c = fpq.gemm_bf16(dev(p), dev(q), alpha)
        check(c, ref, orc, f"bf16 gemm {m}x{n}x{k} alpha={alpha}")
    assert fpq.fpq_get_device_error() == 0


@pytest.mark.parametrize("p_mn,q_mn", [(False, True), (True, False), (True, True)])
@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (200, 272, 136), (16, 7168, 2048), (520, 16, 1000)])
def test_gemm_bf16_mn_major(fpq, orc, p_mn, q_mn, m, n, k):
    """Operands stored with the product's row index contiguous ([k, m] and
    [k, n]) are read through MN-major descriptors, not transposed."""
    p, q = rand((m, k), 920 + m), rand((n, k), 921 + n, std=0.05)
    ref = orc.gemm_bf16_full(p, q, 0.5)
    ps = np.ascontiguousarray(p.T) if p_mn else p
    qs = np.ascontiguousarray(q.T) if q_mn else q
    c = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    fpq.fpq_gemm_bf16_layout(dev(ps), p_mn, dev(qs), q_mn, m, n, k, 0.5, c)
    check(c, ref, orc, f"bf16 gemm mn {p_mn}{q_mn} {m}x{n}x{k}")
    assert fpq.fpq_get_device_error() == 0


def test_transpose_bf16_exact(fpq):
    x = rand((200, 136), 930)
    out = torch.empty((136, 200), dtype=torch.bfloat16, device="cuda")
    fpq.fpq_transpose_bf16(dev(x), out, 200, 136)
    assert np.array_equal(workloads.as_u16(out), np.ascontiguousarray(x.T))


def test_gemm_bf16_integer_exact(fpq, orc):
    """Entries in {-1, 0, 1}: every product and partial sum is exact in fp32,
    and alpha = 0.25 times a sum of at most 64 terms is a multiple of 0.25
    below 16, which bf16 holds exactly: C must match bit for bit."""
    rng = np.random.default_rng(30)
    m, n, k = 256, 512, 64
    ip, iq = rng.integers(-1, 2, (m, k)), rng.integers(-1, 2, (n, k))
    p = workloads.as_u16(torch.from_numpy(ip.astype(np.float32)).to(torch.bfloat16))
    q = workloads.as_u16(torch.from_numpy(iq.astype(np.float32)).to(torch.bfloat16))
    c = fpq.gemm_bf16(dev(p), dev(q), 0.25)
    ref = 0.25 * (ip @ iq.T).astype(np.float64)
    assert np.array_equal(c.float().cpu().numpy().astype(np.float64), ref)


def _qat_inputs(m, n, k, r, seed):
    dy = rand((m, n), seed, std=1.0)
    x_fq = rand((m, k), seed + 1, std=1.0)
    w_fq = rand((n, k), seed + 2, std=0.02)
    a = rand((r, k), seed + 3, std=0.01)
    b = rand((n, r), seed + 4, std=0.01)
    return dy, x_fq, w_fq, a, b


@pytest.mark.parametrize("m,n,k,r", [(256, 272, 384, 16), (136, 64, 520, 8)])
def test_qat_backward_small(fpq, orc, m, n, k, r):
    dy, x_fq, w_fq, a, b = _qat_inputs(m, n, k, r, 950 + m)
    dx, dw, da, db = fpq.qat_backward(dev(dy), dev(x_fq), dev(w_fq), dev(a), dev(b), 2.0)
    rdx, rdw, rda, rdb = orc.qat_backward(dy, x_fq, w_fq, a, b, 2.0)
    check(dx, rdx, orc, "dx")
    check(dw, rdw, orc, "dw")
    check(da, rda, orc, "da")
    check(db, rdb, orc, "db")
    assert fpq.fpq_get_device_error() == 0


def test_qat_backward_full_size_sampled(fpq, orc):
    """The QAT layer of the fine-grained workload's shape (x 8192 x 7168,
    W 2048 x 7168, r = 16): sampled entries of dx and dw, and whole columns
    of da and rows of db (those need whole columns / rows of the oracle's
    bf16 dw)."""
    m, n, k, r = 8192, 2048, 7168, 16
    dy, x_fq, w_fq, a, b = _qat_inputs(m, n, k, r, 970)
    dx, dw, da, db = fpq.qat_backward(dev(dy), dev(x_fq), dev(w_fq), dev(a), dev(b), 2.0)
    assert fpq.fpq_get_device_error() == 0
    rng = np.random.default_rng(31)
    rows, cols = rng.integers(0, m, 256), rng.integers(0, k, 256)
    ref = orc.gemm_bf16_entries(dy, np.ascontiguousarray(w_fq.T), rows, cols)
    check(dx[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()], ref, orc, "dx sampled",
          rms=float(np.sqrt(np.mean(ref ** 2))))
    dyt, xt = np.ascontiguousarray(dy.T), np.ascontiguousarray(x_fq.T)
    rows, cols = rng.integers(0, n, 256), rng.integers(0, k, 256)
    ref = orc.gemm_bf16_entries(dyt, xt, rows, cols)
    check(dw[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()], ref, orc, "dw sampled",
          rms=float(np.sqrt(np.mean(ref ** 2))))
    # da[:, kc] needs dw16[:, kc]; db[nr, :] needs dw16[nr, :]
    kc = rng.integers(0, k, 3)
    nn, kk = np.meshgrid(np.arange(n), kc, indexing="ij")
    dw_cols = orc.bf16_round(orc.gemm_bf16_entries(dyt, xt, nn.ravel(), kk.ravel()).reshape(n, len(kc)))
    ref = orc.gemm_bf16_full(np.ascontiguousarray(b.T), np.ascontiguousarray(dw_cols.T), 2.0)     # [r, 3]
    check(da[:, torch.from_numpy(kc).cuda()], ref, orc, "da columns")
    nr = rng.integers(0, n, 2)
    rr, kk = np.meshgrid(nr, np.arange(k), indexing="ij")
    dw_rows = orc.bf16_round(orc.gemm_bf16_entries(dyt, xt, rr.ravel(), kk.ravel()).reshape(len(nr), k))
    ref = orc.gemm_bf16_full(dw_rows, a, 2.0)                                                       # [2, r]
    check(db[torch.from_numpy(nr).cuda()], ref, orc, "db rows")


def test_qat_backward_rejects_bad_args(fpq):
    t = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpq.FpqError):       # r not a multiple of 8
        fpq.fpq_qat_backward(t, t, t, t, t, 64, 64, 64, 12, 1.0, t, t, t, t, None)
    with pytest.raises(fpq.FpqError):       # m not a multiple of 8
        fpq.fpq_qat_backward(t, t, t, t, t, 60, 64, 64, 8, 1.0, t, t, t, t, None)
    big = torch.zeros(4096 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpq.FpqError):       # misaligned operand
        fpq.fpq_qat_backward(big[1:4097].view(64, 64), t, t, t, t, 64, 64, 64, 8, 1.0, t, t, t, t, None)


def _splitk(fpq, ps, p_mn, qs, q_mn, m, n, k, alpha):
    c = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((fpq.fpq_gemm_bf16_splitk_workspace_bytes(m, n, k),), dtype=torch.uint8, device="cuda")
    fpq.fpq_gemm_bf16_splitk(ps, p_mn, qs, q_mn, m, n, k, alpha, c, ws)
    return c


@pytest.mark.parametrize("p_mn,q_mn", [(False, False), (True, True), (False, True)])
@pytest.mark.parametrize("m,n,k", [(16, 7168, 2048), (2048, 16, 7168), (8, 8, 8), (24, 520, 1000),
                                   (200, 16, 1064), (16, 136, 8200)])
def test_gemm_bf16_splitk(fpq, orc, p_mn, q_mn, m, n, k):
    """Few output tiles, long contraction: the K slices' fp32 partial sums
    are added by a second kernel; ragged K tails land in the last slice."""
    if p_mn and m % 8:
        pytest.skip("MN-major P needs m a multiple of 8")
    p, q = rand((m, k), 940 + m), rand((n, k), 941 + n, std=0.05)
    ref = orc.gemm_bf16_full(p, q, 2.0)
    ps = np.ascontiguousarray(p.T) if p_mn else p
    qs = np.ascontiguousarray(q.T) if q_mn else q
    c = _splitk(fpq, dev(ps), p_mn, dev(qs), q_mn, m, n, k, 2.0)
    check(c, ref, orc, f"bf16 split-k {p_mn}{q_mn} {m}x{n}x{k}")
    assert fpq.fpq_get_device_error() == 0


def test_gemm_bf16_splitk_integer_exact(fpq, orc):
    """Entries in {-1, 0, 1} with K = 4096 (up to 16 slices of the
    contraction): every partial sum is an integer below 2^24, so the fp32
    slice sums and their total are exact, and C must be the round-to-
    nearest-even bf16 of alpha times the exact integer sum; a slice lost or
    added twice changes it."""
    rng = np.random.default_rng(32)
    m, n, k = 16, 512, 4096
    ip, iq = rng.integers(-1, 2, (m, k)), rng.integers(-1, 2, (n, k))
    p = workloads.as_u16(torch.from_numpy(ip.astype(np.float32)).to(torch.bfloat16))
    q = workloads.as_u16(torch.from_numpy(iq.astype(np.float32)).to(torch.bfloat16))
    c = _splitk(fpq, dev(p), False, dev(q), False, m, n, k, 0.25)
    ref = orc.bf16_round(0.25 * (ip @ iq.T).astype(np.float64))       # bf16 bit patterns
    assert np.array_equal(workloads.as_u16(c), ref)


def test_gemm_bf16_splitk_repeatable(fpq):
    """The slices are added in a fixed order: two runs agree bit for bit."""
    m, n, k = 16, 7168, 2048
    p, q = dev(rand((k, m), 960)), dev(rand((k, n), 961, std=0.05))
    c1 = _splitk(fpq, p, True, q, True, m, n, k, 2.0)
    c2 = _splitk(fpq, p, True, q, True, m, n, k, 2.0)
    assert torch.equal(c1.view(torch.int16), c2.view(torch.int16))


def test_gemm_bf16_splitk_rejects_small_workspace(fpq):
    t = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((fpq.fpq_gemm_bf16_splitk_workspace_bytes(64, 64, 64) - 16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(fpq.FpqError):
        fpq.fpq_gemm_bf16_splitk(t, 0, t, 0, 64, 64, 64, 1.0, t, ws)
    with pytest.raises(fpq.FpqError):
        fpq.fpq_gemm_bf16_splitk(t, 0, t, 0, 64, 64, 64, 1.0, t, None)


def _lora_grads(fpq, dw, a, b, n, k, r, aor):
    da = torch.empty((r, k), dtype=torch.bfloat16, device="cuda")
    db = torch.empty((n, r), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((fpq.fpq_qat_lora_grads_workspace_bytes(n, k, r),), dtype=torch.uint8, device="cuda")
    fpq.fpq_qat_lora_grads(dw, a, b, n, k, r, aor, da, db, ws)
    return da, db


@pytest.mark.parametrize("n,k,r", [(8, 8, 8), (272, 136, 16), (136, 1000, 8), (2048, 7168, 16), (520, 264, 64),
                                   (7168, 2048, 32), (200, 8200, 24), (128, 128, 40)])
def test_qat_lora_grads(fpq, orc, n, k, r):
    """dA = (alpha/r) B^T dW and dB = (alpha/r) dW A^T from one pass over
    dW: ragged strips of 128 rows, ragged K tiles, every r the fused kernel
    takes (multiples of 8 up to 64)."""
    dw, a, b = rand((n, k), 980 + n, std=0.05), rand((r, k), 981 + r, std=0.01), rand((n, r), 982 + k, std=0.01)
    da, db = _lora_grads(fpq, dev(dw), dev(a), dev(b), n, k, r, 2.0)
    assert fpq.fpq_get_device_error() == 0
    check(da, orc.gemm_bf16_full(np.ascontiguousarray(b.T), np.ascontiguousarray(dw.T), 2.0), orc, "da")
    check(db, orc.gemm_bf16_full(dw, a, 2.0), orc, "db")


def test_qat_lora_grads_integer_exact(fpq, orc):
    """Entries in {-1, 0, 1}: every partial sum over dW's rows (dA, up to
    2048 terms split by 128-row strips) and over its columns (dB, 4096 terms
    split by K ranges) is an exact integer in fp32, so the outputs must be
    the round-to-nearest-even bf16 of alpha times the exact sums; a strip or
    K range lost or added twice changes them."""
    rng = np.random.default_rng(33)
    n, k, r = 2048, 4096, 16
    idw, ia, ib = rng.integers(-1, 2, (n, k)), rng.integers(-1, 2, (r, k)), rng.integers(-1, 2, (n, r))
    bf = lambda v: workloads.as_u16(torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16))
    da, db = _lora_grads(fpq, dev(bf(idw)), dev(bf(ia)), dev(bf(ib)), n, k, r, 0.25)
    assert np.array_equal(workloads.as_u16(da), orc.bf16_round(0.25 * (ib.T @ idw).astype(np.float64)))
    assert np.array_equal(workloads.as_u16(db), orc.bf16_round(0.25 * (idw @ ia.T).astype(np.float64)))


def test_qat_lora_grads_repeatable(fpq):
    n, k, r = 2048, 7168, 16
    dw, a, b = dev(rand((n, k), 990, std=0.05)), dev(rand((r, k), 991)), dev(rand((n, r), 992))
    da1, db1 = _lora_grads(fpq, dw, a, b, n, k, r, 2.0)
    da2, db2 = _lora_grads(fpq, dw, a, b, n, k, r, 2.0)
    assert torch.equal(da1.view(torch.int16), da2.view(torch.int16))
    assert torch.equal(db1.view(torch.int16), db2.view(torch.int16))


def test_qat_lora_grads_rejects_bad_args(fpq):
    t = torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((fpq.fpq_qat_lora_grads_workspace_bytes(128, 128, 64),), dtype=torch.uint8, device="cuda")
    for r in (12, 72, 0):                   # not a multiple of 8, or outside [8, 64]
        with pytest.raises(fpq.FpqError):
            fpq.fpq_qat_lora_grads(t, t, t, 128, 128, r, 1.0, t, t, ws)
    with pytest.raises(fpq.FpqError):       # k not a multiple of 8
        fpq.fpq_qat_lora_grads(t, t, t, 128, 124, 8, 1.0, t, t, ws)
    small = ws[:fpq.fpq_qat_lora_grads_workspace_bytes(128, 128, 8) - 16]
    with pytest.raises(fpq.FpqError):
        fpq.fpq_qat_lora_grads(t, t, t, 128, 128, 8, 1.0, t, t, small)


@pytest.mark.parametrize("r", [64, 72])
def test_qat_backward_rank_paths(fpq, orc, r):
    """r = 64 takes the fused dA/dB pass, r = 72 the two split-K GEMMs."""
    m, n, k = 256, 272, 520
    dy, x_fq, w_fq, a, b = _qat_inputs(m, n, k, r, 1000 + r)
    dx, dw, da, db = fpq.qat_backward(dev(dy), dev(x_fq), dev(w_fq), dev(a), dev(b), 2.0)
    rdx, rdw, rda, rdb = orc.qat_backward(dy, x_fq, w_fq, a, b, 2.0)
    for got, ref, what in ((dx, rdx, "dx"), (dw, rdw, "dw"), (da, rda, "da"), (db, rdb, "db")):
        check(got, ref, orc, what)
    assert fpq.fpq_get_device_error() == 0
