"""Pin of the oracle's NVFP4 convention against an independent library
implementation: vLLM's reference NVFP4 quantizer (plain torch, CPU).

Both take the per-tensor scale from amax / (6 * 448), the E4M3 block scale
per 16 elements from the block amax / 6 in units of that tensor scale, and
round elements to E2M1 to nearest even with saturation at 6.  They differ in
arithmetic order only: the oracle's code is E2M1 of the IEEE quotient
fp32(x / S) (two roundings, as its definition states), the library
multiplies by reciprocals.  So the block scales must agree everywhere, and an
element may differ only where the quotient sits on a rounding boundary of
E2M1 up to a few ulps; there the oracle's code must be the round-to-nearest-
even of fp32(x / S), which is also the rounding of the exact rational x / S
unless fp32 rounding moved the quotient onto the boundary itself."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

nvu = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils")

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
BOUNDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
GRID = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]


def rne_e2m1(q: Fraction) -> float:
    """Round-to-nearest-even of an exact rational onto the E2M1 grid, saturating at 6."""
    a = abs(q)
    if a >= 6:
        return float(6 if q > 0 else -6)
    best = min(range(8), key=lambda i: (abs(GRID[i] - a), i % 2))   # ties: the even code (0, 2, 4, 6 -> codes 0,2,4,6)
    v = float(GRID[best])
    return v if q >= 0 else -v


def _cases():
    rng = np.random.default_rng(3)
    wide = (rng.integers(0, 0x4780, (64, 256)) | (rng.integers(0, 2, (64, 256)) << 15)).astype(np.uint16)
    return {"normal": workloads.normal_bf16((64, 256), 1.0, seed=1),
            "outliers": workloads.normal_bf16((64, 256), 0.02, seed=2, outlier_frac=0.01),
            "wide": workloads.from_u16(wide),
            "larger": workloads.normal_bf16((256, 1024), 1.0, seed=5)}


@pytest.mark.parametrize("name", ["normal", "outliers", "wide", "larger"])
def test_nvfp4_against_library_reference(name):
    x = _cases()[name]
    q, s, g = oracle.quant_nvfp4(workloads.as_u16(x))
    codes = np.stack([q & 0xF, q >> 4], -1).reshape(q.shape[0], -1)
    ours = E2M1[codes]
    s_ours = torch.from_numpy(np.ascontiguousarray(s)).view(torch.float8_e4m3fn).float().numpy()
    amax = np.float32(x.float().abs().max().item())
    global_scale = torch.tensor([np.float32(2688.0) / amax], dtype=torch.float32)
    lib_q, lib_s = nvu.ref_nvfp4_quant(x.float(), global_scale, 16)
    lib_q, lib_s = lib_q.numpy(), lib_s.numpy()

    # block scales: identical everywhere
    assert np.array_equal(s_ours, lib_s)
    # elements: identical except on E2M1 rounding boundaries
    bad = np.argwhere(ours != lib_q)
    assert len(bad) <= 0.005 * ours.size, f"{len(bad)} of {ours.size} elements differ"
    g32 = np.float32(np.asarray(g).reshape(-1)[0])
    for r, c in bad[:300]:
        xv = np.float32(x[r, c].float().item())
        S = np.float32(np.float32(s_ours[r, c // 16]) * g32)
        quot = np.float32(xv / S)
        near = np.min(np.abs(np.abs(quot) - BOUNDS) / np.spacing(BOUNDS.astype(np.float32)))
        assert near <= 4, f"({r}, {c}): quotient {quot!r} is not on a rounding boundary"
        assert abs(ours[r, c] - lib_q[r, c]) <= 1.0 + 1e-9, "the two codes must be neighbours"
        assert ours[r, c] == rne_e2m1(Fraction(float(quot))), \
            f"({r}, {c}): the oracle's code is not the rounding of fp32(x / S)"
        exact = Fraction(float(xv)) / Fraction(float(S))
        if Fraction(float(abs(quot))) != Fraction(float(BOUNDS[np.argmin(np.abs(np.abs(quot) - BOUNDS))])):
            assert ours[r, c] == rne_e2m1(exact), f"({r}, {c}): off a boundary the two roundings agree"
