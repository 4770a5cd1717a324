"""Oracle pins for the W4A4 path: NVFP4 activation rows (one FP32 scale per row) and the
product with NVFP4 weights. CPU only."""

import json
import os

import numpy as np
import pytest

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(values) -> np.ndarray:
    v = np.asarray(values, dtype=np.float32)
    bits = v.view(np.uint32)
    assert ((bits & 0xFFFF) == 0).all(), "fixture values must be exact bf16"
    return (bits >> 16).astype(np.uint16)


def test_hand_worked_rows():
    with open(os.path.join(GOLDEN, "w4a4_rows.json")) as f:
        g = json.load(f)
    codes, sf, gs = G.quantize_x_rows(_bf16_bits(g["rows"]))
    assert gs.tolist() == g["g"]
    assert sf.tolist() == g["sf"]
    assert codes.tolist() == g["codes"]


def _near_midpoint(v: np.ndarray, grid: np.ndarray, ulps: float = 4.0) -> np.ndarray:
    """True where |v| lies within ``ulps`` fp32 ulps of a midpoint between two grid values."""
    mids = (grid[1:] + grid[:-1]) / 2.0
    a = np.abs(v)
    d = np.min(np.abs(a[..., None] - mids), axis=-1)
    return d <= ulps * np.spacing(np.float32(1.0)) * np.maximum(a, 1e-30)


def test_agrees_with_the_float64_weight_quantiser_except_at_boundaries():
    """Per row, the fp32 decisions agree with the weight quantiser's float64 ones except where
    the float64 value sits within a few fp32 ulps of a rounding midpoint (bf16 inputs hit
    exact midpoints often), or in a block whose scale already differs."""
    _, x = S.random_case(5, 64, 16, 4096)
    codes, sf, g = G.quantize_x_rows(x)
    xf = G.bf16_bits_to_float64(x).astype(np.float32)
    e4m3_pos = np.unique(np.abs(F.E4M3_VALUES[np.isfinite(F.E4M3_VALUES)]))
    e2m1_pos = np.unique(np.abs(F.E2M1_VALUES))
    n_diff = 0
    for m in range(x.shape[0]):
        c64, s64, ts = F.quantize_codes(xf[m:m + 1], tensor_scale_in=g[m])
        assert np.float32(ts) == g[m]
        blocks = xf[m].astype(np.float64).reshape(-1, 16)
        a64 = np.abs(blocks).max(axis=1) / (6.0 * float(g[m]))
        bad_s = s64[0] != sf[m]
        assert _near_midpoint(a64[bad_s], e4m3_pos).all()
        r64 = blocks / (F.E4M3_VALUES[s64[0]][:, None] * float(g[m]))
        bad_c = (c64[0] != codes[m]).reshape(-1, 16) & ~bad_s[:, None]
        assert _near_midpoint(r64[bad_c], e2m1_pos).all()
        n_diff += int(bad_c.sum())
    assert n_diff <= 0.001 * codes.size


def test_dequantised_rows_within_half_a_step():
    _, x = S.random_case(6, 8, 16, 2048)
    codes, sf, g = G.quantize_x_rows(x)
    xh = G.dequantize_x_rows(codes, sf, g)
    xf = G.bf16_bits_to_float64(x)
    S_ = F.E4M3_VALUES[sf]
    step = np.repeat(S_, 16, axis=1) * g[:, None].astype(np.float64) * 2.0   # largest E2M1 gap (4 -> 6)
    assert (np.abs(xh - xf) <= 0.5 * step * 1.0001).all()


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (2, 3, 32), (3, 2, 48)])
def test_w4a4_gemm_brute_force(M, N, K):
    W, x = S.random_case(7 + M + N, M, N, K)
    q, sf, ts = F.quantize_nvfp4(W)
    y = G.gemm_w4a4_ref(x, q, sf, ts)
    xc, xs, g = G.quantize_x_rows(x)
    wc = F.unpack_codes(q)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                xv = F.E2M1_VALUES[xc[m, k]] * F.E4M3_VALUES[xs[m, k // 16]] * float(g[m])
                wv = F.E2M1_VALUES[wc[n, k]] * F.E4M3_VALUES[sf[n, k // 16]] * float(ts)
                acc += xv * wv
            assert y[m, n] == pytest.approx(acc, rel=1e-12, abs=1e-300)


def test_per_tensor_activation_scale_is_caught():
    """A planted per-tensor (not per-row) activation scale changes the hand-worked row 1's scales."""
    with open(os.path.join(GOLDEN, "w4a4_rows.json")) as f:
        g = json.load(f)
    rows = np.asarray(g["rows"], dtype=np.float32)
    c64, s64, _ = F.quantize_codes(rows[1:2], tensor_scale_in=np.float32(np.abs(rows).max() / 2688))
    assert s64[0].tolist() != g["sf"][1]
