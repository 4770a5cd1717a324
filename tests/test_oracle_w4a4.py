"""Oracle pins for the W4A4 path: NVFP4 activation rows (one FP32 scale per row) and the
product with NVFP4 weights. CPU only."""

import json
import os
from fractions import Fraction

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


def _nearest_even(q, values, codes):
    """The value of ``values`` nearest to the exact rational q >= 0, ties to the even code,
    saturating at the largest (a brute-force search over the whole value set)."""
    best = None
    for v, c in zip(values, codes):
        d = abs(Fraction(v) - q)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, v, c)
    return best[2]


def test_rows_against_exact_fractions():
    """Brute force in exact rational arithmetic: g is the fp32 rounding of amax/2688; S is
    the E4M3 value nearest to amax_block/(6 g) and each code the E2M1 value nearest to
    x/(S g), found by search over the whole value sets with ties to the even code. Random
    rows, plus rows built around E4M3 and E2M1 midpoints."""
    e4 = [(float(F.E4M3_VALUES[c]), c) for c in range(0x7F)]
    e2 = [(float(F.E2M1_VALUES[c]), c) for c in range(8)]
    _, x = S.random_case(5, 6, 16, 64)
    xf = G.bf16_bits_to_float64(x)
    xf[1, 16:32] *= 1e-4                                    # one block far below the row amax
    xf[2, :] = np.round(xf[2, :] * 8) / 8                   # many exact halves and quarters: ties
    x = S.f32_to_bf16_bits(xf.astype(np.float32))
    xf = G.bf16_bits_to_float64(x)
    codes, sf, g = G.quantize_x_rows(x)
    for m in range(x.shape[0]):
        amax = float(np.max(np.abs(xf[m])))
        g_ref = np.float32(np.float32(amax) / np.float32(2688.0))   # fp32 quotient, correctly rounded
        assert g[m] == g_ref
        gq = Fraction(float(g_ref))
        for b in range(x.shape[1] // 16):
            blk = xf[m, 16 * b: 16 * b + 16]
            s_code = _nearest_even(Fraction(float(np.max(np.abs(blk)))) / (6 * gq), *zip(*e4)) if gq else 0
            assert sf[m, b] == s_code, (m, b)
            den = Fraction(float(F.E4M3_VALUES[s_code])) * gq
            for k in range(16):
                want = 0 if den == 0 else _nearest_even(abs(Fraction(float(blk[k]))) / den, *zip(*e2)) | \
                    (8 if np.signbit(blk[k]) else 0)
                assert codes[m, 16 * b + k] == want, (m, b, k)


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
