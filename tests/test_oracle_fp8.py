"""Oracle pins for FP8 (E4M3) block-scaled weights and their GEMM. CPU only."""

import json
import os

import numpy as np
import pytest

import synthetic as S
from oracle import fp8 as P
from oracle import gemm as G
from oracle import nvfp4 as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    with open(os.path.join(GOLDEN, "fp8_blocks.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_hand_worked_blocks(case):
    W = np.array(case["W"], dtype=np.float32)
    codes, scales = P.quantize_fp8_blocks(W, tuple(case["block"]))
    assert scales.tolist() == case["scales"]
    assert codes.tolist() == case["codes"]
    assert P.dequantize_fp8_blocks(codes, scales, tuple(case["block"])).tolist() == case["dequant"]


def test_round_trip_of_representable_blocks():
    """Blocks built from E4M3 values times a power-of-two scale, with 448 present, come back
    with the same codes and scale."""
    rng = np.random.default_rng(81)
    finite = np.array([c for c in range(256) if np.isfinite(F.E4M3_VALUES[c])], dtype=np.uint8)
    for e in (-12, -3, 0, 5):
        c = rng.choice(finite, size=(16, 32)).astype(np.uint8)
        c[3, 7] = 126                                       # 448: fixes the block's amax
        W = (F.E4M3_VALUES[c] * 2.0 ** e).astype(np.float32)
        codes, scales = P.quantize_fp8_blocks(W, (16, 32))
        assert scales[0, 0] == np.float32(2.0 ** e)
        zero = F.E4M3_VALUES[c] == 0                       # +0 and -0 dequantise the same
        assert np.array_equal(codes[~zero], c[~zero])


def test_error_within_half_a_step():
    W = (np.random.default_rng(82).standard_normal((200, 300)) * 0.05).astype(np.float32)
    codes, scales = P.quantize_fp8_blocks(W, (64, 128))
    s = np.repeat(np.repeat(scales.astype(np.float64), 64, 0), 128, 1)[:200, :300]
    r = W.astype(np.float64) / s
    rq = F.E4M3_VALUES[codes]
    assert (np.abs(r - rq) <= np.maximum(np.abs(r) * 2.0 ** -4, 2.0 ** -10)).all()
    assert scales.shape == (4, 3)                          # partial edge blocks included


@pytest.mark.parametrize("M,N,K", [(1, 3, 16), (2, 5, 40)])
def test_fp8_gemm_brute_force(M, N, K):
    W, x = S.random_case(83 + M, M, N, K)
    codes, scales = P.quantize_fp8_blocks(W, (2, 8))
    y = P.gemm_fp8_ref(x, codes, scales, (2, 8))
    xf = G.bf16_bits_to_float64(x)
    for m in range(M):
        for n in range(N):
            acc = sum(xf[m, k] * F.E4M3_VALUES[codes[n, k]] * float(scales[n // 2, k // 8]) for k in range(K))
            assert y[m, n] == pytest.approx(acc, rel=1e-12, abs=1e-300)


def test_per_tensor_scale_is_caught():
    """A planted per-tensor scale changes the hand-worked second case's codes."""
    case = _cases()[1]
    W = np.array(case["W"], dtype=np.float32)
    codes, _ = P.quantize_fp8_blocks(W, W.shape)           # one block = the whole tensor
    assert codes.tolist() != case["codes"]
