"""Pins of the oracle's NVFP4 format code against things outside the oracle.

- Values the E2M1 / E4M3 definitions fix, written out literally.
- torch's CPU float8_e4m3fn decode and cast, an independent library implementation.
- Brute-force nearest search on the value grids.
- Hand-worked 2x16 blocks (tests/golden/hand_blocks.json).
- Exhaustive round trip of every E2M1 x E4M3 value.
- Closed forms of the tensor scale.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4 as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- value sets

def test_e2m1_value_set_literal():
    pos = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(F.E2M1_VALUES[:8]) == pos
    assert list(F.E2M1_VALUES[8:]) == [-v for v in pos]
    assert math.copysign(1.0, F.E2M1_VALUES[8]) == -1.0   # code 0x8 is -0


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.E4M3_VALUES
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2                                  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], ours[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(ours[~nan]))


def test_e4m3_literal_points():
    assert F.e4m3_decode(0x7E) == 448.0
    assert F.e4m3_decode(0x38) == 1.0
    assert F.e4m3_decode(0x01) == 2.0 ** -9
    assert F.e4m3_decode(0x08) == 2.0 ** -6
    assert F.e4m3_decode(0x07) == 7 * 2.0 ** -9


# ---------------------------------------------------------------- rounding

def _brute_e2m1(r):
    """Nearest grid value; on a tie the even code (even mantissa bit); saturating at 6."""
    a = min(abs(r), 6.0)
    grid = F.E2M1_VALUES[:8]
    d = np.abs(grid - a)
    best = np.flatnonzero(d == d.min())
    code = int(best[0]) if len(best) == 1 else int([c for c in best if c % 2 == 0][0])
    return code | (8 if math.copysign(1.0, r) < 0 else 0)


def test_e2m1_rounding_brute_force_grid_and_midpoints():
    vals = np.arange(-7.0, 7.0001, 0.125)
    vals = np.concatenate([vals, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 6.5, 1e9, -0.0]])
    got = F.e2m1_encode(vals)
    want = np.array([_brute_e2m1(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_rounding_brute_force_random():
    rng = np.random.default_rng(11)
    vals = rng.uniform(-8, 8, 20000)
    got = F.e2m1_encode(vals)
    want = np.array([_brute_e2m1(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_ties_listed():
    # ties to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2, 2.5->2, 3.5->4, 5->4
    got = F.E2M1_VALUES[F.e2m1_encode(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]))]
    assert list(got) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def test_e4m3_rounding_matches_torch_cast():
    """torch's float32 -> float8_e4m3fn cast rounds to nearest even (it saturates only up to 464)."""
    rng = np.random.default_rng(12)
    pos = F.E4M3_VALUES[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2.0                 # every midpoint, exact in fp32
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(460.0), 50000))
    vals = np.concatenate([pos, mids, rand, [448.0, 455.0, 463.9]]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode(vals.astype(np.float64))
    assert np.array_equal(got, ref)


def test_e4m3_saturates():
    assert F.e4m3_encode(np.array([1e6, 480.0, 449.0]))[0] == 0x7E
    assert list(F.e4m3_encode(np.array([1e6, 480.0, 449.0]))) == [0x7E, 0x7E, 0x7E]


# ---------------------------------------------------------------- hand-worked blocks

@pytest.mark.parametrize("case_idx", [0, 1])
def test_hand_worked_blocks(case_idx):
    with open(os.path.join(GOLDEN, "hand_blocks.json")) as f:
        g = json.load(f)
    W = np.array(g["W"], dtype=np.float32)
    case = g["cases"][case_idx]
    codes, sf, ts = F.quantize_codes(W, case["tensor_scale_in"])
    assert float(ts) == case["ts"]
    assert sf.tolist() == case["sf"]
    assert codes.tolist() == case["codes"]
    q, sf2, _ = F.quantize_nvfp4(W, case["tensor_scale_in"])
    assert q.tolist() == case["q"]
    assert np.array_equal(sf2, sf)


# ---------------------------------------------------------------- round trip

def test_round_trip_every_e2m1_x_e4m3_value():
    """For every positive finite E4M3 scale S and every E2M1 code c: a block whose
    amax is 6*S*ts recovers S exactly, and the element e2m1(c)*S*ts recovers c."""
    ts = 2.0 ** -4                                     # power of two: all products exact in fp32
    S_codes = np.arange(1, 0x7F, dtype=np.uint8)       # 126 positive finite scales
    assert len(S_codes) == 126
    rows = []
    for s in S_codes:
        S = F.E4M3_VALUES[s]
        row = np.empty(32, dtype=np.float64)
        # block 0: amax element, then the 15 other codes
        row[0] = 6.0 * S * ts
        row[1:16] = F.E2M1_VALUES[[c for c in range(16) if c != 7]] * S * ts
        # block 1: amax element first, then code 7 and some repeats
        row[16] = -6.0 * S * ts
        row[17:32] = F.E2M1_VALUES[[7, 8, 0, 15, 1, 9, 2, 10, 3, 11, 4, 12, 5, 13, 6]] * S * ts
        rows.append(row)
    W = np.array(rows)
    assert np.array_equal(W.astype(np.float32).astype(np.float64), W)   # exact in fp32
    codes, sf, got_ts = F.quantize_codes(W.astype(np.float32), ts)
    assert float(got_ts) == ts
    assert np.array_equal(sf[:, 0], S_codes) and np.array_equal(sf[:, 1], S_codes)
    want0 = [7] + [c for c in range(16) if c != 7]
    want1 = [15, 7, 8, 0, 15, 1, 9, 2, 10, 3, 11, 4, 12, 5, 13, 6]
    assert (codes[:, :16] == np.array(want0, dtype=np.uint8)).all()
    assert (codes[:, 16:] == np.array(want1, dtype=np.uint8)).all()
    # and dequant(quant(W)) == W bit for bit, including the sign of zero
    deq = F.dequantize_nvfp4(F.pack_codes(codes), sf, ts)
    assert np.array_equal(deq, W)
    assert np.array_equal(np.signbit(deq), np.signbit(W))


# ---------------------------------------------------------------- scales and degenerate cases

def test_tensor_scale_closed_form():
    W = np.array([[0.0] * 15 + [-2688.0]], dtype=np.float32)
    assert float(F.tensor_scale(W)) == 1.0
    W = np.array([[0.0] * 15 + [1.0]], dtype=np.float32)
    assert float(F.tensor_scale(W)) == float(np.float32(1.0 / 2688.0))


def test_all_zero_weight():
    codes, sf, ts = F.quantize_codes(np.zeros((3, 32), np.float32))
    assert float(ts) == 0.0 and not codes.any() and not sf.any()


def test_zero_block_scale_gives_plus_zero_codes():
    # block 1 is 1e-30 relative to the tensor amax: S rounds to 0, codes must be +0 even for negatives
    W = np.zeros((1, 32), np.float32)
    W[0, 0] = 1000.0
    W[0, 16:] = -1e-27
    codes, sf, ts = F.quantize_codes(W)
    assert sf[0, 1] == 0 and (codes[0, 16:] == 0).all()


def test_negative_zero_code():
    W = np.zeros((1, 16), np.float32)
    W[0, 0] = 6.0
    W[0, 1] = -0.1
    W[0, 2] = -0.0
    codes, _, _ = F.quantize_codes(W, 1.0)
    assert codes[0, 1] == 8 and codes[0, 2] == 8 and codes[0, 3] == 0


def test_block_scale_never_exceeds_448():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    _, sf, _ = F.quantize_codes(W)
    assert F.E4M3_VALUES[sf].max() <= 448.0
    assert (sf == 0x7E).any()                          # the amax block saturates at exactly 448


def test_pack_layout_byte_level():
    codes = np.array([[1, 2, 3, 4, 15, 0, 8, 7]], dtype=np.uint8)
    q = F.pack_codes(codes)
    assert q.tolist() == [[0x21, 0x43, 0x0F, 0x78]]
    assert np.array_equal(F.unpack_codes(q), codes)


def test_dequant_matches_scalar_definition():
    rng = np.random.default_rng(4)
    q = rng.integers(0, 256, size=(3, 16), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, size=(3, 2), dtype=np.uint8)
    ts = np.float32(0.0371)
    got = F.dequantize_nvfp4(q, sf, ts)
    for n in range(3):
        for k in range(32):
            byte = int(q[n, k // 2])
            code = byte & 0xF if k % 2 == 0 else byte >> 4
            want = F.e2m1_decode(code) * F.e4m3_decode(int(sf[n, k // 16])) * float(ts)
            assert got[n, k] == want
