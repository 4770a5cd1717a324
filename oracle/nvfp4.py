"""NVFP4 format, quantiser and dequantiser in plain float64 (oracle; test infrastructure only).

What the pages fix: the weights are NVFP4 with groups of 16 ("Qwen3.8 on DGX Spark
(GB10)", section "The seven targets, and switching between them"). That is 4-bit E2M1
values, one FP8 E4M3 scale for every 16 consecutive elements along K, and one
FP32 scale per tensor.

What the pages leave open, with the reading taken here:

* Bit encodings. E2M1 is sign, 2 exponent bits with bias 1 and 1 mantissa bit; an
  exponent field of 0 is subnormal (value = mantissa/2). E4M3 is sign, 4 exponent
  bits with bias 7 and 3 mantissa bits; exponent 0 is subnormal (2^-6 * m/8). It
  has no infinity, and S.1111.111 is NaN, so the largest finite value is 448.
* Scales. The tensor scale is ``ts = fp32(amax(|W|) / (6 * 448))``. The block
  scale is relative to it: ``S = E4M3(amax_block / (6 * ts))``. That keeps every
  block scale at or below 448.
* Rounding. Round to nearest, ties to even (the even mantissa bit), with
  saturation to the largest finite value. The code of an element is the E2M1
  rounding of ``w / (S * ts)``, using the *rounded* S. The sign of w is kept, so a
  negative value that rounds to zero gets the code 0x8 (-0).
* Degenerate cases. If ts == 0 every code and every scale is 0. If a block's
  S == 0 its codes are all +0.
* Precision of the scale arithmetic. Both quotients are formed in float64. The
  products ``6 * ts`` and ``S * ts`` are exact there: 24 significant bits times 2
  or 4 significant bits.
* Packing. ``q[n, j] = code[n, 2j] | code[n, 2j+1] << 4``, row-major [N, K/2].
  ``sf[n, b]`` holds the E4M3 bits of block b (elements 16b .. 16b+15), row-major
  [N, K/16].
"""

from __future__ import annotations

import math

import numpy as np

GROUP = 16                 # elements per block scale
E2M1_MAX = 6.0             # largest finite E2M1 magnitude
E4M3_MAX = 448.0           # largest finite E4M3 magnitude
TENSOR_SCALE_DIVISOR = E2M1_MAX * E4M3_MAX   # 2688


# ----------------------------------------------------------------------------
# Value sets, from the bit fields
# ----------------------------------------------------------------------------

def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0."""
    sign = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = m * 0.5                        # subnormal: 2^(1-1) * (m / 2)
    else:
        mag = 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return sign * mag


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0."""
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        mag = 2.0 ** -6 * (m / 8.0)          # subnormal
    else:
        mag = 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return sign * mag


E2M1_VALUES = np.array([e2m1_decode(c) for c in range(16)], dtype=np.float64)
E4M3_VALUES = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
# non-negative finite values in code order (codes 0..7 and 0x00..0x7E are monotone)
_E2M1_POS = E2M1_VALUES[:8].copy()
_E4M3_POS = E4M3_VALUES[:0x7F].copy()


# ----------------------------------------------------------------------------
# Round to nearest even with saturation
# ----------------------------------------------------------------------------

def _rne_on_grid(a: np.ndarray, min_exp: int, man_bits: int) -> np.ndarray:
    """Round non-negative ``a`` to the nearest value of a binary format with
    ``man_bits`` mantissa bits and smallest normal exponent ``min_exp``.

    In the binade [2^E, 2^(E+1)) the spacing is 2^(E - man_bits). Below 2^min_exp
    the subnormals share the spacing of the lowest binade. ``a / spacing`` is exact
    (a power-of-two division), and ``np.rint`` rounds halves to even. Within a
    binade an even quotient means an even mantissa bit.
    """
    a = np.asarray(a, dtype=np.float64)
    _, ex = np.frexp(a)                         # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, min_exp)             # floor(log2 a), clamped at the subnormal binade
    spacing_exp = e - man_bits
    n = np.rint(np.ldexp(a, -spacing_exp))
    return np.ldexp(n, spacing_exp)


def e2m1_round_magnitude(a: np.ndarray) -> np.ndarray:
    """RNE of |r| onto {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating at 6."""
    a = np.asarray(a, dtype=np.float64)
    r = _rne_on_grid(np.minimum(a, E2M1_MAX), min_exp=0, man_bits=1)
    return np.minimum(r, E2M1_MAX)


def e4m3_round_magnitude(a: np.ndarray) -> np.ndarray:
    """RNE of |v| onto the finite E4M3 magnitudes, saturating at 448."""
    a = np.asarray(a, dtype=np.float64)
    r = _rne_on_grid(np.minimum(a, E4M3_MAX), min_exp=-6, man_bits=3)
    return np.minimum(r, E4M3_MAX)


def e2m1_encode(r: np.ndarray) -> np.ndarray:
    """E2M1 code (uint8, 0..15) of the RNE-satfinite rounding of r; sign of r kept (so -0 -> 0x8)."""
    r = np.asarray(r, dtype=np.float64)
    if np.isnan(r).any():
        raise ValueError("NaN has no E2M1 code")
    mag = e2m1_round_magnitude(np.abs(r))
    code = np.searchsorted(_E2M1_POS, mag).astype(np.uint8)
    assert np.array_equal(_E2M1_POS[code], mag), "rounded magnitude not on the E2M1 grid"
    return code | (np.signbit(r).astype(np.uint8) << 3)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """E4M3 code (uint8) of the RNE-satfinite rounding of v; sign of v kept. NaN is never produced."""
    v = np.asarray(v, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN is not encoded")
    mag = e4m3_round_magnitude(np.abs(v))
    code = np.searchsorted(_E4M3_POS, mag).astype(np.uint8)
    assert np.array_equal(_E4M3_POS[code], mag), "rounded magnitude not on the E4M3 grid"
    return code | (np.signbit(v).astype(np.uint8) << 7)


# ----------------------------------------------------------------------------
# Quantise / dequantise / pack
# ----------------------------------------------------------------------------

def tensor_scale(W: np.ndarray) -> np.float32:
    """ts = fp32(float64(amax|W|) / 2688). Zero for an all-zero tensor."""
    W = np.asarray(W, dtype=np.float32)
    amax = float(np.max(np.abs(W.astype(np.float64)))) if W.size else 0.0
    return np.float32(amax / TENSOR_SCALE_DIVISOR)


def quantize_codes(W: np.ndarray, tensor_scale_in=None):
    """Two-level NVFP4 quantisation of fp32 W [N, K] (K a multiple of 16).

    Returns ``(codes uint8 [N, K], sf uint8 [N, K/16], ts float32)``; ``codes`` holds
    one E2M1 code per element (unpacked).
    """
    W = np.asarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % GROUP:
        raise ValueError("W must be [N, K] with K a multiple of 16")
    N, K = W.shape
    ts = tensor_scale(W) if tensor_scale_in is None else np.float32(tensor_scale_in)
    ts64 = float(ts)
    blocks = W.astype(np.float64).reshape(N, K // GROUP, GROUP)
    if ts64 == 0.0:
        return (np.zeros((N, K), np.uint8), np.zeros((N, K // GROUP), np.uint8), ts)
    amax_b = np.max(np.abs(blocks), axis=2)
    sf = e4m3_encode(amax_b / (6.0 * ts64))
    S = E4M3_VALUES[sf]
    denom = S[:, :, None] * ts64                    # exact in float64
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(denom > 0, blocks / np.where(denom > 0, denom, 1.0), 0.0)
    codes = e2m1_encode(r)
    codes = np.where(S[:, :, None] > 0, codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(N, K), sf.astype(np.uint8), ts


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """codes uint8 [N, K] -> q uint8 [N, K/2]; element 2j in the low nibble, 2j+1 in the high."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_codes(q: np.ndarray) -> np.ndarray:
    """q uint8 [N, K/2] -> codes uint8 [N, K]."""
    q = np.asarray(q, dtype=np.uint8)
    N, H = q.shape
    codes = np.empty((N, 2 * H), dtype=np.uint8)
    codes[:, 0::2] = q & 0xF
    codes[:, 1::2] = q >> 4
    return codes


def quantize_nvfp4(W: np.ndarray, tensor_scale_in=None):
    """Quantise and pack: returns ``(q uint8 [N, K/2], sf uint8 [N, K/16], ts float32)``."""
    codes, sf, ts = quantize_codes(W, tensor_scale_in)
    return pack_codes(codes), sf, ts


def dequantize_nvfp4(q: np.ndarray, sf: np.ndarray, ts) -> np.ndarray:
    """w_hat[n, k] = e2m1(code[n, k]) * S[n, k // 16] * ts, in float64 (exact)."""
    codes = unpack_codes(q)
    N, K = codes.shape
    S = E4M3_VALUES[np.asarray(sf, dtype=np.uint8)]
    return E2M1_VALUES[codes] * np.repeat(S, GROUP, axis=1) * float(np.float32(ts))
