"""Skinny block-scaled GEMM in float64 (oracle; test infrastructure only).

The operation is ``Y[M, N] = X[M, K] . dequant(W)[N, K]^T``. X is bf16, W is NVFP4
and the accumulation is at least fp32. The pages frame this as the weight pass
that every decode or verify step makes: "TandemLLM", "How it works" (each decode
step of the 27B model streams all of its weights once), and the veloGB10 page,
section "Unique aspects: Engineered to the roofline".

Here both operands are exact in float64: a bf16 value has 8 significant bits and
a dequantised weight at most 6. The only rounding is in the float64 sums, so the
result is the exact product up to summation order.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import (E2M1_VALUES, E4M3_VALUES, GROUP, TENSOR_SCALE_DIVISOR, dequantize_nvfp4, e2m1_encode,
                    e4m3_encode)


def bf16_bits_to_float64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values. A bf16 is the top half of an fp32."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gemm_ref(x_bits: np.ndarray, q: np.ndarray, sf: np.ndarray, ts, row_chunk: int = 8192) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * w_hat[n, k] in float64.

    ``x_bits`` is bf16 [M, K] given as uint16 bit patterns. ``q``, ``sf`` and ``ts``
    are the packed NVFP4 weight. W is dequantised ``row_chunk`` rows at a time
    to bound memory. That changes no arithmetic: each output column is one dot
    product.
    """
    x = bf16_bits_to_float64(x_bits)
    if x.ndim != 2:
        raise ValueError("X must be [M, K]")
    N = q.shape[0]
    y = np.empty((x.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        w_hat = dequantize_nvfp4(q[n0:n1], sf[n0:n1], ts)
        if w_hat.shape[1] != x.shape[1]:
            raise ValueError("K mismatch between X and W")
        y[:, n0:n1] = x @ w_hat.T
    return y


# ----------------------------------------------------------------------------- W4A4 (NVFP4 activations)

def quantize_x_rows(x_bits: np.ndarray):
    """NVFP4 quantisation of bf16 activation rows, one FP32 scale per row.

    The pages run prefill on the block-scaled tensor cores with both operands in
    4 bits ("Qwen3.8 on DGX Spark (GB10)", introduction: NVFP4 on block-scaled tensor
    cores; "TandemLLM", "The parts"). They give no activation recipe. Reading: the
    weights' two-level NVFP4 scheme applied to each row, with the row's amax in place
    of the tensor's. Every decision is taken in fp32, as the kernel takes it (IEEE
    round-to-nearest; numpy float32 arithmetic is the same):

        g   = fp32(amax|x_row| / 2688)
        inv = fp32(1 / fp32(6 * g))
        S   = E4M3_rne_satfinite(fp32(amax_block * inv))
        den = fp32(S * g)
        c   = E2M1_rne_satfinite(fp32(x / den))     (0 where den = 0)

    Returns ``(codes uint8 [M, K], sf uint8 [M, K/16], g float32 [M])``.
    """
    x = bf16_bits_to_float64(x_bits).astype(np.float32)      # exact: bf16 is an fp32 prefix
    if x.ndim != 2 or x.shape[1] % GROUP:
        raise ValueError("X must be [M, K] with K a multiple of 16")
    M, K = x.shape
    amax = np.max(np.abs(x), axis=1)
    g = (amax / np.float32(TENSOR_SCALE_DIVISOR)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(g > 0, np.float32(1.0) / (np.float32(6.0) * g), np.float32(0.0)).astype(np.float32)
    blocks = x.reshape(M, K // GROUP, GROUP)
    a = (np.max(np.abs(blocks), axis=2) * inv[:, None]).astype(np.float32)
    sf = e4m3_encode(a.astype(np.float64))
    S = E4M3_VALUES[sf].astype(np.float32)
    den = (S * g[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(den[:, :, None] > 0, blocks / np.where(den > 0, den, np.float32(1.0))[:, :, None],
                     np.float32(0.0)).astype(np.float32)
    codes = e2m1_encode(r.astype(np.float64))
    codes = np.where(den[:, :, None] > 0, codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(M, K), sf.astype(np.uint8), g


def dequantize_x_rows(codes: np.ndarray, sf: np.ndarray, g: np.ndarray) -> np.ndarray:
    """x_hat[m, k] = e2m1(code) * S[m, k // 16] * g[m], in float64 (exact)."""
    M, K = codes.shape
    vals = E2M1_VALUES[np.asarray(codes, dtype=np.uint8)]
    S = E4M3_VALUES[np.asarray(sf, dtype=np.uint8)]
    return vals * np.repeat(S, GROUP, axis=1) * np.asarray(g, dtype=np.float64)[:, None]


def gemm_w4a4_ref(x_bits: np.ndarray, q: np.ndarray, sf: np.ndarray, ts, row_chunk: int = 8192) -> np.ndarray:
    """Y = x_hat . w_hat^T in float64, x_hat the NVFP4 quantisation of X (quantize_x_rows)."""
    xc, xs, g = quantize_x_rows(x_bits)
    x_hat = dequantize_x_rows(xc, xs, g)
    N = q.shape[0]
    y = np.empty((x_hat.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        w_hat = dequantize_nvfp4(q[n0:n1], sf[n0:n1], ts)
        if w_hat.shape[1] != x_hat.shape[1]:
            raise ValueError("K mismatch between X and W")
        y[:, n0:n1] = x_hat @ w_hat.T
    return y
