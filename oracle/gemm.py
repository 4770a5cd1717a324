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

from .nvfp4 import E2M1_VALUES, E4M3_VALUES, GROUP, dequantize_nvfp4, quantize_codes


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
    weights' two-level NVFP4 scheme (``oracle.nvfp4.quantize_codes``) applied to each
    row on its own, the row's amax taking the place of the tensor's:

        g   = fp32(amax|x_row| / 2688)
        S   = E4M3_rne_satfinite(amax_block / (6 g))
        c   = E2M1_rne_satfinite(x / (S g))            (+0 where S g = 0)

    with both quotients formed exactly (float64, in which 6 g and S g are exact) and
    rounded once, as for the weights.

    Returns ``(codes uint8 [M, K], sf uint8 [M, K/16], g float32 [M])``.
    """
    x = bf16_bits_to_float64(x_bits).astype(np.float32)      # exact: bf16 is an fp32 prefix
    if x.ndim != 2 or x.shape[1] % GROUP:
        raise ValueError("X must be [M, K] with K a multiple of 16")
    M, K = x.shape
    codes = np.zeros((M, K), dtype=np.uint8)
    sf = np.zeros((M, K // GROUP), dtype=np.uint8)
    g = np.zeros(M, dtype=np.float32)
    for m in range(M):                                       # each row is its own "tensor"
        codes[m:m + 1], sf[m:m + 1], g[m] = quantize_codes(x[m:m + 1])
    return codes, sf, g


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
