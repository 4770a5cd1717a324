"""Skinny block-scaled GEMM in float64 (oracle; test infrastructure only).

The operation is ``Y[M, N] = X[M, K] . dequant(W)[N, K]^T``. X is bf16, W is NVFP4
and the accumulation is at least fp32. The pages frame this as the weight pass
that every decode or verify step makes: "TandemLLM", "How it works" ("a decode
step of a 27B model reads every weight once"), and the veloGB10 page, section
"Unique aspects: Engineered to the roofline".

Here both operands are exact in float64: a bf16 value has 8 significant bits and
a dequantised weight at most 6. The only rounding is in the float64 sums, so the
result is the exact product up to summation order.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import dequantize_nvfp4


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
