"""FP8 (E4M3) block-scaled weights and their GEMM in plain float64 (oracle; test
infrastructure only).

What the pages fix: the output head (and, in the vendor's export, the attention
projections) are FP8 E4M3. "TandemLLM", "The parts", loads its output head in FP8
(e4m3) from the vendor's FP8 checkpoint; "Qwen3.8 on DGX Spark (GB10)" describes a
lane whose experts use block-scaled FP8, and its 27B export keeps every linear-
and self-attention projection (48 and 16 of them) in FP8.

What the pages leave open, with the reading taken here:

* Scale granularity. Block scaling is named without a block shape. Reading: one FP32 scale per
  block of ``br x bc`` weights (rows x K), 128 x 128 by default, the block shape the
  vendor's FP8 checkpoints use. The block shape is a parameter so that small blocks
  can be worked by hand.
* Scale value. ``s = fp32(amax_block / 448)``: the block's largest magnitude maps to
  E4M3's largest finite value. A zero block has s = 0 and all codes +0.
* Codes. ``c = E4M3_rne_satfinite(w / s)`` with the quotient formed in float64 and the
  sign kept (a negative value that rounds to zero gives -0, code 0x80), as for the
  NVFP4 weights.
* Dequantisation ``w_hat = e4m3(c) * s`` is exact in float64 (4 + 24 significant
  bits), and so is the product with a bf16 activation; only the float64 sums round.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import E4M3_MAX, E4M3_VALUES, e4m3_encode

BLOCK = (128, 128)


def quantize_fp8_blocks(W: np.ndarray, block=BLOCK):
    """fp32 W [N, K] -> ``(codes uint8 [N, K], scales float32 [ceil(N/br), ceil(K/bc)])``.

    Edge blocks (N or K not a multiple of the block) are the partial blocks that
    remain; their scale comes from the elements they hold.
    """
    W = np.asarray(W, dtype=np.float32)
    if W.ndim != 2:
        raise ValueError("W must be [N, K]")
    N, K = W.shape
    br, bc = block
    nb_r, nb_c = -(-N // br), -(-K // bc)
    scales = np.zeros((nb_r, nb_c), dtype=np.float32)
    codes = np.zeros((N, K), dtype=np.uint8)
    for i in range(nb_r):
        for j in range(nb_c):
            blk = W[i * br:(i + 1) * br, j * bc:(j + 1) * bc].astype(np.float64)
            amax = float(np.max(np.abs(blk))) if blk.size else 0.0
            s = np.float32(amax / E4M3_MAX)
            scales[i, j] = s
            if s == 0:
                continue
            codes[i * br:(i + 1) * br, j * bc:(j + 1) * bc] = e4m3_encode(blk / float(s))
    return codes, scales


def dequantize_fp8_blocks(codes: np.ndarray, scales: np.ndarray, block=BLOCK) -> np.ndarray:
    """w_hat[n, k] = e4m3(code[n, k]) * s[n // br, k // bc], in float64 (exact)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    br, bc = block
    s = np.repeat(np.repeat(np.asarray(scales, dtype=np.float64), br, axis=0), bc, axis=1)[:N, :K]
    return E4M3_VALUES[codes] * s


def gemm_fp8_ref(x_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, block=BLOCK) -> np.ndarray:
    """Y = x . w_hat^T in float64 for bf16 X given as uint16 bit patterns."""
    from .gemm import bf16_bits_to_float64

    x = bf16_bits_to_float64(x_bits)
    w_hat = dequantize_fp8_blocks(codes, scales, block)
    if w_hat.shape[1] != x.shape[1]:
        raise ValueError("K mismatch between X and W")
    return x @ w_hat.T
