"""The oracle over the whole 248,320-row lm_head, chunk by chunk on a process pool (test
infrastructure; it runs only ``oracle/`` and ``synthetic/`` code).

The float64 oracle quantises and multiplies one 4,096-row chunk of the head in about five
seconds on one core, so the full vocabulary takes minutes in one process. Here each chunk
is a task for a pool of worker processes started with ``spawn`` (a forked child of a
process that holds a CUDA context can hang). Each worker draws its chunk of the seeded
weight itself (``synthetic.lmhead_weight_chunk``). It quantises the chunk with the tensor
scale of the whole weight (``oracle.nvfp4.quantize_nvfp4``), multiplies it
(``oracle.gemm.gemm_ref``), and returns the packed bytes with each row's best two logits
and the index of the first maximum. Joining the chunks in index order gives the argmax
over the whole vocabulary with the lowest index on ties (``oracle.verify.argmax_ref``'s
rule) and the top-2 gap (``oracle.verify.top2_gap``).
"""

from __future__ import annotations

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

_CACHE: dict = {}


def _init_worker():
    try:                                    # one BLAS thread per worker: the pool supplies the parallelism
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _chunk_amax(c: int, N: int, K: int) -> float:
    return float(np.max(np.abs(S.lmhead_weight_chunk(c, N, K).astype(np.float64))))


def _chunk_logits(c: int, N: int, K: int, ts, x_bits: np.ndarray):
    W = S.lmhead_weight_chunk(c, N, K)
    q, sf, _ = F.quantize_nvfp4(W, ts)
    y = G.gemm_ref(x_bits, q, sf, ts)                      # [M, rows], float64
    idx = np.argmax(y, axis=1)                             # first maximum of the chunk
    part = -np.partition(-y, 1, axis=1) if y.shape[1] > 1 else np.concatenate([y, np.full_like(y, -np.inf)], 1)
    return c, q, sf, idx + c * S.LMHEAD_CHUNK, part[:, 0], part[:, 1]


def _workers() -> int:
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    return max(1, min(n, 32))


def lmhead_oracle(x_bits: np.ndarray, N: int = S.VOCAB, K: int = S.LMHEAD_K) -> dict:
    """The oracle's result on the seeded lm_head for the activation rows ``x_bits``.

    Returns a dict with ``q`` uint8 [N, K/2], ``sf`` uint8 [N, K/16] and ``ts`` float32 (the
    oracle's packing of the weight), ``t`` int64 [M] (argmax, lowest index on ties),
    ``top1`` and ``top2`` float64 [M] (the two largest logits) and ``gap`` = top1 - top2.
    Cached per (x, N, K) for the life of the process.
    """
    key = (x_bits.tobytes(), N, K)
    if key in _CACHE:
        return _CACHE[key]
    chunks = -(-N // S.LMHEAD_CHUNK)
    ctx = multiprocessing.get_context("spawn")
    with ProcessPoolExecutor(max_workers=_workers(), mp_context=ctx, initializer=_init_worker) as ex:
        amax = max(ex.map(_chunk_amax, range(chunks), [N] * chunks, [K] * chunks))
        ts = F.tensor_scale(np.array([[amax]], dtype=np.float32))          # the oracle's ts of the whole weight
        M = x_bits.shape[0]
        q = np.empty((N, K // 2), dtype=np.uint8)
        sf = np.empty((N, K // 16), dtype=np.uint8)
        parts = [None] * chunks
        for c, qc, sfc, idx, p1, p2 in ex.map(_chunk_logits, range(chunks), [N] * chunks, [K] * chunks,
                                              [ts] * chunks, [x_bits] * chunks):
            n0 = c * S.LMHEAD_CHUNK
            q[n0: n0 + qc.shape[0]] = qc
            sf[n0: n0 + sfc.shape[0]] = sfc
            parts[c] = (idx, p1, p2)
    t = np.zeros(M, dtype=np.int64)
    top1 = np.full(M, -np.inf)
    top2 = np.full(M, -np.inf)
    for idx, p1, p2 in parts:                              # in index order: a strict > keeps the first maximum
        better = p1 > top1
        second = np.where(better, np.maximum(top1, p2), np.maximum(top2, p1))
        t = np.where(better, idx, t)
        top1 = np.where(better, p1, top1)
        top2 = second
    out = {"q": q, "sf": sf, "ts": ts, "t": t, "top1": top1, "top2": top2, "gap": top1 - top2}
    _CACHE[key] = out
    return out


def logit(orc: dict, x_bits: np.ndarray, m: int, n: int) -> float:
    """The oracle's logit y[m, n] from its packed weight (one row, exact in float64)."""
    return float(G.gemm_ref(x_bits[m: m + 1], orc["q"][n: n + 1], orc["sf"][n: n + 1], orc["ts"])[0, 0])
