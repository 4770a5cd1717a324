"""Seeded synthetic inputs for the NVFP4 skinny GEMM and greedy verify.

This module draws random numbers and shapes only. It holds none of the method's
arithmetic: no quantisation, no GEMM, no argmax. Tests hand its arrays to both
the CPU oracle and the CUDA library, and ``bench.py`` uses it too.

Workloads. The pages measure recorded agent sessions; these seeded arrays with
the same shapes stand in for them:

* tiny        M=1, K=N=1024. W ~ N(0, 0.02) from ``default_rng(0)``; X ~ N(0, 1)
              from the next draw of the same generator, rounded to bf16.
* layer       the three matrix shapes of one 27B layer: gate+up fused
              5120->34816, down 17408->5120, and qkv / delta projection
              5120->10240. W seeds 1, 2, 3 and X seeds 101, 102, 103.
* stack       64 layers of the three layer shapes (192 matrices, 11.51 GB
              NVFP4), with M=17 (verify) or M=68 (4 sequences x 17).
* lm_head     K=5120, N=248320, or the first 65,536 rows as the sliced draft
              vocabulary. W is drawn in chunks of 4,096 rows, chunk c from its own
              generator default_rng([7, c]), so any chunk can be drawn alone (the
              full-vocabulary oracle draws them in parallel). X seed 107, prefix
              lengths L* ~ U{0..16} from seed 207.
* sweep       M in {1, 2, 4, 8, 17, 34, 68, 128} on the gate+up shape.
"""

from __future__ import annotations

import numpy as np

W_STD = 0.02

LAYER_SHAPES = {            # name -> (K, N)
    "gate_up": (5120, 34816),
    "down": (17408, 5120),
    "qkv": (5120, 10240),
}
LAYER_ORDER = ("gate_up", "down", "qkv")
LAYER_W_SEEDS = {"gate_up": 1, "down": 2, "qkv": 3}
LAYER_X_SEEDS = {"gate_up": 101, "down": 102, "qkv": 103}
N_LAYERS = 64
VOCAB = 248320
VOCAB_SLICE = 65536
LMHEAD_K = 5120
LMHEAD_W_SEED, LMHEAD_X_SEED, LMHEAD_L_SEED = 7, 107, 207
DRAFT_LEN = 16               # 16 drafted tokens + 1 => M = 17 per sequence
SWEEP_M = (1, 2, 4, 8, 17, 34, 68, 128)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def normal_weight(rng: np.random.Generator, N: int, K: int, std: float = W_STD, row_chunk: int = 4096) -> np.ndarray:
    """fp32 [N, K] ~ N(0, std^2), drawn row-chunk by row-chunk from ``rng``. The
    chunked draw gives the same stream as one ``standard_normal((N, K))`` call."""
    W = np.empty((N, K), dtype=np.float32)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        W[n0:n1] = (rng.standard_normal((n1 - n0, K)) * std).astype(np.float32)
    return W


def normal_x_bits(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    """bf16 [M, K] ~ N(0, 1) as uint16 bit patterns."""
    return f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))


def tiny():
    """The tiny case: returns ``(W fp32 [1024, 1024], x_bits uint16 [1, 1024])``."""
    rng = np.random.default_rng(0)
    W = normal_weight(rng, 1024, 1024)
    x = normal_x_bits(rng, 1, 1024)
    return W, x


def layer(name: str, M: int = 1, w_seed: int | None = None, x_seed: int | None = None):
    """One layer matrix: returns ``(W fp32 [N, K], x_bits uint16 [M, K])``."""
    K, N = LAYER_SHAPES[name]
    W = normal_weight(np.random.default_rng(LAYER_W_SEEDS[name] if w_seed is None else w_seed), N, K)
    x = normal_x_bits(np.random.default_rng(LAYER_X_SEEDS[name] if x_seed is None else x_seed), M, K)
    return W, x


def random_case(seed: int, M: int, N: int, K: int, w_std: float = W_STD):
    """A generic seeded case of any shape: ``(W fp32 [N, K], x_bits [M, K])``."""
    rng = np.random.default_rng(seed)
    return normal_weight(rng, N, K, w_std), normal_x_bits(rng, M, K)


def block_varied_case(seed: int, M: int, N: int, K: int, block: int = 128, spread: int = 4):
    """Like ``random_case``, with each ``block x block`` tile of W multiplied by its own power
    of two 2^e, e ~ U{-spread..spread}: per-block scales then differ by up to 2^(2 spread), so
    a scale applied to the wrong block is visible in Y."""
    rng = np.random.default_rng(seed)
    W = normal_weight(rng, N, K)
    e = rng.integers(-spread, spread + 1, size=(-(-N // block), -(-K // block)))
    f = np.repeat(np.repeat(np.ldexp(1.0, e), block, axis=0), block, axis=1)[:N, :K]
    W = (W * f).astype(np.float32)
    return W, normal_x_bits(rng, M, K)


LMHEAD_CHUNK = 4096


def lmhead_weight_chunk(c: int, N: int = VOCAB, K: int = LMHEAD_K) -> np.ndarray:
    """Rows [4096 c, min(N, 4096 (c + 1))) of the lm_head weight: fp32 ~ N(0, 0.02^2) from
    ``default_rng([7, c])``."""
    n0 = c * LMHEAD_CHUNK
    rows = min(N, n0 + LMHEAD_CHUNK) - n0
    return (np.random.default_rng([LMHEAD_W_SEED, c]).standard_normal((rows, K)) * W_STD).astype(np.float32)


def lmhead_weight(N: int = VOCAB, K: int = LMHEAD_K) -> np.ndarray:
    """The lm_head weight fp32 [N, K], chunk by chunk (see lmhead_weight_chunk)."""
    W = np.empty((N, K), dtype=np.float32)
    for c in range(-(-N // LMHEAD_CHUNK)):
        n0 = c * LMHEAD_CHUNK
        W[n0: n0 + LMHEAD_CHUNK] = lmhead_weight_chunk(c, N, K)
    return W


def lmhead_x(B: int = 1, D: int = DRAFT_LEN, K: int = LMHEAD_K) -> np.ndarray:
    """lm_head hidden states bf16 [B*(D+1), K]; the rows of B sequences start with those of B' < B."""
    return normal_x_bits(np.random.default_rng(LMHEAD_X_SEED), B * (D + 1), K)


def lmhead_lstar(B: int = 1, D: int = DRAFT_LEN) -> np.ndarray:
    """Prefix lengths L* ~ U{0..D}, int64 [B]."""
    return np.random.default_rng(LMHEAD_L_SEED).integers(0, D + 1, size=B)


def lmhead_inputs(N: int = VOCAB, B: int = 1, D: int = DRAFT_LEN, K: int = LMHEAD_K):
    """lm_head weight, hidden states and prefix lengths.

    Returns ``(W fp32 [N, K], x_bits [B*(D+1), K], Lstar int64 [B])``. With N=65536
    this is the sliced draft vocabulary: the first 65,536 rows of the full weight.
    """
    return lmhead_weight(N, K), lmhead_x(B, D, K), lmhead_lstar(B, D)


def drafts_with_prefix(t: np.ndarray, Lstar: np.ndarray, D: int, vocab: int, seed: int = 208) -> np.ndarray:
    """Drafts whose agreement with the target tokens ``t`` is exactly ``Lstar[b]``.

    Slots i < L* copy the target token of slot i. Slots i >= L* are uniform random
    ids. Slot L* is redrawn while it equals the target token, so the first
    disagreement is at L*. Returns int32 [B, D].
    """
    t = np.asarray(t, dtype=np.int64)
    B = len(Lstar)
    rng = np.random.default_rng(seed)
    d = rng.integers(0, vocab, size=(B, D)).astype(np.int64)
    for b in range(B):
        Ls = int(Lstar[b])
        base = b * (D + 1)
        d[b, :Ls] = t[base: base + Ls]
        if Ls < D:
            while d[b, Ls] == t[base + Ls]:
                d[b, Ls] = rng.integers(0, vocab)
    return d.astype(np.int32)


def random_tree(B: int, D: int, seed: int = 209, chain_bias: float = 0.5) -> np.ndarray:
    """Parent arrays of B draft trees with nodes 1..D: int32 [B, D], the parent of node
    k in [0, k-1]. With probability ``chain_bias`` a node hangs under node k-1 (deep
    branches), else under a uniform earlier node (wide trees)."""
    rng = np.random.default_rng(seed)
    p = np.zeros((B, D), dtype=np.int64)
    for b in range(B):
        for k in range(1, D + 1):
            p[b, k - 1] = k - 1 if rng.random() < chain_bias else rng.integers(0, k)
    return p.astype(np.int32)


def tree_drafts(t: np.ndarray, parents: np.ndarray, D: int, vocab: int, agree: float = 0.7,
                seed: int = 210) -> np.ndarray:
    """Draft tokens for the trees in ``parents``: node k copies the target token ``t`` at
    its parent's row with probability ``agree``, else a different uniform id."""
    t = np.asarray(t, dtype=np.int64)
    parents = np.asarray(parents, dtype=np.int64)
    B = parents.shape[0]
    rng = np.random.default_rng(seed)
    d = np.zeros((B, D), dtype=np.int64)
    for b in range(B):
        for k in range(1, D + 1):
            want = t[b * (D + 1) + parents[b, k - 1]]
            if rng.random() < agree:
                d[b, k - 1] = want
            else:
                x = rng.integers(0, vocab)
                while x == want:
                    x = rng.integers(0, vocab)
                d[b, k - 1] = x
    return d.astype(np.int32)
