"""Pins of the oracle's GEMM, argmax and accept rule.

- GEMM: brute-force triple loops over the scalar format definitions (no numpy
  matmul, no vectorised dequant), exact rational arithmetic on a tiny case, and
  linearity.
- argmax: a lowest-index tie-break, checked against torch's CPU argmax.
- Accept rule: invariants (0 <= L <= D, the committed tokens are the target's
  argmax, D = 0 gives L = 0, a known prefix is given back), brute-force
  enumeration on a tiny vocabulary, and the synthetic drafts whose true accept
  length is L*.
"""

import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F
from oracle import verify as V


def _scalar_weight(q, sf, ts, n, k):
    byte = int(q[n, k // 2])
    code = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
    return F.e2m1_decode(code) * F.e4m3_decode(int(sf[n, k // 16])) * float(ts)


def _scalar_bf16(bits):
    b = int(bits)
    sign = -1.0 if b >> 15 else 1.0
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    if e == 0:
        return sign * 2.0 ** -126 * (m / 128.0)
    return sign * 2.0 ** (e - 127) * (1.0 + m / 128.0)


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (2, 3, 32), (4, 4, 64), (3, 5, 48)])
def test_gemm_brute_force_triple_loop(M, N, K):
    W, x = S.random_case(100 + M * N + K, M, N, K, w_std=1.0)
    q, sf, ts = F.quantize_nvfp4(W)
    y = G.gemm_ref(x, q, sf, ts)
    for m in range(M):
        for n in range(N):
            terms = [_scalar_bf16(x[m, k]) * _scalar_weight(q, sf, ts, n, k) for k in range(K)]
            assert y[m, n] == pytest.approx(math.fsum(terms), rel=1e-14, abs=1e-300)


def test_gemm_exact_rational_tiny():
    """Exact rational arithmetic (Fractions) on a 2x2x32 case: float64 BLAS agrees to 1e-15."""
    W, x = S.random_case(7, 2, 2, 32, w_std=1.0)
    q, sf, ts = F.quantize_nvfp4(W)
    y = G.gemm_ref(x, q, sf, ts)
    for m in range(2):
        for n in range(2):
            exact = sum(Fraction(_scalar_bf16(x[m, k])) * Fraction(_scalar_weight(q, sf, ts, n, k)) for k in range(32))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(1, 10 ** 15) * (1 + abs(exact))


def test_gemm_bf16_decode_matches_scalar():
    bits = np.array([0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x4049, 0x8000], dtype=np.uint16)
    got = G.bf16_bits_to_float64(bits)
    want = [_scalar_bf16(b) for b in bits]
    assert list(got) == want


def test_gemm_linear_in_x_and_zero():
    W, x = S.random_case(9, 3, 40, 64)
    q, sf, ts = F.quantize_nvfp4(W)
    y = G.gemm_ref(x, q, sf, ts)
    zero = np.zeros_like(x)
    assert not G.gemm_ref(zero, q, sf, ts).any()
    neg = x ^ np.uint16(0x8000)                       # flip every bf16 sign bit
    assert np.array_equal(G.gemm_ref(neg, q, sf, ts), -y)


def test_gemm_row_chunking_is_invisible():
    W, x = S.random_case(10, 2, 100, 64)
    q, sf, ts = F.quantize_nvfp4(W)
    assert np.array_equal(G.gemm_ref(x, q, sf, ts, row_chunk=7), G.gemm_ref(x, q, sf, ts, row_chunk=1000))


# ---------------------------------------------------------------- argmax

def test_argmax_lowest_index_on_ties():
    y = np.array([[1.0, 3.0, 3.0, 2.0], [5.0, 5.0, 5.0, 5.0], [-1.0, -2.0, -1.0, -3.0]])
    assert V.argmax_ref(y).tolist() == [1, 0, 0]
    assert V.argmax_fast(y).tolist() == [1, 0, 0]


def test_argmax_matches_torch():
    rng = np.random.default_rng(5)
    y = np.round(rng.standard_normal((9, 300)), 1)     # coarse values: many ties
    t = torch.from_numpy(y).argmax(dim=1).numpy()
    assert np.array_equal(V.argmax_ref(y), t)
    assert np.array_equal(V.argmax_fast(y), t)


def test_top2_gap():
    y = np.array([[1.0, 3.0, 2.5], [4.0, 4.0, 0.0]])
    assert V.top2_gap(y).tolist() == [0.5, 0.0]


# ---------------------------------------------------------------- accept rule

def _brute_accept(t, d, D):
    """Longest prefix of d that equals the target tokens, by direct comparison of every prefix."""
    best = 0
    for L in range(D + 1):
        if all(d[i] == t[i] for i in range(L)):
            best = L
    return best


def test_accept_brute_force_enumeration():
    D = 3
    for t in itertools.product(range(2), repeat=D + 1):
        for d in itertools.product(range(2), repeat=D):
            L = V.accept_ref(np.array(t), np.array([d]), D)
            assert L.tolist() == [_brute_accept(t, d, D)]


def test_accept_invariants_random():
    rng = np.random.default_rng(6)
    B, D, vocab = 50, 16, 5
    t = rng.integers(0, vocab, size=B * (D + 1))
    d = rng.integers(0, vocab, size=(B, D))
    L = V.accept_ref(t, d, D)
    assert ((L >= 0) & (L <= D)).all()
    for b, toks in enumerate(V.committed_ref(t, L, D)):
        assert len(toks) == L[b] + 1
        assert np.array_equal(toks, t[b * (D + 1): b * (D + 1) + L[b] + 1])   # committed = target argmax
        assert np.array_equal(toks[:-1], d[b, :L[b]])                        # accepted drafts are the drafts


def test_accept_D_zero():
    t = np.array([4, 9])
    assert V.accept_ref(t, np.zeros((2, 0), np.int64), 0).tolist() == [0, 0]


def test_synthetic_drafts_give_known_prefix():
    rng = np.random.default_rng(7)
    D, vocab, B = 16, 50, 40
    t = rng.integers(0, vocab, size=B * (D + 1))
    Lstar = rng.integers(0, D + 1, size=B)
    d = S.drafts_with_prefix(t, Lstar, D, vocab)
    assert np.array_equal(V.accept_ref(t, d, D), Lstar)


def test_comparable_sequences():
    gap = np.array([1.0, 1e-4, 1.0, 1.0, 1.0, 1.0])
    L = np.array([0, 2])          # B = 2, D = 2
    assert V.comparable_sequences(gap, L, 2).tolist() == [True, True]
    L = np.array([1, 2])
    assert V.comparable_sequences(gap, L, 2).tolist() == [False, True]


# ----------------------------------------------------------------------------- tree verify

def _golden_trees():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "tree_verify.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_trees(), ids=lambda c: c["name"])
def test_tree_verify_hand_worked(case):
    p = np.array([case["parents"]])
    d = np.array([case["drafts"]])
    t = np.array(case["t"])
    D = p.shape[1]
    L, node = V.accept_tree_ref(t, d, p, D)
    assert (L.tolist(), node.tolist()) == ([case["accept_len"]], [case["accept_node"]])
    assert V.committed_tree_ref(t, d, p, node, D)[0].tolist() == case["committed"]


def _brute_tree(t, d, p, D):
    """Every root-to-node path spelled out; a path is kept when each of its drafts equals the
    target token at the row of the node before it. Longest kept path, lowest end node."""
    best_len, best_node = 0, 0
    for end in range(1, D + 1):
        path = []
        k = end
        while k != 0:
            path.append(k)
            k = int(p[k - 1])
        path.reverse()
        prev, ok = 0, True
        for k in path:
            ok = ok and d[k - 1] == t[prev]
            prev = k
        if ok and len(path) > best_len:
            best_len, best_node = len(path), end
    return best_len, best_node


def test_tree_verify_brute_force_random():
    rng = np.random.default_rng(31)
    for _ in range(400):
        D = int(rng.integers(0, 9))
        p = np.array([[int(rng.integers(0, k)) for k in range(1, D + 1)]], dtype=np.int64).reshape(1, D)
        t = rng.integers(0, 3, size=D + 1)
        d = rng.integers(0, 3, size=(1, D))
        L, node = V.accept_tree_ref(t, d, p, D)
        assert (int(L[0]), int(node[0])) == _brute_tree(t, d[0], p[0], D)


def test_tree_verify_chain_is_the_accept_rule():
    rng = np.random.default_rng(32)
    B, D, vocab = 30, 16, 3
    t = rng.integers(0, vocab, size=B * (D + 1))
    d = rng.integers(0, vocab, size=(B, D))
    chain = np.tile(np.arange(D), (B, 1))
    L, node = V.accept_tree_ref(t, d, chain, D)
    assert np.array_equal(L, V.accept_ref(t, d, D))
    assert np.array_equal(node, L)


def test_tree_verify_invariants_and_generators():
    rng = np.random.default_rng(33)
    B, D, vocab = 40, 24, 7
    t = rng.integers(0, vocab, size=B * (D + 1))
    p = S.random_tree(B, D, seed=5)
    assert all(0 <= p[b, k - 1] < k for b in range(B) for k in range(1, D + 1))
    d = S.tree_drafts(t, p, D, vocab, agree=0.8, seed=6)
    L, node = V.accept_tree_ref(t, d, p, D)
    for b, toks in enumerate(V.committed_tree_ref(t, d, p, node, D)):
        path = V.tree_path(p, b, int(node[b]))
        assert len(path) == L[b] and len(toks) == L[b] + 1
        rows = [0] + path                        # committed tokens are the target's greedy tokens along the path
        assert toks.tolist() == [int(t[b * (D + 1) + r]) for r in rows]
    assert (L > 0).any() and (L < D).all()


def test_tree_verify_rejects_bad_parent():
    with pytest.raises(ValueError):
        V.accept_tree_ref(np.array([1, 2, 3]), np.array([[1, 2]]), np.array([[0, 2]]), 2)


def test_comparable_tree_sequences():
    gap = np.array([1.0, 1.0, 1e-4, 1.0, 1.0, 1.0])   # B = 2, D = 2
    assert V.comparable_tree_sequences(gap, None, 2).tolist() == [False, True]
