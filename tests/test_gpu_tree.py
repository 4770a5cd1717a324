"""GPU parity of the draft-tree verify (lmhead_verify_tree, and a weight pass ending
in a tree verify) against the CPU oracle on the same seeded inputs.

Bars as in the chain verify: argmax bit-exact on rows whose oracle top-2 gap is
>= 1e-3; accept length and end node bit-exact on sequences with no near-tie row
(in a tree any row can decide a node's acceptance); the committed tokens rebuilt
from the GPU's end node equal the oracle's.
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F
from oracle import verify as V

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def oracle_logits(W, x):
    q, sf, ts = F.quantize_nvfp4(W)
    return G.gemm_ref(x, q, sf, ts)


def check_tree(t, L, node, y_ref, drafts, parents, D):
    t_ref = V.argmax_fast(y_ref)
    L_ref, node_ref = V.accept_tree_ref(t_ref, drafts, parents, D)
    gap = V.top2_gap(y_ref)
    rows = V.comparable_rows(gap)
    seqs = V.comparable_tree_sequences(gap, parents, D)
    assert np.array_equal(t[rows], t_ref[rows])
    assert np.array_equal(L[seqs], L_ref[seqs]) and np.array_equal(node[seqs], node_ref[seqs])
    got = V.committed_tree_ref(t, drafts, parents, node, D)
    want = V.committed_tree_ref(t_ref, drafts, parents, node_ref, D)
    for b in np.flatnonzero(seqs):
        assert np.array_equal(got[b], want[b])
    return seqs.mean(), L_ref


@pytest.mark.parametrize("B,D,bias", [(1, 16, 0.5), (4, 16, 0.3), (2, 40, 0.7), (3, 1, 0.5)])
def test_verify_tree_small_vocab(nv, B, D, bias):
    N, K = 3000, 512
    # w_std 0.2 spreads the logits so that no row of these seeds is a near tie (checked with the oracle)
    W, x = S.random_case(700 + B * 10 + D, B * (D + 1), N, K, w_std=0.2)
    y_ref = oracle_logits(W, x)
    parents = S.random_tree(B, D, seed=B + D, chain_bias=bias)
    drafts = S.tree_drafts(V.argmax_fast(y_ref), parents, D, N, agree=0.75, seed=B * D)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    t, L, node, _ = nv.verify_tree(to_dev_bf16(x), q, sf, ts, torch.from_numpy(drafts).cuda(),
                                   torch.from_numpy(parents).cuda())
    nv.check()
    frac, L_ref = check_tree(t.cpu().numpy(), L.cpu().numpy(), node.cpu().numpy(), y_ref, drafts, parents, D)
    assert frac == 1.0


def test_verify_tree_chain_matches_chain_verify(nv):
    """A chain-shaped tree gives the chain verify's accept lengths, and the end node is L."""
    B, D, N, K = 4, 16, 5000, 1024
    W, x = S.random_case(811, B * (D + 1), N, K, w_std=0.05)
    y_ref = oracle_logits(W, x)
    Lstar = np.random.default_rng(5).integers(0, D + 1, size=B)
    drafts = S.drafts_with_prefix(V.argmax_fast(y_ref), Lstar, D, N)
    chain = np.tile(np.arange(D, dtype=np.int32), (B, 1))
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    Xd, dd = to_dev_bf16(x), torch.from_numpy(drafts).cuda()
    t1, L1, _ = nv.verify(Xd, q, sf, ts, dd)
    t2, L2, node2, _ = nv.verify_tree(Xd, q, sf, ts, dd, torch.from_numpy(chain).cuda())
    torch.cuda.synchronize()
    assert torch.equal(t1, t2) and torch.equal(L1, L2) and torch.equal(node2, L2)


def test_verify_tree_lmhead_slice_m68(nv):
    """Four trees of 16 drafted nodes over the 65,536-row sliced head (M = 68)."""
    W, x, _ = S.lmhead_inputs(N=S.VOCAB_SLICE, B=4)
    D = S.DRAFT_LEN
    y_ref = oracle_logits(W, x)
    parents = S.random_tree(4, D, seed=41)
    drafts = S.tree_drafts(V.argmax_fast(y_ref), parents, D, S.VOCAB_SLICE, agree=0.8, seed=42)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    t, L, node, vmax = nv.verify_tree(to_dev_bf16(x), q, sf, ts, torch.from_numpy(drafts).cuda(),
                                      torch.from_numpy(parents).cuda())
    nv.check()
    frac, L_ref = check_tree(t.cpu().numpy(), L.cpu().numpy(), node.cpu().numpy(), y_ref, drafts, parents, D)
    # a tree is compared exactly unless one of its 17 rows is a near tie (any row can decide a
    # node); on this draw one of the four has such a row
    assert frac >= 0.75 and (L_ref > 0).any()


def test_pass_with_tree_verify_tail(nv):
    """Two GEMMs and a tree-verify lm_head in one weight pass."""
    B, D = 2, 16
    M = B * (D + 1)
    probs, refs = [], []
    for i, (N, K) in enumerate([(1500, 512), (700, 1280)]):
        W, x = S.random_case(900 + i, M, N, K)
        q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        probs.append((to_dev_bf16(x), q, sf, ts, Y))
        refs.append((W, x))
    N, K = 20000, 1024
    W, x = S.random_case(950, M, N, K, w_std=0.05)
    y_ref = oracle_logits(W, x)
    parents = S.random_tree(B, D, seed=51)
    drafts = S.tree_drafts(V.argmax_fast(y_ref), parents, D, N, agree=0.8, seed=52)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    probs.append((to_dev_bf16(x), q, sf, ts, None))
    t = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    L = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    node = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    vmax = torch.empty(M, dtype=torch.float32, device="cuda")
    p = nv.WeightPass(probs, M, verify=(torch.from_numpy(drafts).cuda(), t, L, vmax,
                                        torch.from_numpy(parents).cuda(), node))
    p.run()
    nv.check()
    for (_, _, _, _, Y), (Wi, xi) in zip(probs[:2], refs):
        y = Y.cpu().numpy().astype(np.float64)
        yr = oracle_logits(Wi, xi)
        assert (np.abs(y - yr).max(axis=1) <= 2e-3 * np.abs(yr).max(axis=1)).all()
    check_tree(t.cpu().numpy(), L.cpu().numpy(), node.cpu().numpy(), y_ref, drafts, parents, D)


def test_verify_tree_bad_parent_is_reported(nv):
    """A parent outside [0, k-1] rejects that node, leaves the other sequence exact, and
    the next check reports an invalid argument."""
    B, D, N, K = 2, 6, 2000, 256
    W, x = S.random_case(960, B * (D + 1), N, K, w_std=0.05)
    y_ref = oracle_logits(W, x)
    parents = S.random_tree(B, D, seed=61)
    drafts = S.tree_drafts(V.argmax_fast(y_ref), parents, D, N, agree=1.0, seed=62)
    bad = parents.copy()
    bad[0, 2] = 5                                   # node 3 may only hang under nodes 0..2
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    t, L, node, _ = nv.verify_tree(to_dev_bf16(x), q, sf, ts, torch.from_numpy(drafts).cuda(),
                                   torch.from_numpy(bad).cuda())
    with pytest.raises(nv.NVFP4WSError):
        nv.check()
    nv.check()                                      # the error word was cleared
    L_ref, node_ref = V.accept_tree_ref(V.argmax_fast(y_ref), drafts, parents, D)
    gap = V.top2_gap(y_ref)
    if V.comparable_tree_sequences(gap, parents, D)[1]:
        assert L.cpu().numpy()[1] == L_ref[1] and node.cpu().numpy()[1] == node_ref[1]
