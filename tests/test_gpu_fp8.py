"""GPU parity of the FP8 (E4M3, 128 x 128 block-scaled) weight path against the oracle
on the same seeded inputs.

Bars:
* fp8_pack: codes and scales bit-exact (both sides form the quotient in float64 and
  round once, ties to even).
* fp8_gemm_skinny: per row max |y - y_ref| <= 1e-5 * max |y_ref|. Each product
  x * e4m3 is exact in fp32 (both exact in f16); what remains is the fp32 sum inside a
  block, one rounding for the scale product and the fp32 sum over blocks. bf16 Y is the
  fp32 result rounded once.
* fp8_lmhead_verify: argmax bit-exact on rows whose oracle top-2 gap is >= 1e-3; accept
  length (and end node for a tree) bit-exact on sequences with no near-tie row that can
  decide them.
The weights vary by up to 2^16 between blocks, so a scale applied to the wrong block
misses the bar by orders of magnitude.
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import fp8 as P
from oracle import gemm as G
from oracle import verify as V

pytestmark = pytest.mark.gpu
TOL = 1e-5
# The E4M3-term path: the activation terms are exact for these inputs up to E4M3's subnormal
# step (2^-14 g per element); the bar leaves room for the FP8 tensor core's accumulation inside
# a 128-wide block, whose precision is what this test measures.
TOL_TERMS = 2e-4
TOLS = {"f16": TOL, "terms": TOL_TERMS}


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def rowwise_err(y, y_ref):
    return (np.abs(y.astype(np.float64) - y_ref).max(axis=1) / np.abs(y_ref).max(axis=1)).max()


def packed(nv, W):
    """Packs on the GPU and checks the bytes against the oracle; returns device and oracle copies."""
    q, s = nv.fp8_pack(torch.from_numpy(W).cuda())
    codes_ref, scales_ref = P.quantize_fp8_blocks(W)
    assert np.array_equal(q.cpu().numpy(), codes_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), scales_ref.view(np.uint32))
    return q, s, codes_ref, scales_ref


@pytest.mark.parametrize("N,K", [(1000, 256), (130, 80), (3, 16), (257, 400)])
def test_fp8_pack_bit_exact(nv, N, K):
    W, _ = S.block_varied_case(900 + N, 1, N, K)
    if N >= 128 and K >= 128:
        W[:128, :128] = 0.0                                   # an all-zero block: s = 0, codes +0
    W[-1, :8] = [448.0, -224.0, 8.5, -0.0, 216.0, 1e-30, -1e-30, 0.0]   # saturating, tie, signed-zero cases
    packed(nv, W)


@pytest.mark.parametrize("path", ["f16", "terms"])
@pytest.mark.parametrize("M,N,K", [(1, 1000, 256), (17, 3000, 1024), (68, 777, 768), (128, 4096, 5120),
                                   (5, 130, 128), (17, 640, 5120), (17, 128, 16384), (40, 1000, 1024),
                                   (49, 333, 512)])
def test_fp8_gemm(nv, M, N, K, path):
    W, x = S.block_varied_case(1000 + M + N, M, N, K)
    q, s, codes_ref, scales_ref = packed(nv, W)
    Y = nv.fp8_gemm(to_dev_bf16(x), q, s, path=path)
    nv.check()
    y_ref = P.gemm_fp8_ref(x, codes_ref, scales_ref)
    assert rowwise_err(Y.cpu().numpy(), y_ref) <= TOLS[path]


@pytest.mark.parametrize("M,N,K", [(5, 700, 1024), (68, 300, 512)])
def test_fp8_gemm_activation_range(nv, M, N, K):
    """Activation rows far above f16's range (|x| up to ~4e6), of ~1e-30 values, and of
    zeros: each row is shifted by a power of two before the f16 conversion, so every row
    meets the bar and the zero row gives exact zeros."""
    W, x = S.block_varied_case(3000 + M, M, N, K)
    xf = (np.asarray(x, np.uint32) << 16).view(np.float32).astype(np.float64)
    for m in range(M):
        xf[m] *= (2.0 ** 20, 1e-30, 1.0, 0.0)[m % 4]
    x = S.f32_to_bf16_bits(xf.astype(np.float32))
    q, s, codes_ref, scales_ref = packed(nv, W)
    Y = nv.fp8_gemm(to_dev_bf16(x), q, s)
    nv.check()
    y_ref = P.gemm_fp8_ref(x, codes_ref, scales_ref)
    y = Y.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    err = np.abs(y - y_ref).max(axis=1)
    assert (err <= TOL * np.abs(y_ref).max(axis=1)).all()


def test_fp8_gemm_bf16_and_repeat(nv):
    M, N, K = 17, 2500, 2048
    W, x = S.block_varied_case(1100, M, N, K)
    q, s, _, _ = packed(nv, W)
    X = to_dev_bf16(x)
    Y1 = nv.fp8_gemm(X, q, s)
    Y2 = nv.fp8_gemm(X, q, s)
    Yb = nv.fp8_gemm(X, q, s, y_dtype=torch.bfloat16)
    nv.check()
    assert torch.equal(Y1, Y2)                                # fixed sum order: deterministic
    assert torch.equal(Yb, Y1.to(torch.bfloat16))


@pytest.mark.parametrize("path", ["f16", "terms"])
def test_fp8_verify_chain(nv, path):
    B, D, N, K = 1, 16, 20077, 2048
    W, x = S.random_case(1200, B * (D + 1), N, K, w_std=0.2)
    q, s, codes_ref, scales_ref = packed(nv, W)
    y_ref = P.gemm_fp8_ref(x, codes_ref, scales_ref)
    t_ref = V.argmax_fast(y_ref)
    Lstar = np.array([9])
    drafts = S.drafts_with_prefix(t_ref, Lstar, D, N)
    t, L, _, vmax = nv.fp8_verify(to_dev_bf16(x), q, s, torch.from_numpy(drafts).cuda(), path=path)
    nv.check()
    t, L = t.cpu().numpy(), L.cpu().numpy()
    gap = V.top2_gap(y_ref)
    rows = V.comparable_rows(gap)
    assert rows.all()                                          # no near tie for this seed (oracle-checked)
    assert np.array_equal(t, t_ref)
    assert L.tolist() == V.accept_ref(t_ref, drafts, D).tolist() == [9]
    np.testing.assert_allclose(vmax.cpu().numpy(), y_ref.max(axis=1), rtol=TOLS[path], atol=0)


def test_fp8_verify_tree(nv):
    B, D, N, K = 4, 16, 9000, 1024
    W, x = S.random_case(1300, B * (D + 1), N, K, w_std=0.2)
    q, s, codes_ref, scales_ref = packed(nv, W)
    y_ref = P.gemm_fp8_ref(x, codes_ref, scales_ref)
    t_ref = V.argmax_fast(y_ref)
    parents = S.random_tree(B, D, seed=31, chain_bias=0.5)
    drafts = S.tree_drafts(t_ref, parents, D, N, agree=0.75, seed=32)
    t, L, node, _ = nv.fp8_verify(to_dev_bf16(x), q, s, torch.from_numpy(drafts).cuda(),
                                  torch.from_numpy(parents).cuda())
    nv.check()
    L_ref, node_ref = V.accept_tree_ref(t_ref, drafts, parents, D)
    gap = V.top2_gap(y_ref)
    assert V.comparable_tree_sequences(gap, parents, D).all()  # no near tie for this seed (oracle-checked)
    assert np.array_equal(t.cpu().numpy(), t_ref)
    assert np.array_equal(L.cpu().numpy(), L_ref) and np.array_equal(node.cpu().numpy(), node_ref)


@pytest.mark.parametrize("M,shapes", [
    (17, [(3000, 1024), (640, 5120), (1500, 2560), (77, 512)]),    # every K a multiple of 256: two blocks per unit
    (17, [(700, 384), (300, 1280), (129, 128)]),                   # odd block counts: one block per unit
    (68, [(1000, 1024), (200, 2048), (64, 256)]),                  # npad 80: one block per unit
])
@pytest.mark.parametrize("path", ["f16", "terms"])
def test_fp8_pass(nv, M, shapes, path):
    probs, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W, x = S.block_varied_case(1400 + 10 * M + i, M, N, K)
        q, s, codes_ref, scales_ref = packed(nv, W)
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        probs.append((to_dev_bf16(x), q, s, Y))
        refs.append(P.gemm_fp8_ref(x, codes_ref, scales_ref))
    p = nv.Fp8Pass(probs, M, path=path)
    p.run()
    nv.check()
    first = [Y.clone() for (_, _, _, Y) in probs]
    for (_, _, _, Y), y_ref in zip(probs, refs):
        assert rowwise_err(Y.cpu().numpy(), y_ref) <= TOLS[path]
    p.run()                                                     # tickets were reset: the same bits again
    nv.check()
    for (_, _, _, Y), Y1 in zip(probs, first):
        assert torch.equal(Y, Y1)


@pytest.mark.parametrize("path", ["f16", "terms"])
def test_fp8_pass_with_verify_tail(nv, path):
    """Two FP8 GEMMs and the FP8 head of the chain-verify test in one launch, ending in the verify."""
    B, D, N, K = 1, 16, 20077, 2048
    M = B * (D + 1)
    Wh, xh = S.random_case(1200, M, N, K, w_std=0.2)
    qh, sh, ch_ref, sch_ref = packed(nv, Wh)
    t_ref = V.argmax_fast(P.gemm_fp8_ref(xh, ch_ref, sch_ref))
    drafts = S.drafts_with_prefix(t_ref, np.array([9]), D, N)
    probs, refs = [], []
    for i, (Ng, Kg) in enumerate([(900, 1024), (333, 2048)]):
        W, x = S.block_varied_case(1500 + i, M, Ng, Kg)
        q, s, codes_ref, scales_ref = packed(nv, W)
        Y = torch.empty((M, Ng), dtype=torch.float32, device="cuda")
        probs.append((to_dev_bf16(x), q, s, Y))
        refs.append(P.gemm_fp8_ref(x, codes_ref, scales_ref))
    probs.append((to_dev_bf16(xh), qh, sh, None))
    t = torch.empty(M, dtype=torch.int32, device="cuda")
    L = torch.empty(B, dtype=torch.int32, device="cuda")
    p = nv.Fp8Pass(probs, M, verify=(torch.from_numpy(drafts).cuda(), t, L, None), path=path)
    p.run()
    nv.check()
    for (_, _, _, Y), y_ref in zip(probs[:2], refs):
        assert rowwise_err(Y.cpu().numpy(), y_ref) <= TOLS[path]
    assert np.array_equal(t.cpu().numpy(), t_ref)              # no near tie for this seed (the chain test checks it)
    assert L.cpu().numpy().tolist() == [9]


def test_fp8_terms_path_extreme_rows(nv):
    """Rows with 100x outliers and rows of tiny values: the row's power-of-two scale follows the
    row maximum, so the second term still carries each element's low bits."""
    M, N, K = 17, 1000, 2048
    W, x = S.block_varied_case(1600, M, N, K)
    xf = G.bf16_bits_to_float64(x).copy()
    rng = np.random.default_rng(1601)
    xf[0, rng.integers(0, K, 20)] *= 100.0                      # outliers
    xf[1] *= 2.0 ** -30                                          # a row of tiny values
    xf[2] = 0.0                                                  # an all-zero row
    x = S.f32_to_bf16_bits(xf.astype(np.float32))
    q, s, codes_ref, scales_ref = packed(nv, W)
    Y = nv.fp8_gemm(to_dev_bf16(x), q, s, path="terms").cpu().numpy()
    nv.check()
    y_ref = P.gemm_fp8_ref(x, codes_ref, scales_ref)
    assert (Y[2] == 0).all()
    rows = [m for m in range(M) if m != 2]
    assert rowwise_err(Y[rows], y_ref[rows]) <= TOL_TERMS


@pytest.mark.parametrize("path", ["f16", "terms"])
def test_fp8_accumulation_keeps_small_products(nv, path):
    """One 128-wide block whose sum needs ~19 significant bits: 448 * 1 plus 127 products of
    2^-10. fp32 accumulation keeps every small product; an accumulator of ~14 bits would drop
    them (an error of ~3e-4 of the result). This measures the tensor core's accumulation width."""
    M, N, K = 1, 128, 128
    W = np.ones((N, K), dtype=np.float32)
    W[:, 0] = 448.0                                            # block scale exactly 1, codes 448 and 1
    x = np.full((M, K), 2.0 ** -10, dtype=np.float32)
    x[0, 0] = 1.0
    xb = S.f32_to_bf16_bits(x)
    q, s, codes_ref, scales_ref = packed(nv, W)
    assert float(scales_ref[0, 0]) == 1.0
    Y = nv.fp8_gemm(to_dev_bf16(xb), q, s, path=path).cpu().numpy()
    nv.check()
    y_ref = 448.0 + 127 * 2.0 ** -10
    assert np.abs(Y.astype(np.float64) - y_ref).max() <= 1e-6 * y_ref
