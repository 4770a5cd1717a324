"""Full-size parity on the configurations the bench times.

* The lm_head verify over the whole 248,320-row vocabulary at M = 1, 17 and 68 (one, one
  and four sequences of 16 drafts + 1), as a single call and as the verify tail of a
  weight pass. The argmax is compared with the oracle's argmax over EVERY row, not a
  sample. A dropped tile or a lost partial would change a winner and fail here. Accept
  lengths are compared exactly too. The drafts copy the oracle's argmax for a prefix of
  L* ~ U{0..16} slots, so accept lengths above zero are exercised.
* Weight passes at the same M over the three 27B layer shapes (gate+up 5120->34816, down
  17408->5120, qkv 5120->10240) with that head as the verify problem. The GEMM outputs
  are compared at 256 sampled rows of each matrix, element by element.

Bars: argmax and accept length bit-exact except near ties (oracle top-2 gap < 1e-3; the
pick there must still be within the band). GEMM rows within 2e-3 of max|y_ref| (the
task's bar), and within 1e-4 on the block-scaled path, whose five residual activation
terms are claimed to reach ~1e-5.

The oracle side (full_vocab_oracle) quantises and multiplies every row of the head in
float64 on a spawn pool. The GPU is given the oracle's packed bytes of the head, so this
compares the GEMM and verify alone; packing is bit-exact in test_gpu_parity's
test_pack_* at all three layer shapes.
"""

import numpy as np
import pytest
import torch

import full_vocab_oracle as FV
import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F
from oracle import verify as V

pytestmark = pytest.mark.gpu
REL_TOL = 2e-3
TERMS_TOL = 1e-4
D = S.DRAFT_LEN
CASES = [(1, 1, 0), (17, 1, D), (68, 4, D)]          # (M, B, D)


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def head(nv):
    """The 68 hidden rows (the first 17 are the one-sequence case, row 0 the M = 1 case),
    the oracle's argmax and logits over the whole head, and its packed bytes on the GPU."""
    x = S.lmhead_x(B=4)
    orc = FV.lmhead_oracle(x)
    dev = (torch.from_numpy(orc["q"]).cuda(), torch.from_numpy(orc["sf"]).cuda(),
           torch.tensor([float(orc["ts"])], dtype=torch.float32, device="cuda"))
    return x, orc, dev


def drafts_for(orc, M, B, Dd):
    """Drafts that copy the oracle's argmax for L* slots, then differ (S.drafts_with_prefix)."""
    if Dd == 0:
        return np.zeros((B, 0), np.int32), np.zeros(B, np.int64)
    Lstar = S.lmhead_lstar(B, Dd)
    d = S.drafts_with_prefix(orc["t"][:M], Lstar, Dd, S.VOCAB)
    assert np.array_equal(V.accept_ref(orc["t"][:M], d, Dd), Lstar)
    return d, Lstar


def check_verify(orc, x, M, Dd, drafts, t, L, vmax):
    t_ref, gap = orc["t"][:M], orc["gap"][:M]
    L_ref = V.accept_ref(t_ref, drafts, Dd)
    rows = V.comparable_rows(gap)
    seqs = V.comparable_sequences(gap, L_ref, Dd)
    bad = np.flatnonzero(t[rows] != t_ref[rows])
    assert bad.size == 0, f"argmax differs from the oracle's on rows {np.flatnonzero(rows)[bad]}"
    assert np.array_equal(L[seqs], L_ref[seqs])
    assert np.array_equal(L, V.accept_ref(t, drafts, Dd))        # stage 2 follows the GPU's own argmax
    for m in range(M):                                           # near ties: the pick stays in the band
        y_t = FV.logit(orc, x, m, int(t[m]))
        assert orc["top1"][m] - y_t <= V.NEAR_TIE
        assert abs(float(vmax[m]) - y_t) <= TERMS_TOL * max(1.0, abs(y_t))
    return rows.mean()


@pytest.mark.parametrize("M,B,Dd", CASES)
def test_verify_full_vocab_exact(nv, head, M, B, Dd):
    """lmhead_verify_argmax_accept on the whole head (the default path: block-scaled)."""
    x, orc, (q, sf, ts) = head
    drafts, _ = drafts_for(orc, M, B, Dd)
    t, L, vmax = nv.verify(to_dev_bf16(x[:M]), q, sf, ts, torch.from_numpy(drafts).cuda())
    nv.check()
    frac = check_verify(orc, x, M, Dd, drafts, t.cpu().numpy(), L.cpu().numpy(), vmax.cpu().numpy())
    assert frac > 0.9


@pytest.mark.parametrize("path,M,B,Dd", [("mma_f16", 17, 1, D), ("gemv", 17, 1, D), ("gemv", 1, 1, 0)])
def test_verify_full_vocab_other_paths(nv, head, path, M, B, Dd):
    """The same head on the f16 tensor-core kernel and on the CUDA-core GEMV."""
    x, orc, (q, sf, ts) = head
    drafts, _ = drafts_for(orc, M, B, Dd)
    t, L, vmax = nv.verify(to_dev_bf16(x[:M]), q, sf, ts, torch.from_numpy(drafts).cuda(), path=path)
    nv.check()
    check_verify(orc, x, M, Dd, drafts, t.cpu().numpy(), L.cpu().numpy(), vmax.cpu().numpy())


@pytest.fixture(scope="module")
def layers(nv):
    """Each 27B layer shape: its packed weight on the GPU, 68 activation rows, and the
    oracle's outputs at 256 sampled weight rows for all 68 tokens."""
    out = []
    rng = np.random.default_rng(2024)
    for name in S.LAYER_ORDER:
        W, x = S.layer(name, M=68)
        q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
        rows = np.sort(rng.choice(W.shape[0], 256, replace=False))
        ts_ref = F.tensor_scale(W)
        q_r, sf_r, _ = F.quantize_nvfp4(W[rows], ts_ref)
        y_s = G.gemm_ref(x, q_r, sf_r, ts_ref)
        out.append((name, W.shape[0], x, (q, sf, ts), rows, y_s))
        del W
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("M,B,Dd", CASES)
def test_pass_full_size(nv, head, layers, M, B, Dd):
    """One weight pass of the three layer GEMMs with the whole head as its verify tail, at
    the M the bench times."""
    x, orc, (ql, sfl, tsl) = head
    drafts, _ = drafts_for(orc, M, B, Dd)
    probs = []
    for name, N, xl, (q, sf, ts), _, _ in layers:
        probs.append((to_dev_bf16(xl[:M]), q, sf, ts, torch.full((M, N), float("nan"), device="cuda")))
    probs.append((to_dev_bf16(x[:M]), ql, sfl, tsl, None))
    t = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    L = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    vmax = torch.empty(M, dtype=torch.float32, device="cuda")
    p = nv.WeightPass(probs, M, verify=(torch.from_numpy(drafts).cuda(), t, L, vmax))
    p.run()
    torch.cuda.synchronize()
    nv.check()
    for (name, N, xl, _, rows, y_s), pr in zip(layers, probs):
        y = pr[4].cpu().numpy()
        assert np.isfinite(y).all(), name
        err = np.abs(y[:, rows].astype(np.float64) - y_s[:M]).max(axis=1)
        scale = np.abs(y_s[:M]).max(axis=1)
        assert (err <= REL_TOL * scale).all(), name
        assert (err <= TERMS_TOL * scale).all(), f"{name}: {np.max(err / scale):.2e} of max|y|"
    check_verify(orc, x, M, Dd, drafts, t.cpu().numpy(), L.cpu().numpy(), vmax.cpu().numpy())
