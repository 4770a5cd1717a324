"""GPU: degenerate activation rows and extreme sizes through a weight pass, against the
oracle. A zero row must give exact zeros; a row whose magnitude is set by one outlier,
rows of tiny magnitude and the largest K must stay within the GEMM bar."""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu
REL_TOL = 2e-3


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return (torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def run_pass(nv, W_list, x_list, M):
    probs = []
    for W, x in zip(W_list, x_list):
        q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
        probs.append((to_dev_bf16(x), q, sf, ts, torch.full((M, W.shape[0]), float("nan"), device="cuda")))
    nv.WeightPass(probs, M).run()
    nv.check()
    return [p[4].cpu().numpy().astype(np.float64) for p in probs]


def test_degenerate_rows(nv):
    M, N, K = 17, 1500, 2048
    rng = np.random.default_rng(71)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0] = 0.0                                    # a zero row
    x[1] = rng.standard_normal(K) * 1e-3          # small values ...
    x[1, 100] = 3.0e4                             # ... under one outlier
    x[2] = rng.standard_normal(K) * 1e-30         # a row of tiny magnitude
    x[3, :] = 0.0
    x[3, 7] = -2.5                                # a single non-zero element
    xb = bf16_bits(x)
    (Y,) = run_pass(nv, [W], [xb], M)
    q, sf, ts = F.quantize_nvfp4(W)
    y_ref = G.gemm_ref(xb, q, sf, ts)
    assert np.isfinite(Y).all()
    assert (Y[0] == 0).all()
    for m in range(1, M):
        assert np.abs(Y[m] - y_ref[m]).max() <= REL_TOL * np.abs(y_ref[m]).max(), f"row {m}"


def test_largest_k_and_single_column(nv):
    M = 17
    W1, x1 = S.random_case(72, M, 300, 32768)
    W2, x2 = S.random_case(73, M, 1, 1024)
    Y1, Y2 = run_pass(nv, [W1, W2], [x1, x2], M)
    for Y, W, x in ((Y1, W1, x1), (Y2, W2, x2)):
        q, sf, ts = F.quantize_nvfp4(W)
        y_ref = G.gemm_ref(x, q, sf, ts)
        assert (np.abs(Y - y_ref).max(axis=1) <= REL_TOL * np.abs(y_ref).max(axis=1)).all()
