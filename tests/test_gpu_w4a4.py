"""GPU parity of the W4A4 path (nvfp4_gemm_w4a4 and W4A4 weight passes) against the
oracle's W4A4 product on the same seeded inputs.

The activation codes and scales are decided in fp32 with correctly rounded operations
on both sides, so they are identical; what remains is the order of the fp32 sums in the
tensor core against the oracle's float64 sum. Bar: per row
max |y - y_ref| <= 2e-5 * max |y_ref| (fp32 accumulation over K/64 block products);
bf16 Y is the fp32 result rounded once. The exact bf16 product is not the reference here:
the W4A4 result differs from it by the activation quantisation (checked to be well
outside the bar, so the test would see a kernel that skipped it).
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu
TOL = 2e-5


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


@pytest.mark.parametrize("M,N,K", [(1, 1000, 256), (17, 3000, 1024), (68, 777, 768), (128, 4096, 5120),
                                   (200, 130, 512), (256, 2000, 2048)])
def test_gemm_w4a4(nv, M, N, K):
    W, x = S.random_case(4000 + M, M, N, K)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    Y = nv.gemm_w4a4(to_dev_bf16(x), q, sf, ts)
    nv.check()
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
    y_ref = G.gemm_w4a4_ref(x, q_ref, sf_ref, ts_ref)
    y = Y.cpu().numpy()
    assert rowwise_err(y, y_ref) <= TOL
    # the exact bf16 product is a different number: the activations were quantised
    assert rowwise_err(y, G.gemm_ref(x, q_ref, sf_ref, ts_ref)) > 10 * TOL


def test_gemm_w4a4_bf16_output_and_repeat(nv):
    M, N, K = 128, 2500, 1024
    W, x = S.random_case(4100, M, N, K)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    X = to_dev_bf16(x)
    Y1 = nv.gemm_w4a4(X, q, sf, ts)
    Y2 = nv.gemm_w4a4(X, q, sf, ts)
    Yb = nv.gemm_w4a4(X, q, sf, ts, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    assert torch.equal(Yb, Y1.to(torch.bfloat16))


def test_w4a4_pass(nv):
    """A W4A4 pass over mixed shapes at M = 128 (prefill-sized), one launch."""
    M = 128
    shapes = [(3000, 1024), (640, 5120), (1500, 2560), (77, 512)]
    probs, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W, x = S.random_case(4200 + i, M, N, K)
        q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        probs.append((to_dev_bf16(x), q, sf, ts, Y))
        refs.append((W, x))
    p = nv.WeightPass(probs, M, w4a4=True)
    p.run()
    nv.check()
    for (_, _, _, _, Y), (W, x) in zip(probs, refs):
        q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
        assert rowwise_err(Y.cpu().numpy(), G.gemm_w4a4_ref(x, q_ref, sf_ref, ts_ref)) <= TOL


def test_w4a4_pass_refuses_a_verify(nv):
    M, N, K = 17, 1000, 512
    W, x = S.random_case(4300, M, N, K)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    t = torch.empty(M, dtype=torch.int32, device="cuda")
    L = torch.empty(1, dtype=torch.int32, device="cuda")
    drafts = torch.zeros((1, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(nv.NVFP4WSError):
        nv.WeightPass([(to_dev_bf16(x), q, sf, ts, None)], M, verify=(drafts, t, L, None), w4a4=True)
