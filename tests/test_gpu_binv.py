"""GPU: batch-invariant weight passes (NVFP4WS_PASS_BATCH_INVARIANT).

"TandemLLM", "The parts": the projection kernels give a row the same bits whatever
other rows share the batch; its feature list names a batch-invariance probe. Here the
same problem list runs at M = 1, 8, 17, 34 and 68 with the same leading activation
rows, and every row must come out bit-identical: GEMM outputs, the verify's argmax and
its winning logit. The M=17 run is also checked against the oracle.
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu
M_LIST = [1, 8, 17, 34, 68]


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def test_pass_rows_identical_for_every_m(nv):
    # 28 GEMMs of K = 5120 hold more activation images than one wave's budget at M = 70,
    # so the list is cut into waves; a mixed tail adds ragged N and other K.
    shapes = [(640, 5120)] * 28 + [(3000, 1024), (1000, 2560), (77, 512)]
    Mmax = max(M_LIST)
    weights, xs = [], []
    for i, (N, K) in enumerate(shapes):
        W, x = S.random_case(1300 + i, Mmax, N, K)
        weights.append((W, nv.pack(torch.from_numpy(W).cuda())))
        xs.append(x)
    Wl, xl = S.random_case(1399, Mmax, 20000, 1024, w_std=0.05)
    ql = nv.pack(torch.from_numpy(Wl).cuda())
    out = {}
    for M in M_LIST:
        probs = []
        for (W, (q, sf, ts)), x in zip(weights, xs):
            Y = torch.full((M, W.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
            probs.append((to_dev_bf16(x[:M]), q, sf, ts, Y))
        probs.append((to_dev_bf16(xl[:M]), *ql, None))
        t = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        L = torch.empty(1, dtype=torch.int32, device="cuda")
        vmax = torch.empty(M, dtype=torch.float32, device="cuda")
        drafts = torch.zeros((1, M - 1), dtype=torch.int32, device="cuda")
        p = nv.WeightPass(probs, M, verify=(drafts, t, L, vmax), batch_invariant=True)
        p.run()
        nv.check()
        out[M] = ([pr[4].cpu().numpy() for pr in probs[:-1]], t.cpu().numpy(), vmax.cpu().numpy())
    Ys, tm, vm = out[Mmax]
    for M in M_LIST[:-1]:
        ys, t, v = out[M]
        for i, (a, b) in enumerate(zip(ys, Ys)):
            assert np.array_equal(a.view(np.uint32), b[:M].view(np.uint32)), f"problem {i}: M={M} rows differ"
        assert np.array_equal(t, tm[:M]) and np.array_equal(v.view(np.uint32), vm[:M].view(np.uint32))
    # and the rows are the right numbers (M = 17 against the oracle)
    ys, _, _ = out[17]
    for i in (0, 27, 28, 29, 30):
        W, x = weights[i][0], xs[i][:17]
        q, sf, ts = F.quantize_nvfp4(W)
        y_ref = G.gemm_ref(x, q, sf, ts)
        err, scale = np.abs(ys[i] - y_ref).max(axis=1), np.abs(y_ref).max(axis=1)
        assert (err <= 2e-3 * scale).all()
        assert (err <= 1e-4 * scale).all()              # the five residual activation terms
