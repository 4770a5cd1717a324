"""The allocation-free GEMM entry point, for callers that cannot allocate device
memory: a host with a fixed device-memory plan, code under another framework's
pooling allocator, or a plugin interface with no scratch buffer.

nvfp4_gemm_skinny_noalloc takes its scratch from a built-in device array instead
of a caller workspace. This test calls it through the C ABI twice in a row. Both
results must match nvfp4_gemm_skinny (which gets a workspace) within the
tolerance used by the other GEMM tests, and must also match the CPU oracle. Around
the second call neither torch's allocator nor the device's free memory may change.
One row of X lies far above f16's range (the f16 path shifts it into range). It
sits in a file of its own, collected last, so that a run which stops at the first
failure has already run every other test. It passes alone in a fresh process too.
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu
REL_TOL = 2e-3


def rowwise_ok(y, y_ref, rel=REL_TOL):
    err = np.abs(np.asarray(y, np.float64) - y_ref).max(axis=1)
    return bool((err <= rel * np.abs(y_ref).max(axis=1)).all())


@pytest.mark.parametrize("M,N,K", [(17, 3000, 5120), (68, 1000, 17408), (1, 520, 256)])
def test_noalloc_matches_workspace_entry_point(M, N, K):
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    lib = nv.lib()
    W, x = S.random_case(900 + M + N, M, N, K)
    if M > 1:                                            # one row far above f16's range (|x| up to ~4e6)
        xf = G.bf16_bits_to_float64(x)
        xf[M // 2] *= 2.0 ** 20
        x = S.f32_to_bf16_bits(xf.astype(np.float32))
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    X = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
    stream = torch.cuda.current_stream().cuda_stream

    ws_bytes = lib.nvfp4_gemm_workspace_bytes(M, N, K)
    ws = torch.zeros(max(16, ws_bytes), dtype=torch.uint8, device="cuda")
    y_ws = torch.empty((M, N), dtype=torch.float32, device="cuda")
    st = lib.nvfp4_gemm_skinny(X.data_ptr(), q.data_ptr(), sf.data_ptr(), ts.data_ptr(), M, N, K,
                               y_ws.data_ptr(), 0, ws.data_ptr(), ws_bytes, stream)
    assert st == 0, lib.nvfp4ws_last_error()

    outs = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    for i, y in enumerate(outs):                         # two calls in a row share the built-in scratch
        if i == 1:                                       # the first call has looked up the scratch address
            torch.cuda.synchronize()
            alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        st = lib.nvfp4_gemm_skinny_noalloc(X.data_ptr(), q.data_ptr(), sf.data_ptr(), ts.data_ptr(), M, N, K,
                                           y.data_ptr(), 0, stream)
        assert st == 0, lib.nvfp4ws_last_error()
        assert lib.nvfp4ws_last_error() == b""
    torch.cuda.synchronize()
    # the call allocated nothing: neither through torch nor from the device
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    nv.check()

    ref_ws = y_ws.cpu().numpy().astype(np.float64)
    q_r, sf_r, ts_r = F.quantize_nvfp4(W)
    y_oracle = G.gemm_ref(x, q_r, sf_r, ts_r)
    assert rowwise_ok(ref_ws, y_oracle)
    for y in outs:
        yn = y.cpu().numpy()
        assert np.isfinite(yn).all()
        assert rowwise_ok(yn, ref_ws)
        assert rowwise_ok(yn, y_oracle)


def test_noalloc_rejects_oversized_and_unsupported():
    import nvfp4_weight_streaming_gemm_b200 as nv
    lib = nv.lib()
    dummy = torch.zeros(64, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    # K not a multiple of 256: outside the tensor-core path
    assert lib.nvfp4_gemm_skinny_noalloc(p, p, p, p, 4, 100, 96, p, 0, stream) == 2
    # M above the tensor-core limit
    assert lib.nvfp4_gemm_skinny_noalloc(p, p, p, p, 200, 100, 256, p, 0, stream) == 2
    # scratch larger than the built-in array (checked before any launch)
    big_n = 1 << 28
    assert lib.nvfp4_gemm_workspace_bytes(128, big_n, 256) > (16 << 20)
    assert lib.nvfp4_gemm_skinny_noalloc(p, p, p, p, 128, big_n, 256, p, 0, stream) == 2
    assert b"scratch" in lib.nvfp4ws_last_error()
