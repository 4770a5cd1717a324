"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle, on the
same seeded inputs.

Bars:
- packing (q, sf, ts) bit-exact;
- GEMM: per row m, max_n |y - y_ref| <= 2e-3 * max_n |y_ref| (fp32 Y), plus a
  bf16-Y check within one bf16 rounding;
- verify: argmax bit-exact on rows whose oracle top-2 gap is >= 1e-3, and
  accept lengths bit-exact on sequences without a near tie at or before their
  oracle accept length.
"""

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import gemm as G
from oracle import nvfp4 as F
from oracle import verify as V

pytestmark = pytest.mark.gpu
REL_TOL = 2e-3
TERMS_TOL = 1e-4          # the block-scaled path's five residual activation terms (~1e-5 measured)


@pytest.fixture(scope="module")
def nv():
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build
    build.build()
    return nv


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def pack_both(nv, W, tensor_scale_in=None):
    Wd = torch.from_numpy(W).cuda()
    tin = None if tensor_scale_in is None else torch.tensor([tensor_scale_in], dtype=torch.float32, device="cuda")
    q, sf, ts = nv.pack(Wd, tin)
    torch.cuda.synchronize()
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W, tensor_scale_in)
    return (q, sf, ts), (q_ref, sf_ref, ts_ref)


def assert_pack_equal(dev, ref):
    q, sf, ts = dev
    q_ref, sf_ref, ts_ref = ref
    assert ts.item() == float(ts_ref)
    assert np.array_equal(sf.cpu().numpy(), sf_ref)
    qn = q.cpu().numpy()
    if not np.array_equal(qn, q_ref):
        bad = np.argwhere(qn != q_ref)
        raise AssertionError(f"{len(bad)} q bytes differ, first at {bad[0]}: got {qn[tuple(bad[0])]:#x} "
                             f"want {q_ref[tuple(bad[0])]:#x}")


def assert_rowwise(y: np.ndarray, y_ref: np.ndarray, rel=REL_TOL):
    err = np.abs(y.astype(np.float64) - y_ref).max(axis=1)
    scale = np.abs(y_ref).max(axis=1)
    worst = (err / np.maximum(scale, 1e-300)).max()
    assert (err <= rel * scale).all(), f"rowwise error {worst:.3e} > {rel}"
    return worst


# ------------------------------------------------------------------ pack

def test_pack_tiny_bit_exact(nv):
    W, _ = S.tiny()
    dev, ref = pack_both(nv, W)
    assert_pack_equal(dev, ref)


@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (1001, 32), (257, 160)])
def test_pack_ragged_bit_exact(nv, N, K):
    W, _ = S.random_case(N * 7 + K, 1, N, K)
    dev, ref = pack_both(nv, W)
    assert_pack_equal(dev, ref)


def test_pack_given_tensor_scale_and_degenerate_blocks(nv):
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    W[3, 16:32] = -1e-30                     # S rounds to 0 -> +0 codes
    W[4, :16] = 0.0                          # all-zero block
    W[5, 0] = -0.0
    W[6, :] = rng.standard_normal(128).astype(np.float32) * 50.0   # saturating block scales
    for tin in (None, 0.001, 2.0 ** -7):
        dev, ref = pack_both(nv, W, tin)
        assert_pack_equal(dev, ref)


def test_pack_all_zero(nv):
    dev, ref = pack_both(nv, np.zeros((8, 64), np.float32))
    assert_pack_equal(dev, ref)


def test_pack_hand_worked_blocks(nv):
    import json, os
    with open(os.path.join(os.path.dirname(__file__), "golden", "hand_blocks.json")) as f:
        g = json.load(f)
    W = np.array(g["W"], dtype=np.float32)
    for case in g["cases"]:
        dev, _ = pack_both(nv, W, case["tensor_scale_in"])
        assert dev[0].cpu().numpy().tolist() == case["q"]
        assert dev[1].cpu().numpy().tolist() == case["sf"]
        assert dev[2].item() == case["ts"]


@pytest.mark.parametrize("name", S.LAYER_ORDER)
def test_pack_layer_shapes_bit_exact(nv, name):
    W, _ = S.layer(name)
    dev, ref = pack_both(nv, W)
    assert_pack_equal(dev, ref)


# ------------------------------------------------------------------ GEMM

def run_gemm(nv, W, x_bits, path="auto", y_dtype=torch.float32):
    Wd = torch.from_numpy(W).cuda()
    q, sf, ts = nv.pack(Wd)
    Y = nv.gemm(to_dev_bf16(x_bits), q, sf, ts, y_dtype=y_dtype, path=path)
    torch.cuda.synchronize()
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
    y_ref = G.gemm_ref(x_bits, q_ref, sf_ref, ts_ref)
    return Y, y_ref


def test_gemm_tiny(nv):
    W, x = S.tiny()
    Y, y_ref = run_gemm(nv, W, x)
    assert_rowwise(Y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("path", ["gemv", "gemv_regs", "auto"])
@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (1, 37, 96), (2, 100, 1024), (3, 1000, 64), (4, 513, 256),
                                   (5, 77, 17408), (7, 130, 5120), (17, 300, 512), (1, 64, 33 * 1024)])
def test_gemm_ragged(nv, M, N, K, path):
    W, x = S.random_case(M * 1000 + N + K, M, N, K)
    Y, y_ref = run_gemm(nv, W, x, path=path)
    assert_rowwise(Y.cpu().numpy(), y_ref)


def test_gemm_bf16_output(nv):
    W, x = S.random_case(31, 3, 700, 1024)
    Y, y_ref = run_gemm(nv, W, x, y_dtype=torch.bfloat16)
    y = Y.float().cpu().numpy().astype(np.float64)
    # one bf16 rounding (2^-8 relative, on top of the fp32 result) per element
    assert (np.abs(y - y_ref) <= 2.0 ** -8 * np.abs(y_ref) + 1e-5 * np.abs(y_ref).max(axis=1, keepdims=True)).all()


def test_gemm_extreme_activations(nv):
    """bf16 activations below f16's normal range inside a row of ordinary values."""
    W, x = S.random_case(41, 2, 64, 256)
    xf = G.bf16_bits_to_float64(x)
    xf[0, ::7] *= 1e-6                       # below 2^-14: f16 subnormal range
    x2 = S.f32_to_bf16_bits(xf.astype(np.float32))
    Y, y_ref = run_gemm(nv, W, x2)
    assert_rowwise(Y.cpu().numpy(), y_ref)


def _extreme_rows(seed, M, K):
    """bf16 rows far outside f16's range: large (|x| up to ~4e6, far above 65504), all tiny
    (~1e-30), one 1e30 outlier among N(0, 1) values, N(0, 1) with every 7th value scaled
    by 1e-6, and all zero; repeated to M rows."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((M, K))
    kinds = [lambda r: r * 2.0 ** 20, lambda r: r * 1e-30, None, None, lambda r: r * 0.0]
    for m in range(M):
        k = kinds[m % len(kinds)]
        if k is not None:
            base[m] = k(base[m])
        elif m % len(kinds) == 2:
            base[m, rng.integers(0, K)] = 1e30
        else:
            base[m, ::7] *= 1e-6
    return S.f32_to_bf16_bits(base.astype(np.float32))


@pytest.mark.parametrize("path,M,N,K", [("gemv", 1, 700, 5120), ("gemv", 5, 300, 1024), ("gemv_regs", 5, 300, 96),
                                        ("mma_f16", 5, 300, 1024), ("mma_f16", 100, 513, 768), ("mma", 10, 400, 512),
                                        ("auto", 1, 1000, 17408)])
def test_gemm_activation_range(nv, path, M, N, K):
    """Activations the f16 paths used to saturate (above 65504) or round away (below
    2^-14): each row is shifted by a power of two before the f16 conversion, so every row
    meets the GEMM bar, the zero row gives exactly zero, and the result is finite."""
    W, _ = S.random_case(4242 + M + K, 1, N, K)
    x = _extreme_rows(17 + M, M, K)
    Y, y_ref = run_gemm(nv, W, x, path=path)
    y = Y.cpu().numpy()
    assert np.isfinite(y).all()
    assert_rowwise(y, y_ref)


def test_verify_activation_range(nv):
    """The fused verify on the GEMV and f16 paths (one row, D = 0) with activations far above
    65504: the argmax follows the oracle. (A row of ~1e-30 values is checked too; its logits
    are all within the tie band, so only the band check bites there.)"""
    N, K = 3000, 1024
    W, _ = S.random_case(99, 1, N, K, w_std=0.05)
    rows = _extreme_rows(5, 5, K)
    for x in (rows[0:1], rows[1:2]):
        run_verify(nv, W, x, np.array([0]), 0, path="gemv")
        run_verify(nv, W, x, np.array([0]), 0, path="mma_f16")


@pytest.mark.parametrize("path", ["auto", "gemv", "gemv_regs"])
@pytest.mark.parametrize("name", S.LAYER_ORDER)
def test_gemm_layer_shapes_m1(nv, name, path):
    """The M=1 decode configuration at the 27B layer shapes, on the default path (the
    block-scaled tensor cores) and on both CUDA-core GEMVs."""
    W, x = S.layer(name, M=1)
    Y, y_ref = run_gemm(nv, W, x, path=path)
    worst = assert_rowwise(Y.cpu().numpy(), y_ref)
    if path == "auto":
        assert worst <= TERMS_TOL, f"{worst:.2e} of max|y|"


# ------------------------------------------------------------------ verify

def run_verify(nv, W, x_bits, Lstar, D, path="auto", planted_tie=None):
    N, K = W.shape
    B = len(Lstar)
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
    y_ref = G.gemm_ref(x_bits, q_ref, sf_ref, ts_ref)
    t_ref = V.argmax_fast(y_ref)
    drafts = S.drafts_with_prefix(t_ref, Lstar, D, N)
    L_ref = V.accept_ref(t_ref, drafts, D)
    assert np.array_equal(L_ref, Lstar)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    t, L, vmax = nv.verify(to_dev_bf16(x_bits), q, sf, ts, torch.from_numpy(drafts).cuda(), path=path)
    torch.cuda.synchronize()
    t, L, vmax = t.cpu().numpy(), L.cpu().numpy(), vmax.cpu().numpy()
    gap = V.top2_gap(y_ref)
    rows = V.comparable_rows(gap)
    seqs = V.comparable_sequences(gap, L_ref, D)
    assert np.array_equal(t[rows], t_ref[rows]), f"argmax mismatch on {np.flatnonzero(t[rows] != t_ref[rows])}"
    assert np.array_equal(L[seqs], L_ref[seqs])
    # the reported max logit is the oracle's logit at the reported index
    ymax = y_ref[np.arange(len(t)), t]
    assert (np.abs(vmax - ymax) <= REL_TOL * np.abs(y_ref).max(axis=1)).all()
    # on near-tie rows the GPU pick must still be within the tie band
    assert (y_ref.max(axis=1) - ymax <= V.NEAR_TIE).all()
    return t, L, rows.mean()


@pytest.mark.parametrize("B,D", [(1, 16), (2, 4), (4, 16), (3, 0)])
def test_verify_small_vocab(nv, B, D):
    N, K = 3000, 256
    W, x = S.random_case(B * 100 + D, B * (D + 1), N, K, w_std=0.05)
    Lstar = np.random.default_rng(B + D).integers(0, D + 1, size=B)
    run_verify(nv, W, x, Lstar, D)


def test_verify_exact_tie_goes_to_lowest_index(nv):
    N, K, D = 2000, 128, 2
    W, x = S.random_case(77, D + 1, N, K, w_std=0.02)
    xf = G.bf16_bits_to_float64(x)
    W[1500] = (np.sign(xf[0]) * 0.5).astype(np.float32)    # dominant row for token 0 ...
    W[700] = W[1500]                                        # ... duplicated at a lower index
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
    y_ref = G.gemm_ref(x, q_ref, sf_ref, ts_ref)
    assert y_ref[0, 700] == y_ref[0, 1500] == y_ref[0].max()
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    drafts = torch.zeros((1, D), dtype=torch.int32, device="cuda")
    t, L, _ = nv.verify(to_dev_bf16(x), q, sf, ts, drafts)
    assert t.cpu().numpy()[0] == 700


def test_verify_lmhead_slice_m17(nv):
    """lm_head verify on the 65,536-row sliced vocabulary, M = 17 (16 drafts + 1)."""
    W, x, Lstar = S.lmhead_inputs(N=S.VOCAB_SLICE, B=1)
    t, L, frac = run_verify(nv, W, x, Lstar, S.DRAFT_LEN)
    assert frac > 0.9


def test_verify_lmhead_slice_m68(nv):
    """Four sequences x 17 rows share one read of the 65,536-row head."""
    W, x, Lstar = S.lmhead_inputs(N=S.VOCAB_SLICE, B=4)
    run_verify(nv, W, x, Lstar, S.DRAFT_LEN)


def test_verify_workspace_too_small(nv):
    W, x = S.random_case(5, 2, 500, 64)
    q, sf, ts = nv.pack(torch.from_numpy(W).cuda())
    lib = nv.lib()
    X = to_dev_bf16(x)
    out = torch.empty(2, dtype=torch.int32, device="cuda")
    acc = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = lib.lmhead_verify_argmax_accept(X.data_ptr(), q.data_ptr(), sf.data_ptr(), ts.data_ptr(), 2, 500, 64,
                                         torch.zeros(1, dtype=torch.int32, device="cuda").data_ptr(), 1, 1,
                                         out.data_ptr(), acc.data_ptr(), None, ws.data_ptr(), 16,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 4
    nv.check()


# ------------------------------------------------------------------ tcgen05 MMA path

@pytest.mark.parametrize("path", ["mma", "mma_f16"])
@pytest.mark.parametrize("M,N,K", [
    (1, 128, 256),        # one tile, one chunk
    (2, 100, 1024),       # ragged N inside one tile
    (16, 256, 4096),      # 2 tiles x 16 chunks: every tile split across many CTAs
    (17, 5000, 512),      # 40 tiles x 2 chunks: every tile split in two
    (5, 1000, 17408),     # down-projection K
    (33, 3000, 2560),     # npad 48
    (68, 700, 5120),      # npad 80
    (100, 513, 768),      # npad 112
    (128, 300, 1280),     # npad 128
])
def test_gemm_mma(nv, M, N, K, path):
    """mma: block-scaled kind::mxf4nvf4 where M*5 <= 352, else f16; mma_f16: the exact f16 kernel."""
    W, x = S.random_case(M * 31 + N + K, M, N, K)
    Y, y_ref = run_gemm(nv, W, x, path=path)
    worst = assert_rowwise(Y.cpu().numpy(), y_ref)
    if path == "mma" and M * 5 <= 352:                 # block-scaled: five residual activation terms
        assert worst <= TERMS_TOL, f"{worst:.2e} of max|y|"


@pytest.mark.parametrize("M", [71, 128, 200])
def test_gemm_auto_row_slices(nv, M):
    """AUTO past M = 70: the block-scaled kernel over ceil(M/70) equal slices of X's rows, one
    launch each, sharing the workspace. A slice is the GEMM of its rows alone, so the result
    equals the slices run as separate calls, bit for bit, and keeps the five-term accuracy."""
    N, K = 1000, 1280
    W, x = S.random_case(M * 7 + 5, M, N, K)
    Wd = torch.from_numpy(W).cuda()
    q, sf, ts = nv.pack(Wd)
    X = to_dev_bf16(x)
    ws = torch.zeros(nv.gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    n0 = nv.lib().nvfp4ws_kernel_launches()
    Y = nv.gemm(X, q, sf, ts, workspace=ws)
    torch.cuda.synchronize()
    nslice = -(-M // 70)
    assert nv.lib().nvfp4ws_kernel_launches() - n0 == 2 * nslice          # prep + GEMM per slice
    nv.check()
    q_ref, sf_ref, ts_ref = F.quantize_nvfp4(W)
    y_ref = G.gemm_ref(x, q_ref, sf_ref, ts_ref)
    worst = assert_rowwise(Y.cpu().numpy(), y_ref)
    assert worst <= TERMS_TOL, f"{worst:.2e} of max|y|"
    mr = -(-M // nslice)
    for m0 in range(0, M, mr):
        Ys = nv.gemm(X[m0: m0 + mr], q, sf, ts, path="mma")
        torch.cuda.synchronize()
        assert torch.equal(Ys, Y[m0: m0 + mr])


@pytest.mark.parametrize("path", ["mma", "mma_f16"])
def test_gemm_mma_bf16_and_deterministic(nv, path):
    W, x = S.random_case(61, 17, 2000, 4096)
    Wd = torch.from_numpy(W).cuda()
    q, sf, ts = nv.pack(Wd)
    X = to_dev_bf16(x)
    ws = torch.zeros(nv.gemm_workspace_bytes(17, 2000, 4096), dtype=torch.uint8, device="cuda")
    Y1 = nv.gemm(X, q, sf, ts, workspace=ws, path=path)
    Y2 = nv.gemm(X, q, sf, ts, workspace=ws, path=path)      # the workspace counters must be zero again
    Yb = nv.gemm(X, q, sf, ts, workspace=ws, path=path, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    assert torch.equal(Yb, Y1.to(torch.bfloat16))
    nv.check()


@pytest.mark.parametrize("path", ["mma", "mma_f16"])
@pytest.mark.parametrize("name", S.LAYER_ORDER)
@pytest.mark.parametrize("M", [17, 68])
def test_gemm_layer_shapes_mma(nv, name, M, path):
    """The M=17 and M=68 launch configurations of the bench at the 27B layer shapes."""
    W, x = S.layer(name, M=M)
    Y, y_ref = run_gemm(nv, W, x, path=path)
    worst = assert_rowwise(Y.cpu().numpy(), y_ref)
    if path == "mma":                                  # block-scaled: five residual activation terms
        assert worst <= TERMS_TOL, f"{worst:.2e} of max|y|"


@pytest.mark.parametrize("path", ["mma", "mma_f16"])
@pytest.mark.parametrize("B,D", [(1, 16), (4, 16), (2, 3)])
def test_verify_mma_small_vocab(nv, B, D, path):
    N, K = 3000, 512
    W, x = S.random_case(B * 7 + D, B * (D + 1), N, K, w_std=0.05)
    Lstar = np.random.default_rng(B * 3 + D).integers(0, D + 1, size=B)
    run_verify(nv, W, x, Lstar, D, path=path)


@pytest.mark.parametrize("path", ["mma", "mma_f16"])
@pytest.mark.parametrize("B", [1, 4])
def test_verify_mma_lmhead_slice(nv, path, B):
    W, x, Lstar = S.lmhead_inputs(N=S.VOCAB_SLICE, B=B)
    run_verify(nv, W, x, Lstar, S.DRAFT_LEN, path=path)


@pytest.mark.parametrize("path", ["gemv", "gemv_regs"])
@pytest.mark.parametrize("B,D", [(1, 0), (1, 16), (2, 1)])
def test_verify_gemv_variants(nv, path, B, D):
    N, K = 2500, 1024
    W, x = S.random_case(B * 13 + D, B * (D + 1), N, K, w_std=0.05)
    Lstar = np.random.default_rng(B * 5 + D).integers(0, D + 1, size=B)
    run_verify(nv, W, x, Lstar, D, path=path)
