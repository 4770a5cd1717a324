"""Planted mistakes: each test patches a plausible bug into the oracle (on the CPU
only) and checks that one of the pins catches it. This shows the pins cover every
part of the oracle."""

import json
import os

import numpy as np
import pytest

from oracle import nvfp4 as F
from oracle import verify as V

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand_blocks_pass():
    with open(os.path.join(GOLDEN, "hand_blocks.json")) as f:
        g = json.load(f)
    W = np.array(g["W"], dtype=np.float32)
    for case in g["cases"]:
        q, sf, ts = F.quantize_nvfp4(W, case["tensor_scale_in"])
        if float(ts) != case["ts"] or sf.tolist() != case["sf"] or q.tolist() != case["q"]:
            return False
    return True


def test_baseline_passes():
    assert _hand_blocks_pass()


def test_swapped_nibbles_caught(monkeypatch):
    monkeypatch.setattr(F, "pack_codes", lambda c: (np.asarray(c)[:, 1::2] & 0xF) | ((np.asarray(c)[:, 0::2] & 0xF) << 4))
    assert not _hand_blocks_pass()


def test_ties_away_from_zero_caught(monkeypatch):
    def bad(a):
        a = np.minimum(np.asarray(a, dtype=np.float64), 6.0)
        _, ex = np.frexp(a)
        e = np.maximum(ex - 1, 0) - 1
        return np.minimum(np.ldexp(np.floor(np.ldexp(a, -e) + 0.5), e), 6.0)
    monkeypatch.setattr(F, "e2m1_round_magnitude", bad)
    assert not _hand_blocks_pass()


def test_unrounded_block_scale_caught(monkeypatch):
    orig = F.e4m3_encode
    # plant: use the unrounded quotient for the element codes by rounding the scale toward zero
    def bad(v):
        v = np.asarray(v, dtype=np.float64)
        c = orig(v)
        down = np.maximum(c.astype(np.int32) - 1, 0).astype(np.uint8)
        return np.where(F.E4M3_VALUES[c] > v, down, c)
    monkeypatch.setattr(F, "e4m3_encode", bad)
    assert not _hand_blocks_pass()


def test_absolute_block_scale_reading_caught(monkeypatch):
    """The literal reading S = amax/6 (ignoring ts) gives different scale bytes."""
    orig = F.quantize_codes
    def bad(W, tensor_scale_in=None):
        codes, sf, ts = orig(W, tensor_scale_in)
        amax_b = np.abs(np.asarray(W, np.float64)).reshape(W.shape[0], -1, 16).max(axis=2)
        return codes, F.e4m3_encode(amax_b / 6.0), ts
    monkeypatch.setattr(F, "quantize_codes", bad)
    assert not _hand_blocks_pass()


def test_dropped_sign_caught(monkeypatch):
    orig = F.e2m1_encode
    monkeypatch.setattr(F, "e2m1_encode", lambda r: orig(np.abs(r)))
    assert not _hand_blocks_pass()


def test_dropped_tensor_scale_in_dequant_caught():
    q, sf, ts = F.quantize_nvfp4(np.array([[6.0] + [1.0] * 15], np.float32), 2.0 ** -4)
    good = F.dequantize_nvfp4(q, sf, ts)
    bad = F.dequantize_nvfp4(q, sf, 1.0)
    assert not np.array_equal(good, bad)
    assert good[0, 0] == 6.0                           # the round-trip pin holds only with ts applied


def test_accept_off_by_one_caught():
    t = np.array([1, 2, 3])
    d = np.array([[1, 9]])
    assert V.accept_ref(t, d, 2).tolist() == [1]
    bad = lambda t, d, D: np.array([min(D, V.accept_ref(t, d, D)[0] + 1)])
    assert bad(t, d, 2).tolist() != [1]


def test_last_index_argmax_caught():
    y = np.array([[1.0, 3.0, 3.0]])
    last = y.shape[1] - 1 - np.argmax(y[:, ::-1], axis=1)
    assert last.tolist() != V.argmax_ref(y).tolist()


def test_tree_child_row_instead_of_parent_row_caught():
    """Checking a node's draft against its own row (not its parent's) breaks the hand-worked tree."""
    with open(os.path.join(GOLDEN, "tree_verify.json")) as f:
        case = json.load(f)["cases"][0]
    p, d, t = np.array([case["parents"]]), np.array([case["drafts"]]), np.array(case["t"])
    D = p.shape[1]

    def wrong(t, d, p, D):
        L, node, acc, depth = 0, 0, [True] + [False] * D, [0] * (D + 1)
        for k in range(1, D + 1):
            q = int(p[0, k - 1])
            depth[k] = depth[q] + 1
            acc[k] = acc[q] and d[0, k - 1] == t[k]
            if acc[k] and depth[k] > L:
                L, node = depth[k], k
        return L, node

    assert wrong(t, d, p, D) != (case["accept_len"], case["accept_node"])
    L, node = V.accept_tree_ref(t, d, p, D)
    assert (int(L[0]), int(node[0])) == (case["accept_len"], case["accept_node"])


# ------------------------------------------------------------------ FP8 block-scaled weights

def _fp8_pins_pass():
    """The FP8 pins: the hand-worked blocks (scales, codes, dequantised values) and a
    brute-force GEMM over non-square blocks."""
    import synthetic as S
    from oracle import fp8 as P8
    from oracle import gemm as G
    with open(os.path.join(GOLDEN, "fp8_blocks.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        W = np.array(case["W"], dtype=np.float32)
        block = tuple(case["block"])
        codes, scales = P8.quantize_fp8_blocks(W, block)
        if scales.tolist() != case["scales"] or codes.tolist() != case["codes"]:
            return False
        if P8.dequantize_fp8_blocks(codes, scales, block).tolist() != case["dequant"]:
            return False
    W, x = S.random_case(85, 2, 5, 40)
    codes, scales = P8.quantize_fp8_blocks(W, (2, 8))
    y = P8.gemm_fp8_ref(x, codes, scales, (2, 8))
    xf = G.bf16_bits_to_float64(x)
    for m in range(2):
        for n in range(5):
            acc = sum(xf[m, k] * F.E4M3_VALUES[codes[n, k]] * float(scales[n // 2, k // 8]) for k in range(40))
            if abs(y[m, n] - acc) > 1e-12 * max(1e-30, abs(acc)):
                return False
    return True


def test_fp8_baseline_passes():
    assert _fp8_pins_pass()


def test_fp8_nvfp4_scale_rule_caught(monkeypatch):
    """s = amax/6 (the NVFP4 rule) in place of amax/448."""
    from oracle import fp8 as P8
    monkeypatch.setattr(P8, "E4M3_MAX", 6.0)
    assert not _fp8_pins_pass()


def test_fp8_ties_away_from_zero_caught(monkeypatch):
    from oracle import fp8 as P8
    orig = P8.e4m3_encode
    monkeypatch.setattr(P8, "e4m3_encode", lambda v: orig(np.asarray(v, np.float64) * (1.0 + 2.0 ** -30)))
    assert not _fp8_pins_pass()


def test_fp8_dropped_sign_caught(monkeypatch):
    from oracle import fp8 as P8
    orig = P8.e4m3_encode
    monkeypatch.setattr(P8, "e4m3_encode", lambda v: orig(np.abs(np.asarray(v, np.float64))))
    assert not _fp8_pins_pass()


def test_fp8_transposed_block_index_caught(monkeypatch):
    """The scale of block (k // bc, n // br) instead of (n // br, k // bc)."""
    from oracle import fp8 as P8

    def bad(codes, scales, block=P8.BLOCK):
        codes = np.asarray(codes, dtype=np.uint8)
        N, K = codes.shape
        br, bc = block
        s = np.asarray(scales, dtype=np.float64)
        flat = s.reshape(-1)
        idx = (np.arange(K)[None, :] // bc) * s.shape[1] + (np.arange(N)[:, None] // br)
        return F.E4M3_VALUES[codes] * flat[np.minimum(idx, flat.size - 1)]
    monkeypatch.setattr(P8, "dequantize_fp8_blocks", bad)
    assert not _fp8_pins_pass()


def test_fp8_unsigned_dequant_caught(monkeypatch):
    from oracle import fp8 as P8
    monkeypatch.setattr(P8, "E4M3_VALUES", np.abs(F.E4M3_VALUES))
    assert not _fp8_pins_pass()


# ------------------------------------------------------------------ W4A4 activation rows

def _w4a4_pins_pass():
    """The W4A4 pins: the hand-worked rows (row scales, block scales, codes) and a brute-force
    product over the dequantised rows."""
    import synthetic as S
    from oracle import gemm as G
    with open(os.path.join(GOLDEN, "w4a4_rows.json")) as f:
        g = json.load(f)
    rows = np.asarray(g["rows"], dtype=np.float32)
    bits = (rows.view(np.uint32) >> 16).astype(np.uint16)
    codes, sf, gs = G.quantize_x_rows(bits)
    if gs.tolist() != g["g"] or sf.tolist() != g["sf"] or codes.tolist() != g["codes"]:
        return False
    W, x = S.random_case(9, 2, 3, 48)
    q, wsf, ts = F.quantize_nvfp4(W)
    y = G.gemm_w4a4_ref(x, q, wsf, ts)
    xc, xs, xg = G.quantize_x_rows(x)
    wc = F.unpack_codes(q)
    for m in range(2):
        for n in range(3):
            acc = sum(F.E2M1_VALUES[xc[m, k]] * F.E4M3_VALUES[xs[m, k // 16]] * float(xg[m]) *
                      F.E2M1_VALUES[wc[n, k]] * F.E4M3_VALUES[wsf[n, k // 16]] * float(ts) for k in range(48))
            if abs(y[m, n] - acc) > 1e-12 * max(1e-30, abs(acc)):
                return False
    return True


def test_w4a4_baseline_passes():
    assert _w4a4_pins_pass()


def test_w4a4_fp8_style_row_scale_caught(monkeypatch):
    """g = amax/448 (an FP8 rule) in place of amax/2688."""
    monkeypatch.setattr(F, "TENSOR_SCALE_DIVISOR", 448.0)
    assert not _w4a4_pins_pass()


def test_w4a4_dropped_sign_caught(monkeypatch):
    orig = F.e2m1_encode
    monkeypatch.setattr(F, "e2m1_encode", lambda r: orig(np.abs(np.asarray(r, np.float64))))
    assert not _w4a4_pins_pass()


def test_w4a4_ties_away_from_zero_caught(monkeypatch):
    orig = F.e2m1_encode
    monkeypatch.setattr(F, "e2m1_encode", lambda r: orig(np.asarray(r, np.float64) * (1.0 + 2.0 ** -30)))
    assert not _w4a4_pins_pass()


def _fp32_activation_quantiser(recip_scale: bool, fp32_codes: bool):
    """A planted mistake: the activation rows quantised with fp32 steps instead of exact
    quotients: the block scale as amax_block * fp32(1 / fp32(6 g)) and/or the code from
    fp32(x / fp32(S g))."""
    from oracle import gemm as G

    def q(x_bits):
        x = G.bf16_bits_to_float64(x_bits).astype(np.float32)
        M, K = x.shape
        amax = np.max(np.abs(x), axis=1)
        g = (amax / np.float32(2688.0)).astype(np.float32)
        blocks = x.reshape(M, K // 16, 16)
        bmax = np.max(np.abs(blocks), axis=2)
        with np.errstate(divide="ignore", invalid="ignore"):
            if recip_scale:
                inv = np.where(g > 0, np.float32(1.0) / (np.float32(6.0) * g), np.float32(0.0)).astype(np.float32)
                a = (bmax * inv[:, None]).astype(np.float64)
            else:
                a = np.where(g[:, None] > 0, bmax.astype(np.float64) / (6.0 * g[:, None].astype(np.float64)), 0.0)
            sf = F.e4m3_encode(a)
            Sv = F.E4M3_VALUES[sf]
            if fp32_codes:
                den = (Sv.astype(np.float32) * g[:, None]).astype(np.float32)
                r = np.where(den[:, :, None] > 0, blocks / np.where(den > 0, den, 1)[:, :, None], 0).astype(np.float32)
            else:
                den = Sv * g[:, None].astype(np.float64)
                r = np.where(den[:, :, None] > 0, blocks / np.where(den > 0, den, 1)[:, :, None], 0.0)
        codes = np.where(Sv[:, :, None] > 0, F.e2m1_encode(np.asarray(r, np.float64)), 0).astype(np.uint8)
        return codes.reshape(M, K), sf.astype(np.uint8), g
    return q


def test_w4a4_plain_form_of_the_planted_quantiser_passes(monkeypatch):
    """The planting helper with exact quotients is the oracle's rule: the pins pass with it."""
    from oracle import gemm as G
    monkeypatch.setattr(G, "quantize_x_rows", _fp32_activation_quantiser(False, False))
    assert _w4a4_pins_pass()


def test_w4a4_reciprocal_block_scale_caught(monkeypatch):
    """S from amax_block * fp32(1 / fp32(6 g)) instead of the exact quotient (golden row 5)."""
    from oracle import gemm as G
    monkeypatch.setattr(G, "quantize_x_rows", _fp32_activation_quantiser(True, False))
    assert not _w4a4_pins_pass()


def test_w4a4_fp32_code_quotient_caught(monkeypatch):
    """Codes from fp32(x / fp32(S g)) instead of the exact quotient (golden row 4)."""
    from oracle import gemm as G
    monkeypatch.setattr(G, "quantize_x_rows", _fp32_activation_quantiser(False, True))
    assert not _w4a4_pins_pass()


def test_w4a4_block_scale_of_the_wrong_block_caught(monkeypatch):
    """Dequantisation with the scale of block k // 8 instead of k // 16."""
    from oracle import gemm as G

    def bad(codes, sf, g):
        codes = np.asarray(codes)
        K = codes.shape[1]
        idx = np.minimum(np.arange(K) // 8, sf.shape[1] - 1)
        return F.E2M1_VALUES[codes] * F.E4M3_VALUES[sf][:, idx] * np.asarray(g, np.float64)[:, None]
    monkeypatch.setattr(G, "dequantize_x_rows", bad)
    assert not _w4a4_pins_pass()
