"""CPU: the seeded input recipes that both the oracle and the CUDA path consume, checked
against their stated definitions (the generators hold no arithmetic of the method)."""

import numpy as np
import torch

import synthetic as S


def test_tiny_is_two_draws_of_one_generator():
    W, x = S.tiny()
    rng = np.random.default_rng(0)
    W_ref = (rng.standard_normal((1024, 1024)) * S.W_STD).astype(np.float32)
    x_ref = S.f32_to_bf16_bits(rng.standard_normal((1, 1024)).astype(np.float32))
    assert np.array_equal(W, W_ref) and np.array_equal(x, x_ref)


def test_chunked_weight_draw_equals_one_draw():
    """normal_weight draws row chunks; the stream is that of one standard_normal((N, K)) call,
    so a sliced vocabulary is the first rows of the full one."""
    a = S.normal_weight(np.random.default_rng(5), 1000, 48, row_chunk=64)
    b = (np.random.default_rng(5).standard_normal((1000, 48)) * S.W_STD).astype(np.float32)
    assert np.array_equal(a, b)
    assert np.array_equal(S.normal_weight(np.random.default_rng(5), 300, 48, row_chunk=7), a[:300])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        # exact ties between two bf16 values: low 16 bits 0x8000, both parities
                        (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32) * 1,
                        np.array([0.0, -0.0, 1e-40, -1e-40, 3.4e38], dtype=np.float32)])
    ours = S.f32_to_bf16_bits(v)
    theirs = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_layer_recipe():
    K, N = S.LAYER_SHAPES["qkv"]
    W, x = S.layer("qkv", M=3, w_seed=3, x_seed=103)
    assert W.shape == (N, K) and x.shape == (3, K)
    assert np.array_equal(x, S.normal_x_bits(np.random.default_rng(103), 3, K))


def test_drafts_with_prefix_fix_the_first_disagreement():
    rng = np.random.default_rng(11)
    B, D, V = 6, 16, 50
    t = rng.integers(0, V, size=B * (D + 1))
    Lstar = np.array([0, 1, 5, 15, 16, 16])
    d = S.drafts_with_prefix(t, Lstar, D, V, seed=3)
    for b in range(B):
        row = t[b * (D + 1): b * (D + 1) + D]
        agree = d[b] == row
        first = int(np.argmin(agree)) if not agree.all() else D
        assert first == Lstar[b]


def test_random_tree_parents_precede_children():
    p = S.random_tree(8, 40, seed=2, chain_bias=0.3)
    k = np.arange(1, 41)
    assert ((p >= 0) & (p <= k - 1)).all()
    assert (S.random_tree(2, 9, seed=1, chain_bias=1.0) == np.arange(9)).all()     # all chains


def test_tree_drafts_agree_or_differ_from_the_parent_row():
    rng = np.random.default_rng(12)
    B, D, V = 3, 20, 30
    t = rng.integers(0, V, size=B * (D + 1))
    p = S.random_tree(B, D, seed=4)
    d = S.tree_drafts(t, p, D, V, agree=1.0, seed=5)
    for b in range(B):
        assert all(d[b, k - 1] == t[b * (D + 1) + p[b, k - 1]] for k in range(1, D + 1))
    d = S.tree_drafts(t, p, D, V, agree=0.0, seed=5)
    for b in range(B):
        assert all(d[b, k - 1] != t[b * (D + 1) + p[b, k - 1]] for k in range(1, D + 1))


def test_block_varied_case_scales_whole_blocks_by_powers_of_two():
    W, x = S.block_varied_case(9, 2, 300, 384)
    rng = np.random.default_rng(9)
    base = S.normal_weight(rng, 300, 384)
    ratio = W.astype(np.float64) / base.astype(np.float64)
    e = rng.integers(-4, 5, size=(3, 3))                      # the next draw: one exponent per block
    for i in range(0, 300, 128):
        for j in range(0, 384, 128):
            r = np.unique(ratio[i:i + 128, j:j + 128])
            assert r.size == 1 and r[0] == 2.0 ** e[i // 128, j // 128]
    assert np.array_equal(x, S.normal_x_bits(rng, 2, 384))


def test_lmhead_weight_is_chunk_seeded():
    """Chunk c of the lm_head weight comes from default_rng([7, c]) alone, so a slice is the
    first rows of the full weight and any chunk can be drawn by itself."""
    K = 32
    W = S.lmhead_weight(N=3 * S.LMHEAD_CHUNK + 5, K=K)
    ref1 = (np.random.default_rng([S.LMHEAD_W_SEED, 1]).standard_normal((S.LMHEAD_CHUNK, K)) * S.W_STD)
    assert np.array_equal(W[S.LMHEAD_CHUNK: 2 * S.LMHEAD_CHUNK], ref1.astype(np.float32))
    assert np.array_equal(W[3 * S.LMHEAD_CHUNK:], S.lmhead_weight_chunk(3, N=3 * S.LMHEAD_CHUNK + 5, K=K))
    assert np.array_equal(S.lmhead_weight(N=S.LMHEAD_CHUNK + 7, K=K), W[:S.LMHEAD_CHUNK + 7])
    x4, x1 = S.lmhead_x(B=4, K=K), S.lmhead_x(B=1, K=K)
    assert x4.shape == (68, K) and np.array_equal(x4[:17], x1)
