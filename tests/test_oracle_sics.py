"""Pins of the SPADE SICS oracle (sum of intra-block cosine similarities, per-head
choice of a slicing from a shape menu) against closed forms and constructed
inputs whose answer the mathematics fixes."""
import numpy as np
import pytest

import oracle as O

MENU = [(4, 4, 4), (1, 8, 8), (2, 4, 8), (16, 2, 2)]


def test_tile_tokens_partition_and_match_tile_order():
    grid, tile = (5, 7, 9), (2, 3, 4)
    nt = 3 * 3 * 3
    parts = [O.tile_tokens(grid, tile, t) for t in range(nt)]
    allidx = np.concatenate(parts)
    assert np.array_equal(np.sort(allidx), np.arange(5 * 7 * 9))
    # concatenated in tile order they are exactly the tile permutation
    assert np.array_equal(allidx, O.tile_order(grid, tile))


def test_sics_equals_squared_norm_of_summed_unit_vectors():
    # sum_{i,j} cos(x_i, x_j) = || sum_i x_i / |x_i| ||^2 (closed form), ragged tiles
    rng = np.random.default_rng(0)
    grid, tile = (3, 5, 7), (2, 2, 3)
    x = rng.standard_normal((2, 105, 3, 16))
    got = O.sics_blocks(x, grid, tile)
    for t in range(2 * 3 * 3):
        idx = O.tile_tokens(grid, tile, t)
        for b in range(2):
            for h in range(3):
                u = x[b, idx, h] / np.linalg.norm(x[b, idx, h], axis=1, keepdims=True)
                assert abs(got[b, h, t] - np.sum(u.sum(axis=0) ** 2)) < 1e-9


def test_identical_orthogonal_and_opposite_vectors():
    grid, tile = (1, 2, 4), (1, 2, 2)              # two blocks of 4 tokens
    x = np.zeros((1, 8, 1, 8))
    base = np.arange(1, 9, dtype=np.float64)
    for i in range(4):
        x[0, O.tile_tokens(grid, tile, 0)[i], 0] = base * (i + 1)   # same direction
    for i in range(4):
        x[0, O.tile_tokens(grid, tile, 1)[i], 0, i] = 1.0           # orthonormal
    s = O.sics_blocks(x, grid, tile)[0, 0]
    assert abs(s[0] - 16.0) < 1e-12 and abs(s[1] - 4.0) < 1e-12
    # x and -x cancel: a block {v, -v} has SICS 2 - 2 = 0; a zero vector adds nothing
    y = np.zeros((1, 3, 1, 4))
    y[0, 0, 0] = [1, 2, 3, 4]
    y[0, 1, 0] = [-1, -2, -3, -4]
    assert abs(O.sics_blocks(y, (1, 1, 3), (1, 1, 3))[0, 0, 0]) < 1e-12


def test_scale_invariance():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 64, 2, 8))
    s = rng.uniform(0.1, 10.0, size=(1, 64, 2, 1))
    a = O.sics_blocks(x, (4, 4, 4), (2, 2, 2))
    b = O.sics_blocks(x * s, (4, 4, 4), (2, 2, 2))
    assert np.allclose(a, b, rtol=0, atol=1e-10)


def _field(grid, D, seed, axis):
    """Token vectors that depend only on the spatial position (axis='space') or only
    on the frame (axis='time')."""
    T, H, W = grid
    rng = np.random.default_rng(seed)
    if axis == "space":
        v = rng.standard_normal((H * W, D))
        return np.stack([v[(n % (H * W))] for n in range(T * H * W)])
    v = rng.standard_normal((T, D))
    return np.stack([v[n // (H * W)] for n in range(T * H * W)])


def test_scheme_picks_the_slicing_the_field_is_constant_along():
    grid, D = (16, 8, 8), 64
    q = np.zeros((1, 16 * 64, 2, D))
    q[0, :, 0] = _field(grid, D, 3, "space")     # head 0: constant along time
    q[0, :, 1] = _field(grid, D, 4, "time")      # head 1: constant within a frame
    k = q.copy()
    scores, choice = O.sics_scheme(q, k, grid, MENU)
    assert choice[0, 0] == 3          # 16x2x2: long in time, thin in space
    assert choice[0, 1] == 1          # 1x8x8: one frame, wide in space
    assert abs(scores[0, 1, 1] - 1.0) < 1e-12      # every pair in a frame agrees
    # time-constant field under 16x2x2: 4 positions x 16 identical tokens per block
    # -> coherence 1/4 plus the (small) cross-position cosines
    assert 0.2 < scores[0, 0, 3] < 0.35


def test_scheme_scores_queries_and_keys_alike():
    # one 8x8 frame, D = 64: Q = 64 orthonormal vectors (SICS = n, the diagonal
    # alone), K = one vector repeated (SICS = n^2).  Shape 1x8x8 is one block of 64
    # tokens, shape 1x4x16 two ragged 4x8 blocks of 32, so the score
    # (SICS_Q + SICS_K) / (2 sum n_b^2) is (64 + 4096) / 8192 and (64 + 2048) / 4096
    grid = (1, 8, 8)
    q = np.eye(64)[None, :, None, :]
    k = np.ones((1, 64, 1, 64))
    scores, choice = O.sics_scheme(q, k, grid, [(1, 8, 8), (1, 4, 16)])
    assert abs(scores[0, 0, 0] - 4160 / 8192) < 1e-12
    assert abs(scores[0, 0, 1] - 2112 / 4096) < 1e-12
    assert choice[0, 0] == 1
    swapped, _ = O.sics_scheme(k, q, grid, [(1, 8, 8), (1, 4, 16)])
    assert np.allclose(swapped, scores, atol=1e-12, rtol=0)


def test_scheme_ties_take_the_first_menu_entry():
    grid = (4, 8, 8)
    x = np.ones((1, 256, 1, 8))
    scores, choice = O.sics_scheme(x, x, grid, MENU[:3])
    assert np.allclose(scores, 1.0) and choice[0, 0] == 0


def test_every_menu_shape_holds_its_block_size():
    from block_sparse_attention_tokens_b200 import configs
    for block, menu in configs.SICS_MENUS.items():
        assert len(menu) >= 3
        for shape in menu:
            assert shape[0] * shape[1] * shape[2] == block, (block, shape)
        assert len(set(menu)) == len(menu)
