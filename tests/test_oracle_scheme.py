"""Pins of the oracle's per-head slicing permute (CPU only).

SPADE summary (gist.science/ja/paper/2608.03335), solution parts 1 and 3: every
head is cut with its own slice shape of a menu.  The oracle's scheme_permute is
tied to a hand-worked fixture with ragged tiles and mixed per-head choices, to the
whole-tensor tile_permute when every head takes the same shape, and to its inverse.
"""
import numpy as np
import pytest

import oracle as O
from tests._golden import load

SHAPES = ((1, 2, 2), (2, 1, 1), (2, 2, 2))
GRID = (2, 3, 2)


def _ids(batch, n, heads):
    """x[b, i, h, 0] = 1000 b + 100 h + i: every element names its source."""
    b, i, h = np.meshgrid(np.arange(batch), np.arange(n), np.arange(heads), indexing="ij")
    return (1000 * b + 100 * h + i).astype(np.float64)[..., None]


def test_scheme_permute_golden_mixed_choices():
    orders = load("scheme_order_2x3x2.txt").astype(int).reshape(3, 12)
    choice = np.array([[1, 2, 0], [2, 0, 1]])
    x = _ids(2, 12, 3)
    y = O.scheme_permute(x, GRID, SHAPES, choice, n_pad=16)
    assert y.shape == (2, 16, 3, 1)
    for b in range(2):
        for h in range(3):
            expect = 1000 * b + 100 * h + orders[choice[b, h]]
            assert y[b, :12, h, 0].tolist() == expect.tolist(), (b, h)
    assert not y[:, 12:].any()


def test_scheme_untile_golden_mixed_choices():
    orders = load("scheme_order_2x3x2.txt").astype(int).reshape(3, 12)
    choice = np.array([[0, 1, 2], [1, 1, 2]])
    y = np.zeros((2, 13, 3, 1))
    y[:, :12] = np.arange(12, dtype=np.float64)[None, :, None, None]   # y[b, p, h] = p
    x = O.scheme_untile(y, GRID, SHAPES, choice)
    for b in range(2):
        for h in range(3):
            # raster token orders[c][p] holds position p
            got = x[b, orders[choice[b, h]], h, 0]
            assert got.tolist() == list(range(12)), (b, h)


@pytest.mark.parametrize("shape", [(4, 4, 4), (1, 8, 8), (16, 2, 2)])
def test_scheme_permute_uniform_choice_is_tile_permute(shape):
    rng = np.random.default_rng(3)
    grid = (5, 9, 7)
    n = 5 * 9 * 7
    x = rng.standard_normal((2, n, 3, 4))
    shapes = ((4, 4, 4), (1, 8, 8), (16, 2, 2))
    choice = np.full((2, 3), shapes.index(shape))
    n_pad = -(-n // 64) * 64
    y = O.scheme_permute(x, grid, shapes, choice, n_pad)
    assert np.array_equal(y, O.tile_permute(x, O.tile_order(grid, shape), n_pad))


def test_scheme_roundtrip_random_choices():
    rng = np.random.default_rng(4)
    grid = (6, 5, 11)
    n = 330
    shapes = ((4, 4, 4), (1, 8, 8), (2, 4, 8), (16, 2, 2))
    x = rng.standard_normal((3, n, 5, 2))
    choice = rng.integers(0, 4, size=(3, 5))
    y = O.scheme_permute(x, grid, shapes, choice, 384)
    assert np.array_equal(O.scheme_untile(y, grid, shapes, choice), x)
    # each head's column of y is a permutation of that head's tokens
    for b in range(3):
        for h in range(5):
            assert np.array_equal(np.sort(y[b, :n, h, 0]), np.sort(x[b, :, h, 0]))
