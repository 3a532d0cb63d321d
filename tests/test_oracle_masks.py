"""Pins of the oracle's permute, STA, radial and CSR builders (CPU only).

Each check ties the oracle to something other than itself: hand-computed
fixtures, closed-form counts, library routines (numpy reshape/transpose, scipy
sparse) or brute-force enumeration of the token-level rule on tiny grids.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.sparse

import oracle as O
from tests._golden import load


# ----------------------------------------------------------------- permute

def test_tile_order_golden_ragged():
    perm = O.tile_order((1, 3, 3), (1, 2, 2))
    assert perm.tolist() == load("tile_order_1x3x3_t1x2x2.txt").astype(int).ravel().tolist()


@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (4, 4, 4)), ((6, 4, 10), (2, 2, 5)),
                                       ((30, 48, 80), (6, 8, 8))])
def test_tile_order_matches_reshape_transpose_when_divisible(grid, tile):
    T, H, W = grid
    tT, tH, tW = tile
    ids = np.arange(T * H * W).reshape(T // tT, tT, H // tH, tH, W // tW, tW)
    expect = ids.transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    assert np.array_equal(O.tile_order(grid, tile), expect)


@pytest.mark.parametrize("grid,tile", [((21, 30, 52), (4, 4, 4)), ((5, 7, 3), (2, 3, 2)),
                                       ((1, 1, 1), (4, 4, 4))])
def test_tile_order_bijection_and_tile_contiguity(grid, tile):
    perm = O.tile_order(grid, tile)
    n = int(np.prod(grid))
    assert np.array_equal(np.sort(perm), np.arange(n))
    T, H, W = grid
    t, h, w = perm // (H * W), (perm // W) % H, perm % W
    tid = ((t // tile[0]) * math.ceil(H / tile[1]) + h // tile[1]) * math.ceil(W / tile[2]) + w // tile[2]
    # tiles appear as contiguous runs in increasing tile order
    assert np.all(np.diff(tid) >= 0)
    # each tile holds exactly its (possibly ragged) volume
    counts = np.bincount(tid)
    for a in range(math.ceil(T / tile[0])):
        for b in range(math.ceil(H / tile[1])):
            for c in range(math.ceil(W / tile[2])):
                vol = (min(tile[0], T - a * tile[0]) * min(tile[1], H - b * tile[1])
                       * min(tile[2], W - c * tile[2]))
                idx = (a * math.ceil(H / tile[1]) + b) * math.ceil(W / tile[2]) + c
                assert counts[idx] == vol


def test_permute_untile_roundtrip_and_zero_tail():
    rng = np.random.default_rng(0)
    grid, tile = (5, 7, 3), (2, 3, 2)
    n = 105
    x = rng.standard_normal((2, n, 6))
    perm = O.tile_order(grid, tile)
    y = O.tile_permute(x, perm, 128)
    assert y.shape == (2, 128, 6)
    assert np.all(y[:, n:] == 0)
    assert np.array_equal(O.tile_untile(y, perm), x)
    # position p holds raster token perm[p]
    assert np.array_equal(y[:, 17], x[:, perm[17]])


# ----------------------------------------------------------------- STA

def test_sta_golden_band():
    m = O.sta_tile_mask((1, 1, 5), (1, 1, 3))
    assert np.array_equal(m, load("sta_band_1x1x5_w1x1x3.txt").astype(np.uint8))


def _axis_count(n, w, shift):
    lo_off, hi_off = (w - 1) // 2, w // 2
    total = 0
    for a in range(n):
        if shift:
            total += min(w, n)
        else:
            total += min(a + hi_off, n - 1) - max(a - lo_off, 0) + 1
    return total


@pytest.mark.parametrize("shift", [False, True])
def test_sta_kept_count_closed_form_720p(shift):
    tile_grid, window = (5, 6, 10), (3, 3, 5)
    m = O.sta_tile_mask(tile_grid, window, shift)
    expect = np.prod([_axis_count(n, w, shift) for n, w in zip(tile_grid, window)])
    assert int(m.sum()) == expect
    assert int(m.sum()) == (9152 if not shift else 13500)


def test_sta_symmetric_and_tiny_all_ones():
    m = O.sta_tile_mask((3, 4, 5), (3, 3, 3))
    assert np.array_equal(m, m.T)
    assert np.all(np.diag(m) == 1)
    # 4x8x8 grid in 4x4x4 tiles is a 1x2x2 tile grid; a 1x3x3 window covers it
    assert np.all(O.sta_tile_mask((1, 2, 2), (1, 3, 3)) == 1)


@pytest.mark.parametrize("shift", [False, True])
def test_sta_matches_token_level_enumeration(shift):
    grid, tile, window = (4, 6, 6), (2, 2, 3), (3, 1, 3)
    T, H, W = grid
    tg = tuple(g // t for g, t in zip(grid, tile))
    n = T * H * W
    vol = int(np.prod(tile))
    # token-level rule in raster order, straight from the window definition
    coords = [(i // (H * W) // tile[0], (i // W) % H // tile[1], i % W // tile[2]) for i in range(n)]
    allowed = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            ok = True
            for ax in range(3):
                a, a2, nn, w = coords[i][ax], coords[j][ax], tg[ax], window[ax]
                if shift:
                    start = min(max(a - (w - 1) // 2, 0), max(nn - w, 0))
                    ok &= start <= a2 < start + w
                else:
                    ok &= -((w - 1) // 2) <= a2 - a <= w // 2
            allowed[i, j] = ok
    perm = O.tile_order(grid, tile)
    tok = allowed[perm][:, perm]
    blocks = tok.reshape(n // vol, vol, n // vol, vol).any(axis=(1, 3)).astype(np.uint8)
    assert np.array_equal(blocks, O.sta_tile_mask(tg, window, shift))


# ----------------------------------------------------------------- radial

def test_radial_token_rule_golden():
    for fq, sq, fk, sk, keep in load("radial_rule_S16_B4.txt").astype(int):
        assert O.radial_token_keep(fq, sq, fk, sk, 16, 4) == bool(keep), (fq, sq, fk, sk)


@pytest.mark.parametrize("frames,S,B,n", [(12, 16, 4, None), (20, 8, 8, None), (9, 6, 8, 50),
                                          (17, 16, 8, 16 * 17 - 5), (33, 4, 8, None),
                                          (11, 5, 8, None)])
def test_radial_block_mask_equals_token_enumeration(frames, S, B, n):
    # (11, 5, 8): block 3 = tokens 24..31 touches frames 4, 5 and 6
    n = frames * S if n is None else n
    nb = math.ceil(n / B)
    brute = np.zeros((nb, nb), dtype=np.uint8)
    for i in range(n):
        for j in range(n):
            if O.radial_token_keep(i // S, i % S, j // S, j % S, S, B):
                brute[i // B, j // B] = 1
    assert np.array_equal(O.radial_block_mask(n, S, B), brute)
    assert np.array_equal(O.radial_block_mask_fast(n, S, B), brute)


def test_radial_symmetry_and_diagonal():
    m = O.radial_block_mask_fast(64 * 40, 64, 16)
    assert np.array_equal(m, m.T)
    assert np.all(np.diag(m) == 1)


def test_radial_kept_pairs_grow_as_n_log_n():
    """Radial explainer, sections 1-3: the kept-pair count is O(n log n).

    Doubling the number of frames quadruples a dense mask; here the growth
    factor falls towards 2 and kept / (NB log2 T) converges (its increments
    shrink geometrically), as O(n log n) requires.
    """
    S, B = 256, 32
    ratios, growth = [], []
    prev = None
    for T in (16, 32, 64, 128, 256, 512):
        m = O.radial_block_mask_fast(T * S, S, B)
        kept = int(m.sum())
        ratios.append(kept / (m.shape[0] * math.log2(T)))
        if prev is not None:
            growth.append(kept / prev)
        prev = kept
    assert all(g < 3.5 for g in growth), growth
    assert all(b < a for a, b in zip(growth, growth[1:])), growth
    assert growth[-1] < 2.45
    inc = np.diff(ratios)
    assert all(b < 0.95 * a for a, b in zip(inc, inc[1:])), ratios


def test_radial_density_at_500_frames_720p_reading():
    m = O.radial_block_mask_fast(126 * 45 * 80, 45 * 80, 128)
    density = m.mean()
    # The Radial explainer (section 4) reports 9x less attention compute at this
    # shape; the oracle's reading of the window constants gives 7.83x.  Record it.
    assert abs(density - 0.127768) < 1e-5
    assert 7.0 < 1.0 / density < 9.5


# ----------------------------------------------------------------- CSR

def test_mask_to_csr_matches_scipy():
    rng = np.random.default_rng(3)
    m = (rng.random((37, 53)) < 0.2).astype(np.uint8)
    m[5] = 0
    rp, ci = O.mask_to_csr(m)
    ref = scipy.sparse.csr_matrix(m)
    assert np.array_equal(rp, ref.indptr)
    assert np.array_equal(ci, ref.indices)
