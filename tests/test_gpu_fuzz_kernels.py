"""Seeded random configurations of the permute, mask, compaction and SICS kernels
against the oracle: integer and byte results bit-exact, SICS within its derived
tolerance (4e-5 * n^2 per block, see tests/test_gpu_sics.py)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from tests._parity import to64

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("seed", range(16))
def test_random_permute_untile(seed):
    rng = np.random.default_rng(700 + seed)
    grid = tuple(int(x) for x in rng.integers(1, 17, size=3))
    tile = tuple(int(rng.integers(1, g + 1)) for g in grid)
    block = int(rng.choice([16, 64, 128]))
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    heads, d = int(rng.integers(1, 4)), int(rng.choice([64, 128]))
    x = torch.randn(int(rng.integers(1, 3)), n, heads, d,
                    generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    perm = O.tile_order(grid, tile)
    y = B.bsa_tile_permute(x.cuda(), grid, tile, n_pad)
    back = B.bsa_tile_untile(y, grid, tile)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), O.tile_permute(_bits(x), perm, n_pad))
    assert np.array_equal(_bits(back), _bits(x))


@pytest.mark.parametrize("seed", range(16))
def test_random_sta_and_radial_masks(seed):
    rng = np.random.default_rng(800 + seed)
    tg = tuple(int(x) for x in rng.integers(1, 12, size=3))
    window = tuple(int(2 * rng.integers(0, 4) + 1) for _ in range(3))
    shift = int(rng.integers(0, 2))
    m = B.bsa_sta_mask(tg, window, shift)
    S = int(rng.integers(2, 200))
    frames = int(rng.integers(1, 40))
    blk = int(rng.choice([4, 16, 64, 128]))
    n = S * frames - int(rng.integers(0, S))
    r = B.bsa_radial_mask(n, S, blk)
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), O.sta_tile_mask(tg, window, bool(shift)))
    assert np.array_equal(r.cpu().numpy(), O.radial_block_mask_fast(n, S, blk))


@pytest.mark.parametrize("seed", range(16))
def test_random_compaction(seed):
    rng = np.random.default_rng(900 + seed)
    rows, kb = int(rng.integers(1, 600)), int(rng.integers(1, 2000))
    m = (rng.random((rows, kb)) < rng.uniform(0.0, 1.0)).astype(np.uint8)
    rp, ci = B.bsa_mask_compact(torch.from_numpy(m).cuda())
    torch.cuda.synchronize()
    ref_rp, ref_ci = O.mask_to_csr(m)
    assert np.array_equal(rp.cpu().numpy(), ref_rp)
    assert np.array_equal(ci.cpu().numpy()[:int(ref_rp[-1])], ref_ci)


@pytest.mark.parametrize("seed", range(8))
def test_random_sics_blocks(seed):
    rng = np.random.default_rng(1000 + seed)
    grid = tuple(int(x) for x in rng.integers(1, 13, size=3))
    tile = tuple(int(rng.integers(1, 9)) for _ in range(3))
    heads, d = int(rng.integers(1, 5)), int(rng.choice([64, 128]))
    n = grid[0] * grid[1] * grid[2]
    x = torch.randn(int(rng.integers(1, 3)), n, heads, d,
                    generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    got = B.bsa_sics_blocks(x.cuda(), grid, tile).cpu().double().numpy()
    torch.cuda.synchronize()
    ref = O.sics_blocks(to64(x), grid, tile)
    nt = ref.shape[2]
    nb = np.array([len(O.tile_tokens(grid, tile, t)) for t in range(nt)], dtype=np.float64)
    assert np.all(np.abs(got - ref) <= 4e-5 * nb[None, None, :] ** 2)
