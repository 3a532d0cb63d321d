"""GPU parity of the bandwidth kernels (permute, static masks, NABLA, compaction)
against the CPU oracle, through the C ABI.  Integer/byte results must be
bit-exact; NABLA rows the oracle marks as near the threshold are exempt."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("grid,tile,block", [((4, 8, 8), (4, 4, 4), 64), ((21, 30, 52), (4, 4, 4), 64),
                                             ((5, 7, 3), (2, 3, 2), 16), ((30, 48, 80), (6, 8, 8), 384),
                                             ((1, 1, 9), (1, 1, 4), 16)])
def test_tile_permute_and_untile_bit_exact(grid, tile, block):
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    heads, d = (2, 64) if n < 50000 else (1, 64)
    x = torch.randn(2, n, heads, d).to(torch.bfloat16)
    perm = O.tile_order(grid, tile)
    ref = O.tile_permute(_bits(x), perm, n_pad)
    y = B.bsa_tile_permute(x.cuda(), grid, tile, n_pad)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), ref)
    back = B.bsa_tile_untile(y, grid, tile)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(back), _bits(x))


@pytest.mark.parametrize("tile_grid,window", [((5, 6, 10), (3, 3, 5)), ((1, 2, 2), (1, 3, 3)),
                                              ((3, 4, 5), (3, 1, 5)), ((7, 3, 9), (5, 3, 3)),
                                              ((2, 5, 4), (4, 2, 3))])
@pytest.mark.parametrize("shift", [0, 1])
def test_sta_mask_bit_exact(tile_grid, window, shift):
    m = B.bsa_sta_mask(tile_grid, window, shift)
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), O.sta_tile_mask(tile_grid, window, bool(shift)))


@pytest.mark.parametrize("n,S,blk", [(16 * 12, 16, 4), (9 * 6 - 4, 6, 8), (33 * 4, 4, 8),
                                     (64 * 40, 64, 16), (126 * 45 * 80, 45 * 80, 128)])
def test_radial_mask_bit_exact(n, S, blk):
    m = B.bsa_radial_mask(n, S, blk)
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), O.radial_block_mask_fast(n, S, blk))


@pytest.mark.parametrize("rows,kb,density", [(1, 1, 1.0), (37, 53, 0.2), (300, 300, 0.1),
                                             (40 * 64, 512, 0.3), (5, 1463, 0.05)])
def test_mask_compact_bit_exact(rows, kb, density):
    m = synth.random_mask(rows, kb, density, seed=rows + kb)
    if rows > 3:
        m[2] = 0
        m[3] = 1
    rp, ci = B.bsa_mask_compact(torch.from_numpy(m).cuda())
    torch.cuda.synchronize()
    ref_rp, ref_ci = O.mask_to_csr(m)
    assert np.array_equal(rp.cpu().numpy(), ref_rp)
    nnz = int(ref_rp[-1])
    assert np.array_equal(ci.cpu().numpy()[:nnz], ref_ci)


def _nabla_reference(q, k, nq, nk, block, p, kb_begin=0, kb_end=None, force_outside=0):
    qf, kf = q.double().numpy(), k.double().numpy()
    QB = math.ceil(nq / block)
    KB = math.ceil(nk / block)
    qpad = np.zeros((qf.shape[0], QB * block) + qf.shape[2:])
    qpad[:, :nq] = qf[:, :nq]
    kpad = np.zeros((kf.shape[0], KB * block) + kf.shape[2:])
    kpad[:, :nk] = kf[:, :nk]
    qbar = O.nabla_pool(qpad, block, nq)
    kbar = O.nabla_pool(kpad, block, nk)
    D = q.shape[-1]
    return O.nabla_mask(qbar, kbar, p, 1.0 / math.sqrt(D), kb_begin,
                        KB if kb_end is None else kb_end, force_outside)


def _assert_nabla_equal(gpu_mask, ref_mask, near, max_near_frac=0.05):
    g = gpu_mask.cpu().numpy()
    diff_rows = np.any(g != ref_mask, axis=-1)
    bad = diff_rows & ~near
    assert not bad.any(), f"{int(bad.sum())} NABLA rows differ away from the threshold"
    assert near.mean() <= max_near_frac


@pytest.mark.parametrize("nq,nk,heads,d,block,p", [(1000, 1000, 2, 64, 64, 0.9),
                                                   (513, 2047, 3, 128, 64, 0.5),
                                                   (4096, 4096, 2, 128, 128, 0.97),
                                                   (640, 640, 1, 128, 32, 0.3)])
def test_nabla_mask_matches_oracle(nq, nk, heads, d, block, p):
    T = 8
    q, k, _, _ = synth.generate(1, heads, d, (T, 1, nk // T + 1), seed=nq + nk,
                                strength_range=(0.5, 3.0))
    q, k = q[:, :nq].contiguous(), k[:, :nk].contiguous()
    mask, near_gpu = B.bsa_nabla_mask(q.cuda(), k.cuda(), block, p)
    torch.cuda.synchronize()
    ref, near = _nabla_reference(q, k, nq, nk, block, p)
    _assert_nabla_equal(mask, ref, near)


def test_nabla_mask_forced_ranges_and_uniform_ties():
    # AR-style composition: blocks outside [kb_begin, kb_end) forced on
    q, k, _, _ = synth.generate(1, 2, 128, (12, 4, 40), seed=77, strength=1.5,
                                q_token_ids=np.arange(9 * 160, 12 * 160))
    nq, nk = q.shape[1], k.shape[1]
    mask, _ = B.bsa_nabla_mask(q.cuda(), k.cuda(), 64, 0.85, 0.0, 5, 24, 1)
    torch.cuda.synchronize()
    ref, near = _nabla_reference(q, k, nq, nk, 64, 0.85, 5, 24, 1)
    _assert_nabla_equal(mask, ref, near)
    # identical keys -> uniform probabilities -> exactly ceil(p * KB) lowest-index blocks
    kc = torch.ones(1, 1024, 1, 64, dtype=torch.bfloat16)
    qc = torch.randn(1, 256, 1, 64).to(torch.bfloat16)
    mask, _ = B.bsa_nabla_mask(qc.cuda(), kc.cuda(), 64, 0.9)
    torch.cuda.synchronize()
    m = mask.cpu().numpy()[0, 0]
    assert np.all(m[:, :15] == 1) and np.all(m[:, 15:] == 0)   # ceil(0.9 * 16) = 15


def test_nabla_p_one_keeps_everything():
    q = torch.randn(1, 300, 2, 64).to(torch.bfloat16).cuda()
    k = torch.randn(1, 500, 2, 64).to(torch.bfloat16).cuda()
    mask, _ = B.bsa_nabla_mask(q, k, 64, 1.0)
    torch.cuda.synchronize()
    assert torch.all(mask == 1)


@pytest.mark.parametrize("grid,tile,block,heads,d", [((21, 30, 52), (4, 4, 4), 64, 3, 128),
                                                     ((5, 7, 3), (2, 3, 2), 16, 2, 64),
                                                     ((20, 32, 52), (4, 4, 4), 64, 2, 128)])
def test_tile_permute_pool_bit_exact_rows_and_means(grid, tile, block, heads, d):
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    x = torch.randn(2, n, heads, d).to(torch.bfloat16)
    perm = O.tile_order(grid, tile)
    y, pooled = B.bsa_tile_permute_pool(x.cuda(), grid, tile, n_pad, block)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), O.tile_permute(_bits(x), perm, n_pad))
    ref = O.nabla_pool(O.tile_permute(x.double().numpy(), perm, n_pad), block, n)
    got = pooled.cpu().double().numpy()
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) < 2e-5        # fp32 sums of <= block bf16 values


def test_nabla_select_with_sta_base_mask_matches_oracle():
    w_grid, tile, block, window = (8, 16, 16), (4, 4, 4), 64, (3, 3, 3)
    n = w_grid[0] * w_grid[1] * w_grid[2]
    q, k, _, _ = synth.generate(1, 3, 128, w_grid, seed=31, strength_range=(0.5, 3.0))
    perm = O.tile_order(w_grid, tile)
    qp, qbar = B.bsa_tile_permute_pool(q.cuda(), w_grid, tile, n, block)
    kp, kbar = B.bsa_tile_permute_pool(k.cuda(), w_grid, tile, n, block)
    tg = tuple(g // t for g, t in zip(w_grid, tile))
    base = B.bsa_sta_mask(tg, window)
    mask, _ = B.bsa_nabla_select(qbar, kbar, 0.7, base_mask=base)
    torch.cuda.synchronize()
    rq = O.nabla_pool(O.tile_permute(q.double().numpy(), perm, n), block, n)
    rk = O.nabla_pool(O.tile_permute(k.double().numpy(), perm, n), block, n)
    ref, near = O.nabla_sta_mask(rq, rk, 0.7, 1 / math.sqrt(128), O.sta_tile_mask(tg, window))
    _assert_nabla_equal(mask, ref, near)
    m = mask.cpu().numpy()
    assert np.all(m >= O.sta_tile_mask(tg, window)[None, None])
