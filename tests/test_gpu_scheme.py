"""GPU parity of the per-head slicing permute (SPADE summary, solution parts 1 and
3) against the CPU oracle, through the C ABI: rows bit-exact, block means within
fp32 summation error, the inverse bit-exact, a choice outside the menu reported."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import configs

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy()


def _choices(batch, heads, n_shapes, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, n_shapes, size=(batch, heads)).astype(np.int32)
    c.reshape(-1)[: min(n_shapes, c.size)] = np.arange(min(n_shapes, c.size))   # every shape used
    return c


@pytest.mark.parametrize("grid,block,heads,d", [((5, 9, 7), 64, 6, 64), ((21, 30, 52), 64, 3, 128),
                                                ((4, 8, 8), 64, 4, 128), ((3, 5, 11), 16, 5, 128),
                                                ((1, 1, 9), 64, 2, 64)])
def test_scheme_permute_rows_means_and_inverse(grid, block, heads, d):
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    menu = configs.sics_menu(64)
    x = torch.randn(2, n, heads, d).to(torch.bfloat16)
    c = _choices(2, heads, len(menu), seed=n + heads)
    choice = torch.from_numpy(c).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, pooled = B.bsa_scheme_permute(x.cuda(), grid, menu, choice, n_pad, block, pool=True,
                                     device_status=status)
    y2, none = B.bsa_scheme_permute(x.cuda(), grid, menu, choice, n_pad, device_status=status)
    torch.cuda.synchronize()
    assert none is None and int(status.item()) == 0
    ref = O.scheme_permute(_bits(x), grid, menu, c, n_pad)
    assert np.array_equal(_bits(y), ref)
    assert np.array_equal(_bits(y2), ref)
    refp = np.zeros((2, heads, n_pad // block, d))
    xd = x.double().numpy()
    yd = O.scheme_permute(xd, grid, menu, c, n_pad)
    for h in range(heads):
        refp[:, h] = O.nabla_pool(yd[:, :, h:h + 1], block, n)[:, 0]
    assert np.max(np.abs(pooled.cpu().double().numpy() - refp)) < 2e-5
    back = B.bsa_scheme_untile(y, grid, menu, choice, device_status=status)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(back), _bits(x))
    assert np.array_equal(_bits(back), O.scheme_untile(_bits(y), grid, menu, c))
    assert int(status.item()) == 0


def test_scheme_permute_uniform_choice_equals_tile_permute():
    grid, block, heads, d = (21, 30, 52), 64, 4, 128
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    menu = configs.sics_menu(64)
    x = torch.randn(1, n, heads, d).to(torch.bfloat16).cuda()
    for s, shape in enumerate(menu):
        choice = torch.full((1, heads), s, dtype=torch.int32, device="cuda")
        y, pooled = B.bsa_scheme_permute(x, grid, menu, choice, n_pad, block, pool=True)
        yt, pt = B.bsa_tile_permute_pool(x, grid, shape, n_pad, block)
        torch.cuda.synchronize()
        assert torch.equal(y, yt), shape
        assert torch.allclose(pooled, pt, rtol=0, atol=2e-6), shape


def test_scheme_permute_on_head_slices_in_place():
    # a range of heads of a wider tensor, through the token-row stride, writing its
    # heads of a wider output
    grid, block, d = (6, 10, 12), 64, 128
    n = grid[0] * grid[1] * grid[2]
    n_pad = math.ceil(n / block) * block
    menu = configs.sics_menu(64)
    x = torch.randn(1, n, 8, d).to(torch.bfloat16).cuda()
    c = _choices(1, 8, len(menu), seed=7)
    choice = torch.from_numpy(c).cuda()
    whole, _ = B.bsa_scheme_permute(x, grid, menu, choice, n_pad)
    y = torch.zeros(1, n_pad, 8, d, dtype=torch.bfloat16, device="cuda")
    back = torch.zeros_like(x)
    for h0, h1 in ((0, 3), (3, 8)):
        part = choice[:, h0:h1].contiguous()
        B.bsa_scheme_permute(x[:, :, h0:h1], grid, menu, part, n_pad, y=y[:, :, h0:h1])
        B.bsa_scheme_untile(y[:, :, h0:h1], grid, menu, part, x=back[:, :, h0:h1])
    torch.cuda.synchronize()
    assert torch.equal(y, whole)
    assert torch.equal(back, x)


def test_choice_outside_the_menu_is_reported_and_zeroed():
    grid, block, heads, d = (4, 8, 8), 64, 3, 64
    n = 256
    menu = configs.sics_menu(64)
    x = torch.randn(1, n, heads, d).to(torch.bfloat16).cuda()
    choice = torch.tensor([[0, 7, 1]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, pooled = B.bsa_scheme_permute(x, grid, menu, choice, n, block, pool=True,
                                     device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1                    # BSA_ERR_INVALID_ARG
    assert not y[:, :, 1].any() and not pooled[:, 1].any()
    c = np.array([[0, 0, 1]])
    ref = O.scheme_permute(_bits(x.cpu()), grid, menu, c, n)
    assert np.array_equal(_bits(y)[:, :, [0, 2]], ref[:, :, [0, 2]])
    status.zero_()
    back = B.bsa_scheme_untile(y, grid, menu, choice, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert not back[:, :, 1].any()
    assert torch.equal(back[:, :, 0], x[:, :, 0]) and torch.equal(back[:, :, 2], x[:, :, 2])
