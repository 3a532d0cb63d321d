"""GPU parity of SPADE scheme generation (SICS per block, per-head slicing choice)
against the float64 oracle, through the C ABI.

Tolerance, derived from the kernel's arithmetic: the bf16 inputs are exact in
both paths; each token is normalised in fp32 (a sum of head_dim squares and an
rsqrt: relative error below 1e-5 for head_dim <= 128), n such unit vectors are
summed in fp32 and the squared norm taken, so a block's SICS (at most n^2) is off
by at most about 2 * n^2 * 1e-5.  The test allows 4e-5 * n^2 per block, and the
scores (SICS / n^2 averages) 4e-5.  The choice (an argmax of floats) must equal
the oracle's unless the oracle's two best scores are within 1e-4; then it must be
one of those."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import configs, synth
from tests._parity import to64

pytestmark = pytest.mark.gpu


def block_sizes(grid, tile):
    nt = 1
    for g, t in zip(grid, tile):
        nt *= -(-g // t)
    return np.array([len(O.tile_tokens(grid, tile, i)) for i in range(nt)], dtype=np.float64)


@pytest.mark.parametrize("grid,tile,heads,D", [((5, 7, 9), (2, 3, 4), 3, 64),
                                               ((4, 8, 8), (4, 4, 4), 2, 128),
                                               ((21, 30, 52), (16, 2, 2), 2, 128),
                                               ((3, 10, 6), (1, 8, 8), 5, 128),
                                               ((2, 3, 3), (2, 3, 3), 1, 64)])
def test_sics_blocks_match_oracle(grid, tile, heads, D):
    n = grid[0] * grid[1] * grid[2]
    g = torch.Generator().manual_seed(n + heads)
    x = torch.randn(2, n, heads, D, generator=g).to(torch.bfloat16)
    x[0, 1] = 0                                    # zero vectors contribute nothing
    got = B.bsa_sics_blocks(x.cuda(), grid, tile).cpu().double().numpy()
    torch.cuda.synchronize()
    ref = O.sics_blocks(to64(x), grid, tile)
    nb = block_sizes(grid, tile)
    assert got.shape == ref.shape
    assert np.all(np.abs(got - ref) <= 4e-5 * nb[None, None, :] ** 2)


def test_structured_fields_choose_the_oracle_shape():
    grid, D = (16, 8, 8), 128
    T, H, W = grid
    rng = np.random.default_rng(5)
    x = np.zeros((1, T * H * W, 2, D), dtype=np.float32)
    sp = rng.standard_normal((H * W, D))
    fr = rng.standard_normal((T, D))
    for n in range(T * H * W):
        x[0, n, 0] = sp[n % (H * W)]              # head 0: constant along time
        x[0, n, 1] = fr[n // (H * W)]             # head 1: constant within a frame
    xt = torch.from_numpy(x).to(torch.bfloat16)
    menu = configs.sics_menu(64)
    scores, choice, _ = B.bsa_sics_scheme(xt.cuda(), xt.cuda(), grid, menu)
    torch.cuda.synchronize()
    rs, rc = O.sics_scheme(to64(xt), to64(xt), grid, menu)
    assert np.all(np.abs(scores.cpu().double().numpy() - rs) <= 4e-5)
    assert choice.cpu().tolist() == rc.tolist() == [[3, 1]]


def _assert_choice(choice, rs, rc):
    for b in range(rs.shape[0]):
        for h in range(rs.shape[1]):
            order = np.argsort(-rs[b, h], kind="stable")
            if rs[b, h, order[0]] - rs[b, h, order[1]] < 1e-4:
                near = [s for s in range(rs.shape[2]) if rs[b, h, order[0]] - rs[b, h, s] < 1e-4]
                assert choice[b, h] in near
            else:
                assert choice[b, h] == rc[b, h]


def test_scheme_on_the_480p_nabla_workload():
    # the NABLA 480p workload at full size: 40 heads x 128, 21x30x52 tokens, 64-token menu
    w = configs.get("nabla_480p")
    q, k, _, _ = synth.workload_inputs(w)
    menu = configs.sics_menu(w.block)
    scores, choice, _ = B.bsa_sics_scheme(q.cuda(), k.cuda(), w.grid, menu)
    torch.cuda.synchronize()
    rs, rc = O.sics_scheme(to64(q), to64(k), w.grid, menu)
    got = scores.cpu().double().numpy()
    assert np.all(np.abs(got - rs) <= 4e-5)
    _assert_choice(choice.cpu().numpy(), rs, rc)
