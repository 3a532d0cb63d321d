"""GPU parity of the block-sparse attention kernel against the float64 oracle,
element by element, through the C ABI.  Sizes span several 128-row tiles and
ragged tails; masks cover empty rows, single kept blocks, per-head lists and
64/128/384-token blocks."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu


def run_case(Bn, H, nq, nk, D, bq, bk, mask, list_heads, seed, scale=0.0, qkv=None):
    if qkv is None:
        g = torch.Generator().manual_seed(seed)
        q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
        k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
        v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    else:
        q, k, v = qkv
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    o, lse, ws = B.bsa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), rp, ci, bq, bk, list_heads,
                                scale=scale)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    ro, rl = O.block_sparse_attention(to64(q), to64(k), to64(v), mask, bq, bk,
                                      scale=None if scale <= 0 else scale)
    og, lg = to64(o), lse.cpu().numpy().astype(np.float64)
    # O rows: [B, nq, H, D] -> rows (b, i, h); LSE [B, H, nq] -> same row order
    return assert_attention_close(og.reshape(-1, D), lg.transpose(0, 2, 1).reshape(-1),
                                  ro.reshape(-1, D), rl.transpose(0, 2, 1).reshape(-1))


def test_tiny_sta_all_ones_equals_dense():
    # 256 tokens, 64-token blocks, all-ones mask, head_dim 64: dense softmax attention
    mask = np.ones((1, 4, 4), np.uint8)
    run_case(1, 2, 256, 256, 64, 64, 64, mask, 1, seed=1)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bq,bk", [(128, 128), (64, 64), (384, 384), (64, 128), (256, 64)])
def test_random_masks_ragged(D, bq, bk):
    nq, nk = 5 * 128 + 37, 6 * 128 + 11
    Bn, H = 2, 2
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = synth.random_mask(Bn * H * QB, KB, 0.45, seed=bq + bk + D).reshape(Bn * H, QB, KB)
    mask[0, 0] = 0                       # empty row
    mask[1, -1] = 0
    mask[1, -1, -1] = 1                  # only the ragged last key block
    mask[2, 1] = 0
    mask[2, 1, 0] = 1                    # a single kept block
    run_case(Bn, H, nq, nk, D, bq, bk, mask, Bn * H, seed=D + bq)


def test_shared_list_across_heads_and_scale():
    nq = nk = 1000
    mask = synth.random_mask(8, 8, 0.5, seed=3).reshape(1, 8, 8)
    run_case(1, 3, nq, nk, 128, 128, 128, mask, 1, seed=4, scale=0.05)


def test_cross_attention_lengths():
    # fewer queries than keys (chunked decode shape), 64-token blocks
    nq, nk = 300, 2000
    QB, KB = math.ceil(nq / 64), math.ceil(nk / 64)
    mask = synth.random_mask(2 * QB, KB, 0.2, seed=5).reshape(2, QB, KB)
    mask[:, :, :3] = 1
    run_case(1, 2, nq, nk, 128, 64, 64, mask, 2, seed=6)


def test_large_logits_exercise_rescaling():
    # strongly peaked scores: the running max moves by much more than the lazy threshold
    nq, nk, D = 256, 1024, 128
    g = torch.Generator().manual_seed(9)
    q = (torch.randn(1, nq, 1, D, generator=g) * 4).to(torch.bfloat16)
    k = (torch.randn(1, nk, 1, D, generator=g) * 4).to(torch.bfloat16)
    # keys grow along the sequence so later tiles raise the row max
    k = (k.float() * torch.linspace(0.2, 1.5, nk).view(1, nk, 1, 1)).to(torch.bfloat16)
    v = torch.randn(1, nk, 1, D, generator=g).to(torch.bfloat16)
    mask = np.ones((1, 2, 8), np.uint8)
    run_case(1, 1, nq, nk, D, 128, 128, mask, 1, seed=0, qkv=(q, k, v))


@pytest.mark.parametrize("D", [64, 128])
def test_second_half_of_a_tile_jumps_above_the_running_max(D):
    # In every key tile after the first the keys of its second half (64..127) score
    # far above everything before them while its first half stays low: a tile's first
    # half passes the fast path's bound against the running max and its second half
    # does not, so the max moves in the middle of a tile.
    nq, nk = 256, 4 * 128
    g = torch.Generator().manual_seed(21)
    q = (torch.randn(1, nq, 1, D, generator=g) * 0.1 + 1.0).to(torch.bfloat16)
    k = torch.randn(1, nk, 1, D, generator=g) * 0.1
    level = torch.zeros(nk)
    for t in range(1, 4):
        level[128 * t + 64:128 * (t + 1)] = 1.2 * t     # scores jump by ~1.2 t * sqrt(D)
    k = (k + level.view(1, nk, 1, 1)).to(torch.bfloat16)
    v = torch.randn(1, nk, 1, D, generator=g).to(torch.bfloat16)
    mask = np.ones((1, 2, 4), np.uint8)
    run_case(1, 1, nq, nk, D, 128, 128, mask, 1, seed=0, qkv=(q, k, v))


def test_all_masked_everywhere():
    mask = np.zeros((1, 3, 3), np.uint8)
    run_case(1, 2, 300, 300, 128, 128, 128, mask, 1, seed=2)


def test_invalid_kept_list_is_reported_not_faulted():
    q = torch.randn(1, 256, 1, 128).to(torch.bfloat16).cuda()
    rp = torch.tensor([0, 2, 3], dtype=torch.int32).cuda()
    ci = torch.tensor([1, 0, 7, 0], dtype=torch.int32).cuda()  # descending row, out-of-range block
    o, lse, ws = B.bsa_attn_fwd(q, q, q, rp, ci, 128, 128, 1)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 1
