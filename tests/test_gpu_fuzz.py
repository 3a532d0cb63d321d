"""Seeded random configurations of the attention forward, backward and paged
forward against the float64 oracle: lengths from a single token to several tiles
with ragged tails, every block-size pair, both head sizes, shared and per-head
kept lists, random densities and scales, random page tables with evictions.
Tolerances as in the dedicated tests (forward: O max-abs 2e-2 / mean-abs 2e-3,
LSE 1e-3; backward: the per-entry envelope of tests/test_gpu_backward.py)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from tests._parity import assert_attention_close, to64
from tests.test_gpu_backward import assert_grad_close, envelopes

pytestmark = pytest.mark.gpu

BLOCKS = (64, 128, 256, 384)


def random_case(seed):
    rng = np.random.default_rng(seed)
    Bn, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    D = int(rng.choice([64, 128]))
    bq, bk = int(rng.choice(BLOCKS)), int(rng.choice(BLOCKS))
    nq = int(rng.choice([1, 7, 64, 65, 127, 128, 129, int(rng.integers(130, 900))]))
    nk = int(rng.choice([1, 5, 64, 100, 128, 200, int(rng.integers(200, 1000))]))
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    shared = bool(rng.integers(0, 2))
    Hm = 1 if shared else Bn * H
    mask = (rng.random((Hm, QB, KB)) < rng.uniform(0.2, 0.9)).astype(np.uint8)
    scale = float(rng.choice([0.0, 0.05, 0.2]))
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    return Bn, H, D, bq, bk, nq, nk, mask, Hm, scale, q, k, v


@pytest.mark.parametrize("seed", range(32))
def test_random_forward_and_backward(seed):
    Bn, H, D, bq, bk, nq, nk, mask, Hm, scale, q, k, v = random_case(100 + seed)
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    o, lse, ws = B.bsa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), rp, ci, bq, bk, Hm, scale=scale)
    do = torch.randn(Bn, nq, H, D, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    dq, dk, dv, bws = B.bsa_attn_bwd(q.cuda(), k.cuda(), v.cuda(), o, do.cuda(), lse, rp, ci, bq, bk,
                                     Hm, scale=scale)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0 and B.bsa_read_status(bws) == 0
    sc = 1.0 / math.sqrt(D) if scale <= 0 else scale
    q64, k64, v64, do64 = to64(q), to64(k), to64(v), to64(do)
    ro, rl = O.block_sparse_attention(q64, k64, v64, mask, bq, bk, scale=sc)
    assert_attention_close(to64(o).reshape(-1, D),
                           lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1).reshape(-1),
                           ro.reshape(-1, D), rl.transpose(0, 2, 1).reshape(-1),
                           what=f"seed {seed} forward")
    rdq, rdk, rdv = O.block_sparse_attention_backward(q64, k64, v64, do64, mask, bq, bk, scale=sc)
    eq, ek, ev = envelopes(q64, k64, v64, do64, ro, rl, mask, bq, bk, sc)
    assert_grad_close(to64(dq), rdq, eq, f"seed {seed} dQ")
    assert_grad_close(to64(dk), rdk, ek, f"seed {seed} dK")
    assert_grad_close(to64(dv), rdv, ev, f"seed {seed} dV")


@pytest.mark.parametrize("seed", range(12))
def test_random_paged_forward(seed):
    rng = np.random.default_rng(500 + seed)
    Bn, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    D = int(rng.choice([64, 128]))
    bk = int(rng.choice([64, 128]))
    bq = int(rng.choice(BLOCKS))
    nq, nk = int(rng.integers(1, 400)), int(rng.integers(1, 1500))
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = (rng.random((Bn * H, QB, KB)) < 0.6).astype(np.uint8)
    n_pages = math.ceil(nk / B.KV_PAGE)
    n_pool = Bn * n_pages + 2
    table = rng.permutation(n_pool)[:Bn * n_pages].reshape(Bn, n_pages).astype(np.int32)
    table[rng.random(table.shape) < 0.25] = -1
    g = torch.Generator().manual_seed(600 + seed)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    kp = torch.randn(n_pool, B.KV_PAGE, H, D, generator=g).to(torch.bfloat16)
    vp = torch.randn(n_pool, B.KV_PAGE, H, D, generator=g).to(torch.bfloat16)
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    o, lse, ws = B.bsa_attn_fwd_paged(q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(table).cuda(),
                                      nk, rp, ci, bq, bk, Bn * H)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    ro, rl = O.paged_block_sparse_attention(to64(q), to64(kp), to64(vp), table, B.KV_PAGE, nk, mask,
                                            bq, bk)
    assert_attention_close(to64(o).reshape(-1, D),
                           lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1).reshape(-1),
                           ro.reshape(-1, D), rl.transpose(0, 2, 1).reshape(-1),
                           what=f"paged seed {seed}")
