"""Head-partitioned path (the multi-GPU split, emulated on one GPU): heads are
independent given Q, K, V and the masks are per head, so a rank can run any
range of heads with no exchange.  Through the C ABI's token-row strides each
range is read in place from the whole-head tensors and written in place into a
whole-head output.  Checked here:
  - two plans over the two halves of the heads give, bit for bit, the output and
    LSE of one plan over all heads, for every mask family and a ragged grid;
  - the halves agree with the float64 oracle on sampled rows;
  - the attention forward and backward on strided views (head slices, Q/K/V of a
    fused projection) equal the same calls on dense copies, bit for bit."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import configs, synth
from block_sparse_attention_tokens_b200.pipeline import Plan, head_range
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu

W = configs.Workload
SMALL = [
    W(name="sta_small", index=11, batch=1, heads=4, head_dim=128, grid=(6, 8, 16), block=64,
      mask="sta", tile=(2, 4, 8), window=(3, 3, 1), strength=1.5),
    W(name="nabla_small", index=12, batch=1, heads=4, head_dim=128, grid=(5, 9, 14), block=64,
      mask="nabla", tile=(4, 4, 4), p=0.9, strength_range=(0.5, 3.0)),
    W(name="radial_small", index=13, batch=1, heads=3, head_dim=64, grid=(20, 6, 10), block=128,
      mask="radial", strength=2.0),
    W(name="ar_small", index=14, batch=1, heads=4, head_dim=128, grid=(24, 6, 10), block=64,
      mask="ar", p=0.85, strength=1.5, q_frames=3, anchor_frames=3, recent_frames=6),
    W(name="nabla_sta_small", index=15, batch=1, heads=2, head_dim=128, grid=(8, 8, 12), block=64,
      mask="nabla_sta", tile=(4, 4, 4), window=(3, 3, 3), p=0.9, strength_range=(0.5, 3.0)),
    W(name="spade_small", index=16, batch=1, heads=4, head_dim=128, grid=(6, 10, 12), block=64,
      mask="spade", p=0.9, strength_range=(1.0, 3.0), extra={"axis_stretch": 6.0}),
    # 128-token slices (2x8x8, 1x8x16, 4x4x8, 32x2x2) on a ragged grid, head_dim 64
    W(name="spade128_small", index=17, batch=1, heads=3, head_dim=64, grid=(9, 12, 20), block=128,
      mask="spade", p=0.85, strength_range=(1.0, 3.0), extra={"axis_stretch": 6.0}),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_head_halves_equal_the_whole_and_the_oracle(w):
    q, k, v, _ = synth.workload_inputs(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    whole = Plan(w)
    o_ref, lse_ref = whole.step(qc, kc, vc)
    o_ref, lse_ref = o_ref.clone(), lse_ref.clone()
    out = torch.full_like(o_ref, float("nan"))
    lses = []
    for r in range(2):
        h0, h1 = head_range(r, 2, w.heads)
        part = Plan(w, heads=(h0, h1))
        part.step(qc, kc, vc, out=out)           # whole-head tensors, read and written in place
        torch.cuda.synchronize()
        assert B.bsa_read_status(part.attn_ws) == 0
        if whole.list_heads > 1:
            assert torch.equal(part.mask, whole.mask[:, h0:h1]), "per-head masks differ"
        lses.append(part.lse.clone())
    assert torch.equal(out, o_ref), "head halves differ from the whole call"
    assert torch.equal(torch.cat(lses, dim=1), lse_ref)
    # the oracle on sampled rows of the first head of each half (path token order)
    from tests.test_gpu_workloads import check_spade_choice, head_perms, oracle_mask
    if w.mask == "spade":
        check_spade_choice(w, whole, q, k)
    ref_mask, near = oracle_mask(w, whole, q, k)
    op = (whole.op if whole.permuted else whole.o).cpu()
    rows = np.unique(np.r_[0, w.nq - 1, np.random.default_rng(w.seed).integers(0, w.nq, 24)])
    perms = head_perms(w, whole)
    for h in (0, head_range(1, 2, w.heads)[0]):
        perm = perms[h]
        hm = 0 if ref_mask.shape[0] == 1 else h
        keep = rows if near is None else rows[~near[hm, rows // w.block]]
        qh, kh, vh = (to64(t[:, :, h:h + 1]) for t in (q, k, v))
        if perm is not None:
            qh, kh, vh = (O.tile_permute(t, perm, whole.n_pad) for t in (qh, kh, vh))
            qh, kh, vh = qh[:, :w.nq], kh[:, :w.nk], vh[:, :w.nk]
        if not np.array_equal(whole.mask.cpu().numpy().reshape(-1, whole.QB, whole.KB)[hm],
                              ref_mask[hm]):
            continue                              # a NABLA row decided within 1e-5 of p
        ro, rl = O.block_sparse_attention(qh, kh, vh, ref_mask[hm:hm + 1], w.block, w.block,
                                          rows=keep)
        assert_attention_close(to64(op[0, keep, h]), lse_ref.cpu().numpy()[0, h, keep]
                               .astype(np.float64), ro[0, keep, 0], rl[0, 0, keep],
                               what=f"{w.name} head {h}")


def _dense(t):
    return t.contiguous()


@pytest.mark.parametrize("D,bq,bk", [(128, 128, 128), (64, 64, 64), (128, 384, 384)])
def test_strided_views_equal_dense_copies_forward_and_backward(D, bq, bk):
    g = torch.Generator().manual_seed(D + bq)
    Bn, H, n = 2, 3, 5 * 128 + 29
    qkv = torch.randn(Bn, n, 3, H + 2, D, generator=g).to(torch.bfloat16).cuda()
    # Q, K, V of a fused projection, heads 1..H of H + 2: rows 3 * (H + 2) * D apart
    q, k, v = (qkv[:, :, i, 1:H + 1] for i in range(3))
    QB, KB = math.ceil(n / bq), math.ceil(n / bk)
    mask = synth.random_mask(Bn * H * QB, KB, 0.5, seed=D).reshape(Bn * H, QB, KB)
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    o_wide = torch.zeros(Bn, n, H + 3, D, dtype=torch.bfloat16, device="cuda")
    o_s = o_wide[:, :, 2:H + 2]
    _, lse_s, ws = B.bsa_attn_fwd(q, k, v, rp, ci, bq, bk, Bn * H, o=o_s)
    o_d, lse_d, _ = B.bsa_attn_fwd(_dense(q), _dense(k), _dense(v), rp, ci, bq, bk, Bn * H)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    assert torch.equal(o_s, o_d) and torch.equal(lse_s, lse_d)
    assert torch.all(o_wide[:, :, :2] == 0) and torch.all(o_wide[:, :, H + 2:] == 0)
    # backward: gradients into a fused dQKV buffer, dO a head slice of a tensor as wide as O's
    do_wide = torch.randn(Bn, n, H + 3, D, generator=g).to(torch.bfloat16).cuda()
    do = do_wide[:, :, 2:H + 2]                     # same row stride as o
    dqkv = torch.zeros_like(qkv)
    dq, dk, dv = (dqkv[:, :, i, 1:H + 1] for i in range(3))
    _, _, _, bws = B.bsa_attn_bwd(q, k, v, o_s, do, lse_s, rp, ci, bq, bk, Bn * H, dq=dq, dk=dk,
                                  dv=dv)
    rq, rk, rv, _ = B.bsa_attn_bwd(_dense(q), _dense(k), _dense(v), o_d, _dense(do), lse_d, rp, ci,
                                   bq, bk, Bn * H)
    torch.cuda.synchronize()
    assert B.bsa_read_status(bws) == 0
    assert torch.equal(dq, rq) and torch.equal(dk, rk) and torch.equal(dv, rv)
    assert torch.all(dqkv[:, :, :, 0] == 0) and torch.all(dqkv[:, :, :, H + 1] == 0)


def test_strided_nabla_mask_and_permutes_equal_dense_copies():
    w = SMALL[1]
    q, k, _, _ = synth.generate(1, 6, 128, w.grid, 77, strength_range=(0.5, 3.0))
    qc, kc = q.cuda(), k.cuda()
    qs, ks = qc[:, :, 2:5], kc[:, :, 2:5]
    m_s, _ = B.bsa_nabla_mask(qs, ks, 64, 0.9)
    m_d, _ = B.bsa_nabla_mask(_dense(qs), _dense(ks), 64, 0.9)
    assert torch.equal(m_s, m_d)
    n_pad = math.ceil(w.n_tokens / 64) * 64
    wide = torch.zeros(1, n_pad, 7, 128, dtype=torch.bfloat16, device="cuda")
    y_s = wide[:, :, 1:4]
    B.bsa_tile_permute(qs, w.grid, w.tile, n_pad, y=y_s)
    y_d = B.bsa_tile_permute(_dense(qs), w.grid, w.tile, n_pad)
    assert torch.equal(y_s, y_d) and torch.all(wide[:, :, 4:] == 0)
    yp_s, pool_s = B.bsa_tile_permute_pool(ks, w.grid, w.tile, n_pad, 64)
    yp_d, pool_d = B.bsa_tile_permute_pool(_dense(ks), w.grid, w.tile, n_pad, 64)
    assert torch.equal(yp_s, yp_d) and torch.equal(pool_s, pool_d)
    back = torch.zeros(1, w.n_tokens, 6, 128, dtype=torch.bfloat16, device="cuda")
    B.bsa_tile_untile(y_s, w.grid, w.tile, x=back[:, :, 2:5])
    assert torch.equal(back[:, :, 2:5], qs) and torch.all(back[:, :, :2] == 0)


@pytest.mark.parametrize("name", ["radial_small", "ar_small"])
def test_query_block_halves_equal_the_whole(name):
    # the split for raster-order workloads whose heads do not divide over the ranks:
    # each of two plans takes half of the query blocks of every head (all keys),
    # reading its rows of Q and writing its rows of O in place
    from block_sparse_attention_tokens_b200.pipeline import qblock_range
    w = next(x for x in SMALL if x.name == name)
    q, k, v, _ = synth.workload_inputs(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    whole = Plan(w)
    o_ref, lse_ref = whole.step(qc, kc, vc)
    o_ref, lse_ref = o_ref.clone(), lse_ref.clone()
    QB = math.ceil(w.nq / w.block)
    out = torch.full_like(o_ref, float("nan"))
    lses = []
    for r in range(2):
        b0, b1 = qblock_range(r, 2, QB, granule=max(1, 128 // w.block))
        part = Plan(w, qblocks=(b0, b1))
        part.step(qc, kc, vc, out=out)
        torch.cuda.synchronize()
        assert B.bsa_read_status(part.attn_ws) == 0
        assert part.nq == min(w.nq, b1 * w.block) - b0 * w.block
        if whole.list_heads > 1:
            assert torch.equal(part.mask, whole.mask[:, :, b0:b1]), "per-head masks differ"
        lses.append(part.lse.clone())
    assert torch.equal(out, o_ref), "query-block halves differ from the whole call"
    assert torch.equal(torch.cat(lses, dim=2), lse_ref)


def test_query_block_range_needs_a_raster_workload():
    w = next(x for x in SMALL if x.name == "sta_small")
    with pytest.raises(ValueError):
        Plan(w, qblocks=(0, 1))


@pytest.mark.parametrize("name", ["sta_small", "nabla_small", "radial_small", "ar_small",
                                  "spade_small"])
def test_cuda_graph_replay_equals_eager_steps(name):
    # the whole path captured once into a CUDA graph: a replay gives the eager
    # step's O and LSE bit for bit, also after new inputs are copied in place
    w = next(x for x in SMALL if x.name == name)
    q, k, v, _ = synth.workload_inputs(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    eager = Plan(w)
    o1, l1 = (t.clone() for t in eager.step(qc, kc, vc))
    q2 = torch.flip(q, dims=[1]).contiguous().cuda()
    o2, l2 = (t.clone() for t in eager.step(q2, kc, vc))
    plan = Plan(w)
    qs = qc.clone()
    graph = plan.capture(qs, kc, vc)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(plan.out, o1) and torch.equal(plan.lse, l1)
    qs.copy_(q2)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(plan.out, o2) and torch.equal(plan.lse, l2)
    assert B.bsa_read_status(plan.attn_ws) == 0
