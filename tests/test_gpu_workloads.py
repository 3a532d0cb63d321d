"""Whole-path parity at the full workload sizes (the launch configuration the
benchmark times): masks bit-exact against the oracle (NABLA rows near the
threshold exempt), attention on sampled rows against the float64 oracle, and the
inverse permute bit-exact."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import configs, synth
from block_sparse_attention_tokens_b200.pipeline import Plan
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu


def sample_blocks(nblocks: int, count: int, seed: int):
    rng = np.random.default_rng(seed)
    picks = {0, nblocks - 1, nblocks // 2}
    picks.update(int(x) for x in rng.choice(nblocks, size=min(nblocks, count), replace=False))
    return sorted(picks)


def sample_rows_in_blocks(blocks, block, n_valid, per_block, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for b in blocks:
        lo, hi = b * block, min((b + 1) * block, n_valid)
        rows.update((lo, hi - 1))
        rows.update(int(x) for x in rng.integers(lo, hi, size=per_block))
    return np.array(sorted(rows), dtype=np.int64)


def head_perms(w, plan):
    """Token order of every head in the path (None: raster order).  The spade family's
    per-head shapes are the plan's SICS choice, which tests/test_gpu_sics.py and
    check_spade_choice hold to the oracle's."""
    if not plan.permuted:
        return [None] * w.heads
    if w.mask == "spade":
        choice = plan.choice.cpu().numpy()
        return [O.tile_order(w.grid, plan.menu[int(choice[0, h])]) for h in range(w.heads)]
    perm = O.tile_order(w.grid, w.tile)
    return [perm] * w.heads


def check_spade_choice(w, plan, q, k):
    """The plan's per-head slice choice against the oracle's SICS scheme (near ties
    may go either way)."""
    rs, rc = O.sics_scheme(to64(q), to64(k), w.grid, plan.menu)
    choice = plan.choice.cpu().numpy()
    for h in range(w.heads):
        order = np.argsort(-rs[0, h], kind="stable")
        near = [s for s in range(rs.shape[2]) if rs[0, h, order[0]] - rs[0, h, s] < 1e-4]
        assert choice[0, h] == rc[0, h] or choice[0, h] in near, h
    return choice


def oracle_mask(w, plan, q, k):
    """The oracle's own block mask for the workload ([Hm, QB, KB] plus near flags)."""
    if w.mask == "sta":
        return O.sta_tile_mask(plan.tile_grid, w.window)[None], None
    if w.mask == "radial":
        return O.radial_block_mask_fast(w.nk, w.tokens_per_frame, w.block)[None], None
    D = w.head_dim
    scale = 1.0 / math.sqrt(D)
    if w.mask in ("nabla", "nabla_sta", "spade"):
        perms = head_perms(w, plan)
        qbar = np.zeros((w.batch, w.heads, plan.QB, D))
        kbar = np.zeros((w.batch, w.heads, plan.KB, D))
        for h in range(w.heads):
            qh = O.tile_permute(to64(q[:, :, h:h + 1]), perms[h], plan.n_pad)
            kh = O.tile_permute(to64(k[:, :, h:h + 1]), perms[h], plan.n_pad)
            qbar[:, h] = O.nabla_pool(qh, w.block, w.nq)[:, 0]
            kbar[:, h] = O.nabla_pool(kh, w.block, w.nk)[:, 0]
        if w.mask in ("nabla", "spade"):
            m, near = O.nabla_mask(qbar, kbar, w.p, scale)
        else:
            m, near = O.nabla_sta_mask(qbar, kbar, w.p, scale,
                                       O.sta_tile_mask(plan.tile_grid, w.window))
    else:  # ar
        QBp, KBp = plan.QB * w.block, plan.KB * w.block
        qbar = np.zeros((w.batch, w.heads, plan.QB, D))
        kbar = np.zeros((w.batch, w.heads, plan.KB, D))
        for h in range(w.heads):
            qh = np.zeros((w.batch, QBp, 1, D))
            qh[:, :w.nq] = to64(q[:, :, h:h + 1])
            kh = np.zeros((w.batch, KBp, 1, D))
            kh[:, :w.nk] = to64(k[:, :, h:h + 1])
            qbar[:, h] = O.nabla_pool(qh, w.block, w.nq)[:, 0]
            kbar[:, h] = O.nabla_pool(kh, w.block, w.nk)[:, 0]
        m, near = O.ar_mask(qbar, kbar, w.p, scale, w.nk, w.tokens_per_frame, w.block,
                            w.anchor_frames, w.recent_frames)
    return m.reshape(-1, plan.QB, plan.KB), near.reshape(-1, plan.QB)


@pytest.mark.parametrize("name", [w.name for w in configs.WORKLOADS + configs.EXTRA])
def test_workload_path(name):
    w = configs.get(name)
    q, k, v, _ = synth.workload_inputs(w)
    plan = Plan(w)
    o, lse = plan.step(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    from block_sparse_attention_tokens_b200 import binding as B
    assert B.bsa_read_status(plan.attn_ws) == 0

    if w.mask == "spade":
        check_spade_choice(w, plan, q, k)
        assert int(plan.scheme_status.item()) == 0

    # --- mask: bit-exact against the oracle's own mask
    ref_mask, near = oracle_mask(w, plan, q, k)
    gpu_mask = plan.mask.cpu().numpy().reshape(-1, plan.QB, plan.KB)
    differs = np.any(gpu_mask != ref_mask, axis=-1)
    if near is None:
        assert not differs.any(), f"{int(differs.sum())} mask rows differ"
        skip_rows = np.zeros_like(differs)
    else:
        assert not (differs & ~near).any(), "NABLA rows differ away from the threshold"
        skip_rows = differs

    # --- attention on sampled rows (path token order) against the oracle
    perms = head_perms(w, plan)
    blocks = sample_blocks(plan.QB, 6 if w.nk > 200000 else 12, seed=w.seed)
    rows = sample_rows_in_blocks(blocks, w.block, w.nq, 6, seed=w.seed + 1)
    op = (plan.op if plan.permuted else plan.o).cpu()
    lse_g = lse.cpu().numpy().astype(np.float64)
    for h in range(w.heads):
        hm = 0 if ref_mask.shape[0] == 1 else h
        keep_rows = rows[~skip_rows[hm, rows // w.block]]
        if keep_rows.size == 0:
            continue
        if plan.permuted:
            qh = O.tile_permute(to64(q[:, :, h:h + 1]), perms[h], plan.n_pad)
            kh = O.tile_permute(to64(k[:, :, h:h + 1]), perms[h], plan.n_pad)
            vh = O.tile_permute(to64(v[:, :, h:h + 1]), perms[h], plan.n_pad)
            qh, kh, vh = qh[:, :w.nq], kh[:, :w.nk], vh[:, :w.nk]
        else:
            qh, kh, vh = to64(q[:, :, h:h + 1]), to64(k[:, :, h:h + 1]), to64(v[:, :, h:h + 1])
        ro, rl = O.block_sparse_attention(qh, kh, vh, ref_mask[hm:hm + 1], w.block, w.block,
                                          rows=keep_rows)
        og = to64(op[0, keep_rows, h])
        assert_attention_close(og, lse_g[0, h, keep_rows], ro[0, keep_rows, 0],
                               rl[0, 0, keep_rows], what=f"{name} head {h}")

    # --- inverse permute: O in raster order is op[perm^-1], bit-exact
    if plan.permuted:
        ob = o.cpu().view(torch.int16).numpy()
        opb = op.view(torch.int16).numpy()
        r = rows[rows < w.nq]
        for h in range(w.heads):
            assert np.array_equal(ob[:, perms[h][r], h], opb[:, r, h]), h
