"""GPU parity of the block-sparse attention backward (dQ, dK, dV) against the
float64 oracle, element by element, through the C ABI.

The forward kernel's own O and LSE feed the backward (as in training); the
oracle recomputes everything in float64 from the same bf16 Q, K, V, dO.

Tolerance, derived from the kernel's arithmetic.  Inputs are bf16 and exact in
both paths.  The kernel rounds to bf16 (unit roundoff u = 2^-9): P before
dV += P^T dO, dS before dQ += dS K and dK += dS^T Q, and the three outputs.
Delta = rowsum(dO * O) is taken from the forward's bf16 O, itself a sum of
bf16-rounded probabilities times V, so |Delta error| <= u * W_i with
W_i = sum_d |dO_id| * ((P|V|)_id + |O_id|) up to second order.  fp32
accumulation over <= 10^3 terms and the approximate exp2 add far less than u.
So, elementwise,
    |dV_jd err| <= u * sum_i P_ij |dO_id|                              + u |dV_jd|
    |dQ_id err| <= u * scale * sum_j E_ij |K_jd|                        + u |dQ_id|
    |dK_jd err| <= u * scale * sum_i E_ij |Q_id|                        + u |dK_jd|
with E_ij = P_ij (|dP_ij| + |Delta_i| + W_i) bounding |dS_ij| and its Delta
error before cancellation (first order in u).  The test allows 4u times the
envelope (the sums above) plus 2u |ref|.
Entries with no kept pair (keys no query keeps, rows that keep nothing) must be
exactly zero.  A dropped term, a wrong quadrant or a transposed operand moves
an entry by a sizeable fraction of its envelope and fails."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth
from tests._parity import to64

pytestmark = pytest.mark.gpu

U = 2.0 ** -9


def envelopes(q, k, v, do, o_ref, lse_ref, mask, bq, bk, scale):
    """Per-entry error envelopes (see the module docstring); float64 numpy.
    q, do, o_ref: [B, nq, H, D]; k, v: [B, nk, H, D]; lse_ref: [B, H, nq]."""
    Bn, nq, H, D = q.shape
    nk = k.shape[1]
    env_q, env_k, env_v = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(Bn):
        for h in range(H):
            m = mask[0 if mask.shape[0] == 1 else b * H + h]
            allowed = O.token_mask_from_blocks(m, nq, nk, bq, bk)
            s = q[b, :, h] @ k[b, :, h].T * scale
            lse = lse_ref[b, h]
            fin = np.isfinite(lse)
            p = np.where(allowed & fin[:, None],
                         np.exp(np.minimum(s - np.where(fin, lse, 0.0)[:, None], 0.0)), 0.0)
            g = do[b, :, h]
            dp = g @ v[b, :, h].T
            delta = (g * (p @ v[b, :, h])).sum(axis=1)
            w = (np.abs(g) * (p @ np.abs(v[b, :, h]) + np.abs(o_ref[b, :, h]))).sum(axis=1)
            e = p * (np.abs(dp) + np.abs(delta)[:, None] + w[:, None])
            env_v[b, :, h] = p.T @ np.abs(g)
            env_q[b, :, h] = scale * (e @ np.abs(k[b, :, h]))
            env_k[b, :, h] = scale * (e.T @ np.abs(q[b, :, h]))
    return env_q, env_k, env_v


def assert_grad_close(got, ref, env, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    err = np.abs(got - ref)
    bound = 4 * U * env + 2 * U * np.abs(ref)
    zero = env == 0
    assert np.all(got[zero] == 0), f"{what}: entries without kept pairs must be exactly 0"
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} entries outside the envelope; worst at "
                             f"{i}: got {got[i]:.6e} ref {ref[i]:.6e} bound {bound[i]:.3e}")
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30))
    return rel


def run_bwd(Bn, H, nq, nk, D, bq, bk, mask, list_heads, seed, scale=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    do = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse, ws = B.bsa_attn_fwd(qc, kc, vc, rp, ci, bq, bk, list_heads, scale=scale)
    dq, dk, dv, bws = B.bsa_attn_bwd(qc, kc, vc, o, doc, lse, rp, ci, bq, bk, list_heads,
                                     scale=scale)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    assert B.bsa_read_status(bws) == 0
    sc = 1.0 / math.sqrt(D) if scale <= 0 else scale
    q64, k64, v64, do64 = to64(q), to64(k), to64(v), to64(do)
    rdq, rdk, rdv = O.block_sparse_attention_backward(q64, k64, v64, do64, mask, bq, bk, scale=sc)
    ro, rl = O.block_sparse_attention(q64, k64, v64, mask, bq, bk, scale=sc)
    eq, ek, ev = envelopes(q64, k64, v64, do64, ro, rl, mask, bq, bk, sc)
    return (assert_grad_close(to64(dq), rdq, eq, "dQ"), assert_grad_close(to64(dk), rdk, ek, "dK"),
            assert_grad_close(to64(dv), rdv, ev, "dV"))


def test_tiny_all_ones_equals_dense():
    run_bwd(1, 2, 256, 256, 64, 64, 64, np.ones((1, 4, 4), np.uint8), 1, seed=3)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bq,bk", [(128, 128), (64, 64), (384, 384), (64, 128), (256, 64)])
def test_random_masks_ragged(D, bq, bk):
    nq, nk = 5 * 128 + 37, 6 * 128 + 11
    Bn, H = 2, 2
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = synth.random_mask(Bn * H * QB, KB, 0.45, seed=bq + bk + D + 7).reshape(Bn * H, QB, KB)
    mask[0, 0] = 0                       # a row that keeps nothing
    mask[1, :, 1] = 0                    # a key block no row keeps
    mask[1, -1] = 0
    mask[1, -1, -1] = 1                  # only the ragged last key block
    mask[2, 1] = 0
    mask[2, 1, 0] = 1                    # a single kept block
    run_bwd(Bn, H, nq, nk, D, bq, bk, mask, Bn * H, seed=D + bq + bk)


def test_shared_list_custom_scale_cross_lengths():
    nq, nk, bq, bk = 3 * 128 + 5, 9 * 64 + 63, 64, 64
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = synth.random_mask(QB, KB, 0.5, seed=11).reshape(1, QB, KB)
    run_bwd(1, 3, nq, nk, 128, bq, bk, mask, 1, seed=5, scale=0.05)


def test_all_masked_gives_zero_gradients():
    mask = np.zeros((1, 3, 3), np.uint8)
    run_bwd(1, 1, 300, 300, 64, 128, 128, mask, 1, seed=9)


def test_sta_mask_on_a_tiled_grid():
    # Sliding-Tile mask over a 4x8x8 token grid with 4x4x4 tiles (64-token blocks)
    tg, window = (1, 2, 2), (1, 3, 3)
    m = O.sta_tile_mask(tg, window)[None].astype(np.uint8)
    run_bwd(1, 2, 256, 256, 128, 64, 64, m, 1, seed=13)


def key_envelopes(qh, kh, vh, doh, mask, block, keys, sc):
    """Envelopes of dK and dV (module docstring) on the given key rows of one head:
    every query block that keeps one of their blocks is evaluated over its whole
    kept row (P, dP, Delta and W need all of the row's keys).  Arrays [1, n, 1, D]."""
    nq, nk = qh.shape[1], kh.shape[1]
    want = np.unique(keys // block)
    env_k = np.zeros((len(keys), qh.shape[-1]))
    env_v = np.zeros_like(env_k)
    for qb in range(mask.shape[1]):
        kept = np.nonzero(mask[0, qb])[0]
        if not np.isin(want, kept).any():
            continue
        rows = np.arange(qb * block, min((qb + 1) * block, nq))
        cols = np.concatenate([np.arange(kb * block, min((kb + 1) * block, nk)) for kb in kept])
        qq, kk, vv, g = qh[0, rows, 0], kh[0, cols, 0], vh[0, cols, 0], doh[0, rows, 0]
        s = (qq @ kk.T) * sc
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ vv
        dp = g @ vv.T
        delta = (g * o).sum(axis=1)
        w = (np.abs(g) * (p @ np.abs(vv) + np.abs(o))).sum(axis=1)
        e = p * (np.abs(dp) + np.abs(delta)[:, None] + w[:, None])
        idx = np.minimum(np.searchsorted(cols, keys), cols.size - 1)   # cols ascending
        hit = cols[idx] == keys
        env_v[hit] += p[:, idx[hit]].T @ np.abs(g)
        env_k[hit] += sc * (e[:, idx[hit]].T @ np.abs(qq))
    return env_k, env_v


def test_full_size_sta_720p_sampled_rows_keys_and_identities():
    """The 720p Sliding-Tile workload at full size (24 heads, 115,200 tokens, the
    benchmark's launch), element by element within the per-entry envelope:
    dQ on sampled query rows and dK, dV on every key of sampled 128-key tiles,
    against the oracle (its key sampling evaluates every query block that keeps a
    sampled key).  Both kernel passes are persistent (one CTA per SM takes work
    items in (head, tile) order from a global counter), so every item past the
    first SM-count ones -- all of head 13's, and head 0's tiles beyond the first
    148 -- is a CTA's second or later item: barrier phases, TMEM reuse and the
    transposed lists at scale are compared, not only summed.  Two identities that
    involve every dK and dV entry follow: sum_i q_i . dQ_i = sum_j k_j . dK_j (both
    equal scale * sum dS_ij q_i.k_j) and sum_j dV_j = sum of dO_i over rows that
    keep a key; they are coarse (1 % of the absolute sums) and catch a lost
    quadrant, term or factor anywhere."""
    from block_sparse_attention_tokens_b200 import configs
    from block_sparse_attention_tokens_b200.pipeline import Plan
    w = configs.get("sta_720p")
    q, k, v, _ = synth.workload_inputs(w)
    plan = Plan(w)
    plan.step(q.cuda(), k.cuda(), v.cuda())
    do = synth.grad_output(w)
    dq, dk, dv, ws = B.bsa_attn_bwd(plan.qp, plan.kp, plan.vp, plan.op, do.cuda(), plan.lse,
                                    plan.row_ptr, plan.col_idx, w.block, w.block, plan.list_heads,
                                    nq=plan.nq, nk=plan.nk)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    perm = O.tile_order(w.grid, w.tile)
    mask = O.sta_tile_mask(plan.tile_grid, w.window)[None]
    sc = 1.0 / math.sqrt(w.head_dim)
    rng = np.random.default_rng(3)
    qbs = [0, plan.QB - 1] + list(rng.choice(plan.QB, 2, replace=False))
    rows = np.unique(np.concatenate([qb * w.block + np.array([0, 191, w.block - 1]) for qb in qbs]))
    # 8 key tiles of 128 keys: the first and last, and two of the three tiles of
    # three random 384-key blocks
    KT = math.ceil(w.nk / 128)
    kbs = rng.choice(np.arange(1, plan.QB - 1), 3, replace=False)
    tiles = [0, KT - 1] + [int(kb) * 3 + t for kb in kbs for t in (0, 2)]
    keys = np.unique(np.concatenate([np.arange(t * 128, min((t + 1) * 128, w.nk)) for t in tiles]))
    dq_g = to64(dq[:, :w.nq])
    dk_g, dv_g = to64(dk[:, :w.nk]), to64(dv[:, :w.nk])
    for h in (0, 13):
        qh = O.tile_permute(to64(q[:, :, h:h + 1]), perm, plan.n_pad)[:, :w.nq]
        kh = O.tile_permute(to64(k[:, :, h:h + 1]), perm, plan.n_pad)[:, :w.nk]
        vh = O.tile_permute(to64(v[:, :, h:h + 1]), perm, plan.n_pad)[:, :w.nk]
        doh = to64(do[:, :, h:h + 1])
        rdq, _, _ = O.block_sparse_attention_backward(qh, kh, vh, doh, mask, w.block, w.block,
                                                      rows=rows)
        ro, rl = O.block_sparse_attention(qh, kh, vh, mask, w.block, w.block, rows=rows)
        for i in rows:
            kept = np.nonzero(mask[0, i // w.block])[0]
            cols = np.concatenate([np.arange(kb * w.block, min((kb + 1) * w.block, w.nk))
                                   for kb in kept])
            kk, vv, g = kh[0, cols, 0], vh[0, cols, 0], doh[0, i, 0]
            p = np.exp((kk @ qh[0, i, 0]) * sc - rl[0, 0, i])
            dp = vv @ g
            delta = g @ ro[0, i, 0]
            wi = np.sum(np.abs(g) * (p @ np.abs(vv) + np.abs(ro[0, i, 0])))
            env = sc * ((p * (np.abs(dp) + abs(delta) + wi)) @ np.abs(kk))
            err = np.abs(dq_g[0, i, h] - rdq[0, i, 0])
            assert np.all(err <= 4 * U * env + 2 * U * np.abs(rdq[0, i, 0])), (h, i)
        # dK and dV of the sampled key tiles
        _, rdk, rdv = O.block_sparse_attention_backward(qh, kh, vh, doh, mask, w.block, w.block,
                                                        cols=keys)
        env_k, env_v = key_envelopes(qh, kh, vh, doh, mask, w.block, keys, sc)
        assert_grad_close(dk_g[0, keys, h], rdk[0, keys, 0], env_k, f"dK head {h}")
        assert_grad_close(dv_g[0, keys, h], rdv[0, keys, 0], env_v, f"dV head {h}")
    # identities over all heads and every entry of dK and dV
    qp, kp, vpd = to64(plan.qp[:, :w.nq]), to64(plan.kp[:, :w.nk]), dv_g
    lhs = np.einsum("bnhd,bnhd->h", qp, dq_g)
    rhs = np.einsum("bnhd,bnhd->h", kp, dk_g)
    scale_abs = (np.einsum("bnhd,bnhd->h", np.abs(qp), np.abs(dq_g))
                 + np.einsum("bnhd,bnhd->h", np.abs(kp), np.abs(dk_g)))
    assert np.all(np.abs(lhs - rhs) <= 1e-2 * scale_abs)
    do64 = to64(do)
    dv_sum = vpd.sum(axis=1)
    do_sum = do64.sum(axis=1)                       # every STA query row keeps keys
    assert np.all(np.abs(dv_sum - do_sum) <= 1e-2 * np.abs(do64).sum(axis=1))
