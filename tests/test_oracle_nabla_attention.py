"""Pins of the oracle's NABLA selection, AR composition and attention (CPU only)."""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from tests._golden import load


# ----------------------------------------------------------------- pooling

def test_pool_mean_over_valid_tokens_only():
    x = np.zeros((1, 8, 1, 2))
    x[0, :, 0, 0] = np.arange(8)
    x[0, :, 0, 1] = 1.0
    # n_valid = 6: block 0 = tokens 0..3, block 1 = tokens 4, 5 (6, 7 are padding)
    x[0, 6:] = 123.0
    out = O.nabla_pool(x, 4, 6)
    assert np.allclose(out[0, 0, 0], [1.5, 1.0])
    assert np.allclose(out[0, 0, 1], [4.5, 1.0])


# ----------------------------------------------------------------- top-p selection

def _brute_min_cardinality(probs, p):
    n = len(probs)
    for k in range(1, n + 1):
        best = max(sum(probs[list(c)]) for c in itertools.combinations(range(n), k))
        if best >= p:
            return k
    return n


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("p", [0.3, 0.7, 0.9, 0.97])
def test_select_is_minimal_and_covers_p_brute_force(seed, p):
    rng = np.random.default_rng(seed)
    n = 9
    z = rng.normal(0, 1.5, n)
    probs = scipy.special.softmax(z)
    kept, cum, k_star, _ = O.nabla_select_row(probs, p)
    assert len(kept) == k_star == _brute_min_cardinality(probs, p)
    assert probs[kept].sum() >= p                       # coverage
    top = np.sort(probs)[::-1]
    assert top[:k_star - 1].sum() < p                   # minimality
    # the kept set is a top set: nothing dropped is larger than anything kept
    dropped = np.setdiff1d(np.arange(n), kept)
    if dropped.size:
        assert probs[dropped].max() <= probs[kept].min()


def test_select_uniform_keeps_ceil_p_lowest_indices():
    kb = 40
    probs = np.full(kb, 1.0 / kb)
    for p in (0.1, 0.5, 0.9, 0.925):
        kept, _, k_star, _ = O.nabla_select_row(probs, p)
        expect = math.ceil(round(p * kb, 9))
        assert k_star == expect
        assert sorted(kept.tolist()) == list(range(expect))


def test_select_small_p_is_argmax_and_p_one_keeps_all():
    probs = scipy.special.softmax(np.array([0.1, 2.0, -1.0, 1.9]))
    kept, _, _, _ = O.nabla_select_row(probs, 1e-9)
    assert kept.tolist() == [1]
    kept, _, k_star, _ = O.nabla_select_row(probs, 1.0)
    assert k_star == 4


def test_select_reaching_p_exactly_covers_it():
    # dyadic probabilities are exact in binary floating point: a prefix whose mass
    # equals p reaches it (READING: the kept set is the smallest one whose mass is
    # at least p), and of two equal entries the lower index comes first
    probs = np.array([0.25, 0.5, 0.125, 0.125])
    kept, cum, k_star, _ = O.nabla_select_row(probs, 0.75)
    assert cum[1] == 0.75 and k_star == 2 and sorted(kept.tolist()) == [0, 1]
    kept, _, k_star, _ = O.nabla_select_row(probs, 0.875)
    assert k_star == 3 and sorted(kept.tolist()) == [0, 1, 2]


def test_nabla_mask_dominant_block_and_constant_queries():
    rng = np.random.default_rng(7)
    Bn, H, QB, KB, D = 1, 2, 3, 16, 8
    qbar = np.zeros((Bn, H, QB, D))
    qbar[..., 0] = 10.0
    qbar[..., 1:] = rng.normal(size=(Bn, H, QB, D - 1)) * 0.01
    kbar = rng.normal(size=(Bn, H, KB, D)) * 0.01
    # head 0: key block 5 has logit 10 * 5 * sqrt(D) / sqrt(D) = +50 against every query
    kbar[0, 0, 5] = 0.0
    kbar[0, 0, 5, 0] = 5.0 * math.sqrt(D)
    mask, near = O.nabla_mask(qbar, kbar, 0.9, 1.0 / math.sqrt(D))
    for qb in range(QB):
        assert mask[0, 0, qb].tolist() == [1 if c == 5 else 0 for c in range(KB)]
    # head 1: identical pooled keys -> uniform -> ceil(0.9 * 16) = 15 lowest blocks
    kbar[0, 1] = 0.3
    mask, near = O.nabla_mask(qbar, kbar, 0.9, 1.0 / math.sqrt(D))
    assert np.all(mask[0, 1, :, :15] == 1) and np.all(mask[0, 1, :, 15] == 0)


def test_nabla_mask_range_and_forced_outside():
    rng = np.random.default_rng(9)
    qbar = rng.normal(size=(1, 1, 4, 8))
    kbar = rng.normal(size=(1, 1, 20, 8))
    mask, _ = O.nabla_mask(qbar, kbar, 0.8, 0.35, kb_begin=3, kb_end=15, force_outside=1)
    assert np.all(mask[..., :3] == 1) and np.all(mask[..., 15:] == 1)
    # middle range: softmax renormalised over blocks 3..14 only
    z = (qbar[0, 0] @ kbar[0, 0, 3:15].T) * 0.35
    probs = scipy.special.softmax(z, axis=1)
    for qb in range(4):
        kept = np.nonzero(mask[0, 0, qb, 3:15])[0]
        assert probs[qb, kept].sum() >= 0.8
        assert np.sort(probs[qb])[::-1][:len(kept) - 1].sum() < 0.8


def test_ar_mask_forces_anchors_and_recent_and_selects_the_middle():
    # 10 frames of 8 tokens, 4-token blocks: 2 anchor frames are blocks 0..3, the
    # last 3 frames touch blocks 14..19; NABLA picks among blocks 4..13 with the
    # softmax renormalised over them
    rng = np.random.default_rng(13)
    qbar = rng.normal(size=(1, 2, 5, 8))
    kbar = rng.normal(size=(1, 2, 20, 8))
    mask, _ = O.ar_mask(qbar, kbar, 0.7, 0.5, 80, 8, 4, 2, 3)
    assert np.all(mask[..., :4] == 1) and np.all(mask[..., 14:] == 1)
    for h in range(2):
        probs = scipy.special.softmax((qbar[0, h] @ kbar[0, h, 4:14].T) * 0.5, axis=1)
        for qb in range(5):
            kept = np.nonzero(mask[0, h, qb, 4:14])[0]
            assert probs[qb, kept].sum() >= 0.7
            assert np.sort(probs[qb])[::-1][:len(kept) - 1].sum() < 0.7


def test_nabla_sta_union_contains_both_masks():
    rng = np.random.default_rng(12)
    qbar = rng.normal(size=(1, 2, 12, 8))
    kbar = rng.normal(size=(1, 2, 12, 8))
    sta = O.sta_tile_mask((1, 3, 4), (1, 3, 3))
    m, near = O.nabla_sta_mask(qbar, kbar, 0.6, 0.35, sta)
    alone, _ = O.nabla_mask(qbar, kbar, 0.6, 0.35)
    assert np.all(m >= alone) and np.all(m >= sta[None, None])
    assert np.array_equal(m, np.maximum(alone, sta[None, None]))


def test_ar_ranges_match_the_decode_workload():
    # 60 frames of 30x52 = 1560 tokens, 64-token blocks, 3 anchor frames, last 6 dense
    a_end, r_begin = O.ar_block_ranges(60 * 1560, 1560, 64, 3, 6)
    kb = math.ceil(60 * 1560 / 64)
    assert kb == 1463
    assert a_end == 74                   # blocks touching tokens [0, 4680)
    assert kb - r_begin == 147           # blocks touching tokens [84240, 93600)


def test_near_threshold_flag():
    probs_z = np.log(np.array([0.5, 0.4, 0.1]))
    qbar = np.zeros((1, 1, 1, 1))
    kbar = np.zeros((1, 1, 3, 1))
    # z = qbar.kbar * scale: encode the logits in kbar with qbar = 1
    qbar[...] = 1.0
    kbar[0, 0, :, 0] = probs_z
    _, near = O.nabla_mask(qbar, kbar, 0.9, 1.0)       # 0.5 + 0.4 == 0.9 exactly
    assert near[0, 0, 0]
    _, near = O.nabla_mask(qbar, kbar, 0.8, 1.0)
    assert not near[0, 0, 0]
    # the prefix before the cut (0.5) lies 1e-7 below p: a float32 sum may reach p there
    _, near = O.nabla_mask(qbar, kbar, 0.5 + 1e-7, 1.0)
    assert near[0, 0, 0]
    # last kept and first dropped probabilities tie (0.3, 0.3): either may be kept
    kbar[0, 0, :, 0] = np.log(np.array([0.4, 0.3, 0.3]))
    mask, near = O.nabla_mask(qbar, kbar, 0.6, 1.0)
    assert mask[0, 0, 0].tolist() == [1, 1, 0] and near[0, 0, 0]


# ----------------------------------------------------------------- attention

def test_attention_golden_two_keys():
    q, k0, k1, v0, v1, o, lse = load("attention_two_keys.txt")[0]
    out, l = O.dense_masked_attention(np.array([[q]]), np.array([[k0], [k1]]),
                                      np.array([[v0], [v1]]), np.ones((1, 2), bool), 1.0)
    assert abs(out[0, 0] - o) < 1e-12 and abs(l[0] - lse) < 1e-12


def _rand_qkv(Bn, nq, nk, H, D, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((Bn, nq, H, D)), rng.standard_normal((Bn, nk, H, D)),
            rng.standard_normal((Bn, nk, H, D)))


def test_all_ones_mask_equals_sdpa_float64():
    q, k, v = _rand_qkv(2, 130, 200, 3, 16, 1)
    mask = np.ones((1, math.ceil(130 / 64), math.ceil(200 / 64)), np.uint8)
    o, lse = O.block_sparse_attention(q, k, v, mask, 64, 64)
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(o - ref)) < 1e-12
    s = np.einsum("bihd,bjhd->bhij", q, k) / 4.0
    assert np.max(np.abs(lse - scipy.special.logsumexp(s, axis=-1))) < 1e-12


@pytest.mark.parametrize("bq,bk", [(64, 64), (128, 64), (64, 128), (384, 384)])
def test_block_mask_equals_token_level_definition(bq, bk):
    Bn, H, D = 1, 2, 8
    nq, nk = 3 * bq - 17, 4 * bk - 5                    # ragged last blocks
    q, k, v = _rand_qkv(Bn, nq, nk, H, D, 2)
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    rng = np.random.default_rng(4)
    mask = (rng.random((Bn * H, QB, KB)) < 0.5).astype(np.uint8)
    mask[1, 1] = 0                                      # an empty row
    o, lse = O.block_sparse_attention(q, k, v, mask, bq, bk)
    for h in range(H):
        allowed = O.token_mask_from_blocks(mask[h], nq, nk, bq, bk)
        ro, rl = O.dense_masked_attention(q[0, :, h], k[0, :, h], v[0, :, h], allowed,
                                          1 / math.sqrt(D))
        assert np.allclose(o[0, :, h], ro, atol=1e-12, rtol=0)
        assert np.array_equal(np.isneginf(lse[0, h]), np.isneginf(rl))
        fin = np.isfinite(rl)
        assert np.allclose(lse[0, h][fin], rl[fin], atol=1e-12)
    rows = np.arange(bq, 2 * bq)
    assert np.all(o[0, rows, 1] == 0) and np.all(np.isneginf(lse[0, 1, rows]))


def test_per_batch_head_masks_index_b_times_h_plus_h():
    # a mask per (batch, head) is row b * H + h of the mask stack
    Bn, H, D, blk = 2, 3, 8, 64
    nq, nk = 150, 190
    q, k, v = _rand_qkv(Bn, nq, nk, H, D, 8)
    QB, KB = math.ceil(nq / blk), math.ceil(nk / blk)
    mask = (np.random.default_rng(9).random((Bn * H, QB, KB)) < 0.5).astype(np.uint8)
    mask[:, :, 0] = 1
    o, lse = O.block_sparse_attention(q, k, v, mask, blk, blk)
    for b in range(Bn):
        for h in range(H):
            allowed = O.token_mask_from_blocks(mask[b * H + h], nq, nk, blk, blk)
            ro, rl = O.dense_masked_attention(q[b, :, h], k[b, :, h], v[b, :, h], allowed,
                                              1 / math.sqrt(D))
            assert np.allclose(o[b, :, h], ro, atol=1e-12, rtol=0)
            assert np.allclose(lse[b, h], rl, atol=1e-12, rtol=0)


def test_single_kept_block_is_softmax_over_that_block_and_lse_normalises():
    Bn, H, D, blk = 1, 1, 16, 64
    q, k, v = _rand_qkv(Bn, 128, 256, H, D, 5)
    mask = np.zeros((1, 2, 4), np.uint8)
    mask[0, 0, 2] = 1
    mask[0, 1, 3] = 1
    o, lse = O.block_sparse_attention(q, k, v, mask, blk, blk)
    s = q[0, :64, 0] @ k[0, 128:192, 0].T / 4.0
    w = scipy.special.softmax(s, axis=1)
    assert np.allclose(o[0, :64, 0], w @ v[0, 128:192, 0], atol=1e-12)
    assert np.allclose(np.exp(s - lse[0, 0, :64, None]).sum(axis=1), 1.0, atol=1e-12)


def test_sampled_rows_match_full_evaluation():
    q, k, v = _rand_qkv(1, 300, 300, 2, 8, 6)
    mask = (np.random.default_rng(1).random((1, 5, 5)) < 0.6).astype(np.uint8)
    o, lse = O.block_sparse_attention(q, k, v, mask, 64, 64)
    rows = np.array([0, 63, 64, 200, 299])
    o2, lse2 = O.block_sparse_attention(q, k, v, mask, 64, 64, rows=rows)
    assert np.allclose(o[:, rows], o2[:, rows], atol=1e-13, rtol=0)
    assert np.allclose(lse[..., rows], lse2[..., rows], atol=1e-13, rtol=0)


# ----------------------------------------------------------------- backward

@pytest.mark.parametrize("bq,bk", [(64, 64), (128, 64), (384, 384)])
def test_backward_matches_autograd_float64(bq, bk):
    Bn, H, D = 1, 2, 16
    nq, nk = 2 * bq + 9, 3 * bk - 7
    q, k, v = _rand_qkv(Bn, nq, nk, H, D, 21)
    do = np.random.default_rng(22).standard_normal((Bn, nq, H, D))
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = (np.random.default_rng(23).random((Bn * H, QB, KB)) < 0.6).astype(np.uint8)
    mask[0, 1] = 0                                      # a row without kept blocks
    dq, dk, dv = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = []
    for h in range(H):
        allowed = torch.from_numpy(O.token_mask_from_blocks(mask[h], nq, nk, bq, bk))
        s = (tq[0, :, h] @ tk[0, :, h].T) / math.sqrt(D)
        s = s.masked_fill(~allowed, float("-inf"))
        pr = torch.softmax(s, dim=1)
        pr = torch.nan_to_num(pr, nan=0.0)              # rows with nothing allowed
        out.append(pr @ tv[0, :, h])
    o = torch.stack(out, dim=1)[None]
    o.backward(torch.from_numpy(do))
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(got - ref.numpy())) < 1e-12


def test_backward_row_sampling_is_exact_on_dq_and_additive_on_dk_dv():
    Bn, H, D, bq, bk = 1, 2, 16, 64, 64
    nq, nk = 200, 300
    q, k, v = _rand_qkv(Bn, nq, nk, H, D, 31)
    do = np.random.default_rng(32).standard_normal((Bn, nq, H, D))
    mask = (np.random.default_rng(33).random((Bn * H, 4, 5)) < 0.6).astype(np.uint8)
    full = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk)
    rows_a = np.arange(0, nq, 3)
    rows_b = np.setdiff1d(np.arange(nq), rows_a)
    ga = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk, rows=rows_a)
    gb = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk, rows=rows_b)
    assert np.allclose(ga[0][:, rows_a], full[0][:, rows_a], atol=1e-12)
    assert np.all(ga[0][:, rows_b] == 0)
    for i in (1, 2):                                    # dK, dV: the two halves add up
        assert np.allclose(ga[i] + gb[i], full[i], atol=1e-12)


def test_backward_column_sampling_is_exact_on_dk_dv():
    # key sampling evaluates every query block that keeps a wanted key's block, each
    # over its whole kept row: dk and dv on the wanted keys equal the full evaluation
    Bn, H, D, bq, bk = 1, 2, 16, 128, 64
    nq, nk = 300, 330
    q, k, v = _rand_qkv(Bn, nq, nk, H, D, 41)
    do = np.random.default_rng(42).standard_normal((Bn, nq, H, D))
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = (np.random.default_rng(43).random((Bn * H, QB, KB)) < 0.6).astype(np.uint8)
    mask[:, :, 2] = 0
    mask[:, 0, 2] = 1                                   # block 2: only query block 0
    mask[:, :, 4:] = 1
    mask[:, 0, 4:] = 0                                  # blocks 4, 5: query blocks 1, 2
    mask[1, :, 4] = 0                                   # head 1: block 4 kept by nobody
    full = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk)
    cols = np.array([4 * bk, 4 * bk + 37, 5 * bk + 3, nk - 1])
    part = O.block_sparse_attention_backward(q, k, v, do, mask, bq, bk, cols=cols)
    for i in (1, 2):
        assert np.allclose(part[i][:, cols], full[i][:, cols], atol=1e-12, rtol=0)
        assert np.any(part[i][:, cols] != 0)
    assert np.all(part[1][0, 4 * bk, 1] == 0) and np.all(part[2][0, 4 * bk, 1] == 0)
    # rows of query blocks that keep none of the wanted blocks are not evaluated
    wanted = np.unique(cols // bk)
    for h in range(H):
        for qb in range(QB):
            if not mask[h, qb, wanted].any():
                assert np.all(part[0][0, qb * bq:(qb + 1) * bq, h] == 0)


def test_nabla_mask_at_long_key_ranges():
    # 7,088 key blocks (453,600 tokens in 64-token blocks): a closed-form row --
    # five blocks at logit 12, the rest at 0, so the five hold 5e^12 / (5e^12 + 7083)
    # > 0.9 of the mass and no four of them reach 0.9 -- keeps exactly those five;
    # random rows keep the shortest prefix reaching p (checked against the sorted
    # probabilities directly)
    KB, D, p = 7088, 16, 0.9
    hot = np.array([3, 1000, 4096, 7000, KB - 1])
    kbar = np.zeros((1, 1, KB, D))
    kbar[0, 0, hot, 0] = 3.0
    qbar = np.zeros((1, 1, 2, D))
    qbar[0, 0, 0, 0] = 4.0
    qbar[0, 0, 1] = np.random.default_rng(7).standard_normal(D)
    kbar[0, 0, :, 1:] = np.random.default_rng(8).standard_normal((KB, D - 1))
    kbar_hot_only = kbar.copy()
    kbar_hot_only[0, 0, :, 1:] = 0.0
    m, near = O.nabla_mask(qbar[:, :, :1], kbar_hot_only, p, 1.0)
    assert np.array_equal(np.nonzero(m[0, 0, 0])[0], hot) and not near.any()
    m, _ = O.nabla_mask(qbar[:, :, 1:], kbar, p, 0.3)
    z = (kbar[0, 0] @ qbar[0, 0, 1]) * 0.3
    pr = np.exp(z - z.max())
    pr /= pr.sum()
    kept = m[0, 0, 0] != 0
    srt = np.sort(pr)[::-1]
    k = int(kept.sum())
    assert pr[kept].sum() >= p and srt[:k - 1].sum() < p
    assert pr[kept].min() >= pr[~kept].max()
