"""Pins of the paged-KV-cache oracle (persistent anchors, recent pages, a budget of
important middle pages) and of NABLA restricted to resident key blocks."""
import math

import numpy as np

import oracle as O


def _pool_from(k, page_tokens, perm):
    """Physical pool holding logical page pg at physical page perm[pg]."""
    Bn, n, H, D = k.shape
    n_pages = math.ceil(n / page_tokens)
    pool = np.full((Bn * n_pages, page_tokens, H, D), np.nan)
    table = np.zeros((Bn, n_pages), dtype=np.int64)
    for b in range(Bn):
        for pg in range(n_pages):
            phys = perm[b * n_pages + pg]
            lo, hi = pg * page_tokens, min((pg + 1) * page_tokens, n)
            pool[phys, :hi - lo] = k[b, lo:hi]
            table[b, pg] = phys
    return pool, table


def test_paged_view_identity_shuffled_and_evicted():
    rng = np.random.default_rng(0)
    k = rng.standard_normal((2, 300, 2, 8))
    n_pages = 3
    for perm in (np.arange(6), rng.permutation(6)):
        pool, table = _pool_from(k, 128, perm)
        got, res = O.paged_view(pool, table, 128, 300)
        assert np.array_equal(got, k) and res.all()
    table[1, 1] = -1
    got, res = O.paged_view(pool, table, 128, 300)
    assert np.all(got[1, 128:256] == 0) and not res[1, 128:256].any()
    assert np.array_equal(got[0], k[0]) and res[1, :128].all() and res[1, 256:].all()


def test_paged_attention_equals_plain_and_drops_evicted_pages():
    rng = np.random.default_rng(1)
    Bn, H, nq, nk, D, blk = 1, 2, 100, 512, 16, 64
    q = rng.standard_normal((Bn, nq, H, D))
    k = rng.standard_normal((Bn, nk, H, D))
    v = rng.standard_normal((Bn, nk, H, D))
    mask = np.ones((1, 2, 8), dtype=np.uint8)
    perm = rng.permutation(4)
    kp, table = _pool_from(k, 128, perm)
    vp, _ = _pool_from(v, 128, perm)
    o1, l1 = O.paged_block_sparse_attention(q, kp, vp, table, 128, nk, mask, blk, blk)
    o2, l2 = O.block_sparse_attention(q, k, v, mask, blk, blk)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    # page 2 (tokens 256..383) holds keys that would dominate every score; evicting it
    # must give the dense softmax over the other tokens
    k2 = k.copy()
    k2[:, 256:384] = 50.0 * q[:, :1].mean(axis=1, keepdims=True)
    kp2, _ = _pool_from(k2, 128, perm)
    table_e = table.copy()
    table_e[0, 2] = -1
    o3, _ = O.paged_block_sparse_attention(q, kp2, vp, table_e, 128, nk, mask, blk, blk)
    allowed = np.ones((nq, nk), dtype=bool)
    allowed[:, 256:384] = False
    for h in range(H):
        ref, _ = O.dense_masked_attention(q[0, :, h], k[0, :, h], v[0, :, h], allowed,
                                          1 / math.sqrt(D))
        assert np.allclose(o3[0, :, h], ref, atol=1e-12)


def test_page_scores_sum_to_rows_and_follow_a_dominant_block():
    rng = np.random.default_rng(2)
    Bn, H, QB, KB, D = 1, 3, 5, 12, 8
    qbar = rng.standard_normal((Bn, H, QB, D))
    kbar = rng.standard_normal((Bn, H, KB, D))
    s = O.kv_page_scores(qbar, kbar, 0.3, 2, 10, 64, 128, 6)
    assert abs(s.sum() - H * QB) < 1e-9                       # each softmax row sums to 1
    assert s[0, 0] == 0 and s[0, 5] == 0                      # pages outside [2, 10)
    kbar[:, :, 7] = 50.0 * qbar[:, :, :, :].mean(axis=2)      # block 7 (page 3) dominates
    qbar[:] = qbar.mean(axis=2, keepdims=True)
    s = O.kv_page_scores(qbar, kbar, 1.0, 2, 10, 64, 128, 6)
    assert abs(s[0, 3] - H * QB) < 1e-6
    allowed = np.ones((Bn, KB), dtype=bool)
    allowed[0, 7] = False                                     # evicted: not a candidate
    s2 = O.kv_page_scores(qbar, kbar, 1.0, 2, 10, 64, 128, 6, key_allowed=allowed)
    assert abs(s2.sum() - H * QB) < 1e-9 and s2[0, 3] < H * QB * 0.9


def test_keep_pages_anchors_recent_and_budget():
    rng = np.random.default_rng(3)
    n_pages, a, r, budget = 40, 4, 32, 10
    scores = rng.random((2, n_pages))
    scores[0, 10] = scores[0, 11] = 5.0                       # a tie: lower page first
    resident = np.ones((2, n_pages), dtype=bool)
    resident[1, 5:15] = False
    keep = O.kv_keep_pages(scores, resident, a, r, budget)
    for b in range(2):
        assert keep[b, :a].all() and keep[b, r:].all()
        mid = np.arange(a, r)
        kept = mid[keep[b, mid]]
        dropped = mid[~keep[b, mid] & resident[b, mid]]
        assert len(kept) == min(budget, resident[b, mid].sum())
        assert not (keep[b] & ~resident[b] & (np.arange(n_pages) >= a) & (np.arange(n_pages) < r)).any()
        if len(dropped):
            assert scores[b, kept].min() >= scores[b, dropped].max()
    keep1 = O.kv_keep_pages(scores, resident, a, r, 1)
    assert keep1[0, 10] and not keep1[0, 11]


def test_nabla_with_allowed_blocks_equals_nabla_on_the_allowed_subset():
    rng = np.random.default_rng(4)
    Bn, H, QB, KB, D = 1, 2, 6, 20, 16
    qbar = rng.standard_normal((Bn, H, QB, D))
    kbar = rng.standard_normal((Bn, H, KB, D))
    allowed = rng.random((Bn, KB)) < 0.6
    m, _ = O.nabla_mask(qbar, kbar, 0.8, 0.25, 3, 17, 1, key_allowed=allowed)
    cand = np.arange(3, 17)[allowed[0, 3:17]]
    sub, _ = O.nabla_mask(qbar, kbar[:, :, cand], 0.8, 0.25)
    assert np.array_equal(m[..., cand], sub)
    others = np.setdiff1d(np.arange(3, 17), cand)
    assert not m[..., others].any()
    assert m[..., :3].all() and m[..., 17:].all()             # forced outside the range
    full, _ = O.nabla_mask(qbar, kbar, 0.8, 0.25, 3, 17, 1)
    m_all, _ = O.nabla_mask(qbar, kbar, 0.8, 0.25, 3, 17, 1,
                            key_allowed=np.ones((Bn, KB), dtype=bool))
    assert np.array_equal(full, m_all)
