"""GPU parity of the paged KV cache (page writes, paged pooling, residency, NABLA
restricted to resident blocks, page importance, the keep policy and attention
through a page table) against the float64 oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu
PAGE = B.KV_PAGE


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy()


def make_table(batch, n_pages, n_pool, seed, evict=()):
    rng = np.random.default_rng(seed)
    phys = rng.permutation(n_pool)[:batch * n_pages].reshape(batch, n_pages)
    table = phys.astype(np.int32)
    for b, pg in evict:
        table[b, pg] = -1
    return table


def test_kv_write_roundtrip_and_paged_pool():
    Bn, H, D, n = 2, 3, 128, 700
    n_pages = math.ceil(n / PAGE)
    x = torch.randn(Bn, n, H, D).to(torch.bfloat16)
    table = make_table(Bn, n_pages, 16, seed=1)
    pool = torch.zeros(16, PAGE, H, D, dtype=torch.bfloat16, device="cuda")
    tab = torch.from_numpy(table).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xc = x.cuda()
    B.bsa_kv_write(xc[:, :300].contiguous(), 0, tab, pool, status)
    B.bsa_kv_write(xc[:, 300:].contiguous(), 300, tab, pool, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    view, res = O.paged_view(_bits(pool).astype(np.float64), table, PAGE, n)
    assert res.all() and np.array_equal(view.astype(np.int16), _bits(x))
    # block means through the page table and of the contiguous tensor
    blk = 64
    KB = math.ceil(n / blk)
    out = torch.zeros(Bn, H, KB, D, dtype=torch.float32, device="cuda")
    B.bsa_block_pool(pool, n, blk, 0, KB, out, page_table=tab, batch=Bn)
    out2 = torch.zeros_like(out)
    B.bsa_block_pool(xc, n, blk, 3, KB - 3, out2)
    torch.cuda.synchronize()
    xpad = np.zeros((Bn, KB * blk, H, D))
    xpad[:, :n] = to64(x)
    ref = O.nabla_pool(xpad, blk, n)
    assert np.max(np.abs(out.cpu().double().numpy() - ref)) < 2e-5
    assert np.max(np.abs(out2.cpu().double().numpy()[:, :, 3:] - ref[:, :, 3:])) < 2e-5
    assert np.all(out2.cpu().numpy()[:, :, :3] == 0)
    # a row whose page is not assigned is reported, not written
    tab2 = tab.clone()
    tab2[0, 1] = -1
    B.bsa_kv_write(xc[:, 128:130].contiguous(), 128, tab2, pool, status)
    torch.cuda.synchronize()
    assert status.item() == 1


@pytest.mark.parametrize("Bn,H,D,nq,nk,blk", [(1, 2, 128, 300, 1000, 64), (2, 2, 64, 257, 777, 128),
                                              (1, 3, 128, 128, 4096, 64)])
def test_paged_attention_matches_oracle_and_the_contiguous_kernel(Bn, H, D, nq, nk, blk):
    g = torch.Generator().manual_seed(nq + nk)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    n_pages = math.ceil(nk / PAGE)
    n_pool = Bn * n_pages + 3
    QB, KB = math.ceil(nq / blk), math.ceil(nk / blk)
    mask = synth.random_mask(Bn * H * QB, KB, 0.5, seed=blk + nk).reshape(Bn * H, QB, KB)
    mask[0, 0] = 0
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    kpool = torch.zeros((n_pool, PAGE, H, D), dtype=torch.bfloat16, device="cuda")
    vpool = torch.zeros((n_pool, PAGE, H, D), dtype=torch.bfloat16, device="cuda")
    table = make_table(Bn, n_pages, n_pool, seed=nk)
    tab = torch.from_numpy(table).cuda()
    B.bsa_kv_write(k.cuda(), 0, tab, kpool)
    B.bsa_kv_write(v.cuda(), 0, tab, vpool)
    # pool pages nobody maps hold large values: reading one would show
    used = set(table.ravel().tolist())
    for pg in range(n_pool):
        if pg not in used:
            kpool[pg] = 30.0
            vpool[pg] = 30.0
    o1, l1, ws = B.bsa_attn_fwd_paged(q.cuda(), kpool, vpool, tab, nk, rp, ci, blk, blk, Bn * H)
    o2, l2, _ = B.bsa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), rp, ci, blk, blk, Bn * H)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    # same kernel, same tiles: bit-identical to the contiguous layout
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # evict two pages of batch 0: their blocks drop out
    table_e = table.copy()
    table_e[0, 1] = -1
    table_e[0, n_pages - 1] = -1
    o3, l3, ws = B.bsa_attn_fwd_paged(q.cuda(), kpool, vpool, torch.from_numpy(table_e).cuda(), nk,
                                      rp, ci, blk, blk, Bn * H)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    kp64 = to64(kpool.cpu())
    vp64 = to64(vpool.cpu())
    ro, rl = O.paged_block_sparse_attention(to64(q), kp64, vp64, table_e, PAGE, nk, mask, blk, blk)
    D_ = D
    assert_attention_close(to64(o3).reshape(-1, D_), l3.cpu().numpy().astype(np.float64)
                           .transpose(0, 2, 1).reshape(-1), ro.reshape(-1, D_),
                           rl.transpose(0, 2, 1).reshape(-1), what="paged, evicted pages")


def test_resident_blocks_and_nabla_restricted_to_them():
    Bn, H, QB, KB, D = 2, 3, 9, 40, 128
    blk = 64
    n_pages = KB * blk // PAGE
    table = make_table(Bn, n_pages, 64, seed=7, evict=[(0, 3), (0, 4), (1, 10), (1, 0)])
    allowed = B.bsa_kv_resident_blocks(torch.from_numpy(table).cuda(), blk, KB)
    torch.cuda.synchronize()
    ref_allowed = O.resident_blocks(table, PAGE, blk, KB * blk)
    assert np.array_equal(allowed.cpu().numpy() != 0, ref_allowed)
    rng = np.random.default_rng(8)
    qbar = rng.standard_normal((Bn, H, QB, D)).astype(np.float32)
    kbar = rng.standard_normal((Bn, H, KB, D)).astype(np.float32)
    mask, _ = B.bsa_nabla_select(torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), 0.85,
                                 0.0, 5, 34, 1, key_allowed=allowed)
    torch.cuda.synchronize()
    ref, near = O.nabla_mask(qbar.astype(np.float64), kbar.astype(np.float64), 0.85,
                             1 / math.sqrt(D), 5, 34, 1, key_allowed=ref_allowed)
    got = mask.cpu().numpy()
    differs = np.any(got != ref, axis=-1)
    assert not (differs & ~near).any()
    assert not got[0][..., [6, 7, 8, 9]].any()    # the blocks of evicted pages 3, 4 of batch 0
    # p = 1 keeps exactly the allowed blocks of the range
    m1, _ = B.bsa_nabla_select(torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), 1.0,
                               0.0, 5, 34, 0, key_allowed=allowed)
    torch.cuda.synchronize()
    exp = np.zeros((Bn, KB), dtype=np.uint8)
    exp[:, 5:34] = ref_allowed[:, 5:34]
    assert np.array_equal(m1.cpu().numpy(), np.broadcast_to(exp[:, None, None, :], m1.shape))


def test_page_scores_and_keep_policy():
    Bn, H, QB, KB, D, blk = 2, 4, 7, 96, 128, 64
    n_pages = KB * blk // PAGE
    rng = np.random.default_rng(9)
    qbar = rng.standard_normal((Bn, H, QB, D)).astype(np.float32)
    kbar = (0.5 * rng.standard_normal((Bn, H, KB, D))).astype(np.float32)
    table = make_table(Bn, n_pages, 200, seed=10, evict=[(0, 20), (1, 21), (1, 22)])
    tab = torch.from_numpy(table).cuda()
    allowed = B.bsa_kv_resident_blocks(tab, blk, KB)
    scores = B.bsa_kv_page_scores(torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(),
                                  6, 80, blk, n_pages, key_allowed=allowed)
    torch.cuda.synchronize()
    ref = O.kv_page_scores(qbar.astype(np.float64), kbar.astype(np.float64), 1 / math.sqrt(D), 6, 80,
                           blk, PAGE, n_pages,
                           key_allowed=O.resident_blocks(table, PAGE, blk, KB * blk))
    got = scores.cpu().double().numpy()
    # fp32 softmax probabilities (relative error ~1e-6) summed over H * QB rows
    assert np.max(np.abs(got - ref)) <= 2e-5 * H * QB
    anchor, recent, budget = 3, 40, 12
    freed = torch.full((Bn * (recent - anchor),), -7, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = table.copy()
    B.bsa_kv_keep_pages(scores, anchor, recent, budget, tab, freed, count)
    torch.cuda.synchronize()
    after = tab.cpu().numpy()
    # the decision on the kernel's own scores, by the oracle's rule
    keep = O.kv_keep_pages(got, before >= 0, anchor, recent, budget)
    assert np.array_equal(after >= 0, keep & (before >= 0))
    assert np.array_equal(after[keep & (before >= 0)], before[keep & (before >= 0)])
    n = count.item()
    evicted = before[(before >= 0) & ~keep]
    assert n == evicted.size
    assert sorted(freed.cpu().numpy()[:n].tolist()) == sorted(evicted.tolist())


def test_paged_ar_cache_decode_loop_matches_the_oracle():
    """Four chunks of an autoregressive run through PagedARCache (append, attend,
    evict) against an oracle simulation of the same cache."""
    import dataclasses
    from block_sparse_attention_tokens_b200 import configs
    from block_sparse_attention_tokens_b200.pipeline import PagedARCache
    w = dataclasses.replace(configs.get("ar_decode"), heads=2, grid=(12, 8, 16))
    S, blk, p = w.tokens_per_frame, w.block, w.p
    chunk = w.q_frames * S
    q, k, v, _ = synth.generate(1, w.heads, w.head_dim, w.grid, seed=21, strength=1.5,
                                q_token_ids=np.arange(w.n_tokens))
    budget = 2
    cache = PagedARCache(w, w.n_tokens, budget)
    scale = 1 / math.sqrt(w.head_dim)
    resident_pages = np.zeros(math.ceil(w.n_tokens / PAGE), dtype=bool)
    q64, k64, v64 = to64(q), to64(k), to64(v)
    for c in range(w.n_tokens // chunk):
        lo, hi = c * chunk, (c + 1) * chunk
        cache.append(k[:, lo:hi].contiguous().cuda(), v[:, lo:hi].contiguous().cuda())
        resident_pages[lo // PAGE: math.ceil(hi / PAGE)] = True
        qc = q[:, lo:hi].contiguous().cuda()
        o, lse, mask = cache.attend(qc, p)
        torch.cuda.synchronize()
        assert cache.status.item() == 0
        nk = hi
        n_pages = math.ceil(nk / PAGE)
        # GPU residency so far must be the oracle's
        assert np.array_equal(cache.table_host.numpy()[0, :n_pages] >= 0, resident_pages[:n_pages])
        table = np.where(resident_pages[:n_pages], np.arange(n_pages), -1)[None].astype(np.int64)
        allowed = O.resident_blocks(table, PAGE, blk, nk)
        QB, KB = math.ceil(chunk / blk), math.ceil(nk / blk)
        qpad = np.zeros((1, QB * blk, w.heads, w.head_dim))
        qpad[:, :chunk] = q64[:, lo:hi]
        kpad = np.zeros((1, KB * blk, w.heads, w.head_dim))
        kpad[:, :nk] = k64[:, :nk]
        qbar, kbar = O.nabla_pool(qpad, blk, chunk), O.nabla_pool(kpad, blk, nk)
        a_end, r_begin = O.ar_block_ranges(nk, S, blk, w.anchor_frames, w.recent_frames)
        ref_mask, near = O.nabla_mask(qbar, kbar, p, scale, a_end, r_begin, 1, key_allowed=allowed)
        got_mask = mask.cpu().numpy()
        differs = np.any(got_mask != ref_mask, axis=-1)
        assert not (differs & ~near).any(), f"chunk {c}: mask rows differ away from the threshold"
        # attention over the resident pages, rows whose mask row is not near the cut
        m_eff = (ref_mask * allowed[:, None, None, :]).reshape(w.heads, QB, KB).astype(np.uint8)
        ro, rl = O.block_sparse_attention(q64[:, lo:hi], k64[:, :nk], v64[:, :nk], m_eff, blk, blk)
        og, lg = to64(o), lse.cpu().numpy().astype(np.float64)
        for h in range(w.heads):
            rows = np.nonzero(~np.repeat(near[0, h] | differs[0, h], blk)[:chunk])[0]
            assert_attention_close(og[0, rows, h], lg[0, h, rows], ro[0, rows, h], rl[0, h, rows],
                                   what=f"chunk {c} head {h}")
        # importance scores and the keep decision (taken on the kernel's own scores)
        cache.evict()
        torch.cuda.synchronize()
        ref_scores = O.kv_page_scores(qbar, kbar, scale, a_end, r_begin, blk, PAGE, n_pages,
                                      key_allowed=allowed)
        got_scores = cache.last_scores.cpu().double().numpy()
        assert np.max(np.abs(got_scores - ref_scores)) <= 2e-5 * w.heads * QB
        anchor_pages, recent_begin = cache.last_pages
        keep = O.kv_keep_pages(got_scores, resident_pages[None, :n_pages], anchor_pages, recent_begin,
                               budget)
        resident_pages[:n_pages] &= keep[0]
        assert np.array_equal(cache.table_host.numpy()[0, :n_pages] >= 0, resident_pages[:n_pages])
    # the cache ends with anchors + recent + budget pages, fewer than the plain cache
    assert cache.resident_bytes() < 2 * w.n_tokens * w.heads * w.head_dim * 2
