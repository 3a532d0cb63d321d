"""CPU oracle for block-sparse 3D spatio-temporal video attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Plain, slow, float64 NumPy written for reading against the pages:

* "Fast Video Generation with Sliding Tile Attention" explainer
  (aibr.jp/archives/60739), section 2 (tile-wise vs token-wise windows) and
  section 3 (3D locality, tiles as the unit of work, hardware-aware kernel).
* "Radial Attention: O(n log n) Sparse Attention with Energy Decay for Long Video
  Generation" explainer (aibr.jp/archives/112136), sections 1-3 (static mask,
  window shrinking with temporal distance, O(n log n) cost) and section 4
  (9x less attention compute at 500 frames 720p).
* "NABLA (Neighborhood Adaptive Block-Level Attention)" explainer
  (aibr.jp/archives/124678), section 3 (mean-pool Q and K per block, full
  attention on the pooled tokens, CDF threshold, binary block mask).
* "Sparse Forcing: Native Trainable Sparse Attention for Real-time Autoregressive
  Diffusion Video Generation" summary (gist.science/ja/paper/2604.21221),
  part 2 (persistent anchors, recent frames looked at closely, sparse selection
  elsewhere).
* SPADE summary (gist.science/ja/paper/2608.03335), solution parts 1 (a menu of
  3D slice shapes) and 2 (scheme generation with SICS, the sum of intra-block
  cosine similarities).

Where the pages leave a step open, the reading taken is marked READING and is
the contract the CUDA path is held to.  Parity status: every function here is
pinned by ``tests/test_oracle_*.py`` against brute-force enumeration, closed
forms, library routines or hand-computed golden values; the radial constants,
the STA edge rule (clip vs shift) and the NABLA logit scale are readings that
the pages do not fix (no page prints them), so their *parameters* are unpinned
by the pages even though the implementation of each reading is pinned.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# ---------------------------------------------------------------------------
# 1. 3D tile permutation
# ---------------------------------------------------------------------------

def tile_order(grid: Tuple[int, int, int], tile: Tuple[int, int, int]) -> np.ndarray:
    """Tile-major token order of a T x H x W grid (STA explainer, section 3).

    The grid is cut into tT x tH x tW tiles; tokens are stably sorted by
    (tile index in raster order over the tile grid, position inside the tile in
    raster order).  Edge tiles may be smaller (READING: ragged edge tiles are
    not padded; padding only appears at the end of the whole sequence).
    Returns perm with perm[p] = raster index of the token placed at position p.
    """
    T, H, W = grid
    tT, tH, tW = tile
    nH, nW = ceil_div(H, tH), ceil_div(W, tW)
    idx = np.arange(T * H * W, dtype=np.int64)
    t, h, w = idx // (H * W), (idx // W) % H, idx % W
    tile_id = ((t // tT) * nH + (h // tH)) * nW + (w // tW)
    inner = ((t % tT) * tH + (h % tH)) * tW + (w % tW)
    key = tile_id * (tT * tH * tW) + inner
    return np.argsort(key, kind="stable")


def tile_permute(x: np.ndarray, perm: np.ndarray, n_pad: int) -> np.ndarray:
    """y[:, p] = x[:, perm[p]] for p < N; rows N..n_pad-1 are zero.  x: [B, N, ...]."""
    n = perm.shape[0]
    y = np.zeros((x.shape[0], n_pad) + x.shape[2:], dtype=x.dtype)
    y[:, :n] = x[:, perm]
    return y


def tile_untile(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of tile_permute: x[:, perm[p]] = y[:, p]; the padded tail is dropped."""
    n = perm.shape[0]
    x = np.empty((y.shape[0], n) + y.shape[2:], dtype=y.dtype)
    x[:, perm] = y[:, :n]
    return x


def scheme_permute(x: np.ndarray, grid: Tuple[int, int, int], shapes, choice: np.ndarray,
                   n_pad: int) -> np.ndarray:
    """Per-head slicing (SPADE summary, solution parts 1 and 3): head h of batch b
    is put in the tile order of the slice shape shapes[choice[b, h]].

    x: [B, N, H, D] raster; returns y [B, n_pad, H, D], rows N.. zero.
    y[b, p, h] = x[b, perm_bh[p], h] with perm_bh = tile_order(grid, shape of (b, h)).
    """
    Bt, n, H = x.shape[0], x.shape[1], x.shape[2]
    y = np.zeros((Bt, n_pad) + x.shape[2:], dtype=x.dtype)
    for b in range(Bt):
        for h in range(H):
            perm = tile_order(grid, tuple(shapes[int(choice[b, h])]))
            y[b, :n, h] = x[b, perm, h]
    return y


def scheme_untile(y: np.ndarray, grid: Tuple[int, int, int], shapes, choice: np.ndarray) -> np.ndarray:
    """Inverse of scheme_permute: x[b, perm_bh[p], h] = y[b, p, h] for p < N."""
    n = grid[0] * grid[1] * grid[2]
    Bt, H = y.shape[0], y.shape[2]
    x = np.empty((Bt, n) + y.shape[2:], dtype=y.dtype)
    for b in range(Bt):
        for h in range(H):
            perm = tile_order(grid, tuple(shapes[int(choice[b, h])]))
            x[b, perm, h] = y[b, :n, h]
    return x


# ---------------------------------------------------------------------------
# 2. Sliding Tile Attention mask
# ---------------------------------------------------------------------------

def sta_axis_keep(n: int, w: int, shift: bool = False) -> np.ndarray:
    """Kept (a, a2) tile pairs along one axis of length n for a window of w tiles.

    STA explainer, sections 2-3: each query tile attends to a window of
    neighbouring tiles, counted in tiles rather than tokens.
    READING (default, ``shift=False``): the window is centred on the query tile,
    offsets -floor((w-1)/2) .. +ceil((w-1)/2), and clipped at the grid edge.
    Alternative (``shift=True``): the window keeps its full width and slides
    inward at the edges, start = clamp(a - floor((w-1)/2), 0, n - w).
    """
    keep = np.zeros((n, n), dtype=bool)
    lo_off, hi_off = (w - 1) // 2, w // 2
    for a in range(n):
        if shift:
            start = min(max(a - lo_off, 0), max(n - w, 0))
            lo, hi = start, min(start + w, n) - 1
        else:
            lo, hi = max(a - lo_off, 0), min(a + hi_off, n - 1)
        keep[a, lo:hi + 1] = True
    return keep


def sta_tile_mask(tile_grid: Tuple[int, int, int], window: Tuple[int, int, int],
                  shift: bool = False) -> np.ndarray:
    """Tile-level STA mask [n_tiles, n_tiles] (uint8), tiles in raster order.

    Query tile (a, b, c) keeps key tile (a2, b2, c2) iff every axis keeps its pair.
    """
    nT, nH, nW = tile_grid
    kt, kh, kw = (sta_axis_keep(n, w, shift) for n, w in zip(tile_grid, window))
    n = nT * nH * nW
    out = np.zeros((n, n), dtype=np.uint8)
    for a in range(nT):
        for b in range(nH):
            for c in range(nW):
                q = (a * nH + b) * nW + c
                out[q] = (kt[a][:, None, None] & kh[b][None, :, None] & kw[c][None, None, :]).reshape(-1)
    return out


# ---------------------------------------------------------------------------
# 3. Radial (energy-decay) mask
# ---------------------------------------------------------------------------

def _radial_params(dist: int, S: int, B: int):
    """Window parameters for frame distance dist >= 2 (Radial explainer, section 3).

    READING: the spatial window is dense for |dt| <= 1; for frame distance dist,
    r = floor(log2 dist) and the half-width is S / 2^(r+1) tokens (S tokens per
    frame, distance measured along the raster index inside a frame), i.e. the
    window halves each time the distance doubles.  Once that half-width would drop
    below half a block, the half-width stays at B/2 and only every 2^c-th frame is
    kept, c the smallest integer with S * 2^c >= B * 2^r, which keeps the
    halving of density per doubling of distance and at least one block per kept
    frame.  Returns (frame_kept, twice_half_width_num, twice_half_width_den)
    meaning: keep iff frame_kept and 2*|ds| * den < num.
    """
    dist = int(dist)
    r = dist.bit_length() - 1
    if S >= B * (1 << r):
        # |ds| < S / 2^(r+1)  <=>  2|ds| * 2^r < S
        return True, S, 1 << r
    c = 0
    while S * (1 << c) < B * (1 << r):
        c += 1
    if dist % (1 << c) != 0:
        return False, 0, 1
    # |ds| < B/2  <=>  2|ds| < B
    return True, B, 1


def radial_token_keep(fq: int, sq: int, fk: int, sk: int, S: int, B: int) -> bool:
    """Token-level radial rule for query (frame fq, in-frame index sq) and key (fk, sk)."""
    dist = abs(fq - fk)
    if dist <= 1:
        return True
    kept, num, den = _radial_params(dist, S, B)
    return kept and 2 * abs(sq - sk) * den < num


def _block_segments(b: int, block: int, n: int, S: int):
    """(frame, first in-frame index, last in-frame index) pieces of token block b."""
    lo, hi = b * block, min((b + 1) * block, n)
    segs = []
    while lo < hi:
        f = lo // S
        end = min(hi, (f + 1) * S)
        segs.append((f, lo - f * S, end - 1 - f * S))
        lo = end
    return segs


def radial_block_mask(n_tokens: int, tokens_per_frame: int, block: int) -> np.ndarray:
    """Block-level radial mask [NB, NB] (uint8), raster token order.

    A block pair is kept iff some token pair in it is kept by ``radial_token_keep``
    (block mask = OR over its token pairs).  Evaluated per pair of per-frame
    segments: the closest spatial distance between two index intervals is their
    gap max(0, b0 - a1, a0 - b1).
    """
    S = tokens_per_frame
    nb = ceil_div(n_tokens, block)
    segs = [_block_segments(b, block, n_tokens, S) for b in range(nb)]
    out = np.zeros((nb, nb), dtype=np.uint8)
    for qb in range(nb):
        for kb in range(nb):
            keep = False
            for fq, a0, a1 in segs[qb]:
                for fk, b0, b1 in segs[kb]:
                    dist = abs(fq - fk)
                    if dist <= 1:
                        keep = True
                        break
                    kept, num, den = _radial_params(dist, S, block)
                    gap = max(0, b0 - a1, a0 - b1)
                    if kept and 2 * gap * den < num:
                        keep = True
                        break
                if keep:
                    break
            out[qb, kb] = keep
    return out


def radial_block_mask_fast(n_tokens: int, tokens_per_frame: int, block: int) -> np.ndarray:
    """Same mask as ``radial_block_mask``, vectorised over key blocks for large grids.

    Blocks span at most ceil(block / S) + 1 frames; each (query segment, key
    segment) slot is evaluated with array arithmetic and OR-ed.
    """
    S = tokens_per_frame
    nb = ceil_div(n_tokens, block)
    lo = np.arange(nb, dtype=np.int64) * block
    hi = np.minimum(lo + block, n_tokens)          # exclusive
    max_segs = ceil_div(block, S) + 1
    seg_f, seg_a, seg_b, seg_ok = [], [], [], []
    for j in range(max_segs):
        f = lo // S + j
        start = np.maximum(lo, f * S)
        end = np.minimum(hi, (f + 1) * S)
        ok = start < end
        seg_f.append(f)
        seg_a.append(start - f * S)
        seg_b.append(end - 1 - f * S)
        seg_ok.append(ok)
    max_dist = ceil_div(n_tokens, S) + max_segs + 1
    frame_kept = np.zeros(max_dist + 1, dtype=bool)
    num = np.zeros(max_dist + 1, dtype=np.int64)
    den = np.ones(max_dist + 1, dtype=np.int64)
    for dist in range(max_dist + 1):
        if dist <= 1:
            frame_kept[dist] = True
            num[dist] = -1
            continue
        k, nu, de = _radial_params(dist, S, block)
        frame_kept[dist], num[dist], den[dist] = k, nu, de
    out = np.zeros((nb, nb), dtype=bool)
    for qb in range(nb):
        row = np.zeros(nb, dtype=bool)
        for i in range(max_segs):
            if not seg_ok[i][qb]:
                continue
            fq, a0, a1 = seg_f[i][qb], seg_a[i][qb], seg_b[i][qb]
            for j in range(max_segs):
                ok = seg_ok[j]
                dist = np.abs(seg_f[j] - fq)
                gap = np.maximum(0, np.maximum(seg_a[j] - a1, a0 - seg_b[j]))
                near = dist <= 1
                far = frame_kept[dist] & (2 * gap * den[dist] < num[dist])
                row |= ok & (near | far)
        out[qb] = row
    return out.astype(np.uint8)


# ---------------------------------------------------------------------------
# 4. NABLA dynamic mask
# ---------------------------------------------------------------------------

def nabla_pool(x: np.ndarray, block: int, n_valid: int) -> np.ndarray:
    """Mean of each block's tokens, per head (NABLA explainer, section 3).

    x: [B, N_pad, H, D] (float64), N_pad a multiple of ``block``.
    READING: the mean is over the block's valid tokens (index < n_valid), so the
    zero padding at the end of the sequence does not dilute the last block.
    Returns [B, H, NB, D].
    """
    Bn, n_pad, H, D = x.shape
    nb = n_pad // block
    out = np.zeros((Bn, H, nb, D), dtype=np.float64)
    for b in range(nb):
        lo, hi = b * block, min((b + 1) * block, n_valid)
        out[:, :, b, :] = x[:, lo:hi].mean(axis=1)
    return out


def nabla_select_row(probs: np.ndarray, p: float):
    """Smallest set of entries whose probability mass reaches p (NABLA section 3).

    Entries are taken in descending probability, ties to the lower index
    (READING); the kept set is the shortest such prefix whose cumulative sum is
    >= p.  p >= 1 keeps every entry.
    Returns (kept_indices, prefix_sums_of_sorted_probs, k_star).
    """
    n = probs.shape[0]
    order = np.argsort(-probs, kind="stable")
    cum = np.cumsum(probs[order])
    if p >= 1.0:
        k_star = n
    else:
        hit = np.nonzero(cum >= p)[0]
        k_star = int(hit[0]) + 1 if hit.size else n
    return order[:k_star], cum, k_star, order


def nabla_mask(qbar: np.ndarray, kbar: np.ndarray, p: float, scale: float,
               kb_begin: int = 0, kb_end: Optional[int] = None, force_outside: int = 0,
               near_tol: float = 1e-5, tie_tol: float = 1e-5,
               key_allowed: Optional[np.ndarray] = None):
    """Per-(batch, head) NABLA block mask from pooled queries and keys.

    Logits z[qb, kb] = qbar[qb] . kbar[kb] * scale (READING: the same 1/sqrt(D)
    scale as the attention itself), softmax over the key blocks in
    [kb_begin, kb_end), then ``nabla_select_row`` per query block.  Key blocks
    outside the range are set to ``force_outside`` (used by the autoregressive
    composition, where those blocks are forced on).
    Returns (mask [B, H, QB, KB] uint8, near [B, H, QB] bool).  ``near`` marks rows
    where a prefix sum next to the cut lies within ``near_tol`` of p, or where
    the last kept and first dropped probabilities tie within ``tie_tol``
    (relative): on those rows a float32 evaluation may legitimately choose
    differently.
    ``key_allowed`` ([B, KB] bool, optional): key blocks that may be chosen at all.
    READING (Sparse Forcing summary, part 2: the cache keeps only the important
    past): blocks evicted from a paged cache are not candidates -- they are left
    out of the softmax and never selected.
    """
    Bn, H, QB, D = qbar.shape
    KB = kbar.shape[2]
    kb_end = KB if kb_end is None else kb_end
    mask = np.zeros((Bn, H, QB, KB), dtype=np.uint8)
    near = np.zeros((Bn, H, QB), dtype=bool)
    if force_outside:
        mask[:, :, :, :kb_begin] = 1
        mask[:, :, :, kb_end:] = 1
    if kb_end <= kb_begin:
        return mask, near
    for b in range(Bn):
        cand = np.arange(kb_begin, kb_end)
        if key_allowed is not None:
            cand = cand[key_allowed[b, kb_begin:kb_end]]
        if cand.size == 0:
            continue
        for h in range(H):
            z = (qbar[b, h] @ kbar[b, h, cand].T) * scale                    # [QB, n_cand]
            z = z - z.max(axis=1, keepdims=True)
            e = np.exp(z)
            probs = e / e.sum(axis=1, keepdims=True)
            for qb in range(QB):
                kept, cum, k_star, order = nabla_select_row(probs[qb], p)
                mask[b, h, qb, cand[kept]] = 1
                if p < 1.0:
                    c_last = cum[k_star - 1]
                    c_prev = cum[k_star - 2] if k_star >= 2 else 0.0
                    flag = abs(c_last - p) < near_tol or abs(c_prev - p) < near_tol
                    n = probs.shape[1]
                    if k_star < n:
                        a, bb = probs[qb, order[k_star - 1]], probs[qb, order[k_star]]
                        flag = flag or abs(a - bb) <= tie_tol * max(a, bb)
                    near[b, h, qb] = flag
    return mask, near


# ---------------------------------------------------------------------------
# 5. Autoregressive chunk mask: anchors + recent + NABLA elsewhere
# ---------------------------------------------------------------------------

def ar_block_ranges(n_tokens_k: int, tokens_per_frame: int, block: int,
                    anchor_frames: int, recent_frames: int) -> Tuple[int, int]:
    """(first middle key block, first recent key block) of the AR chunk mask.

    Sparse Forcing summary, part 2: the anchor frames at the start are kept as
    persistent memory, the most recent frames are looked at closely, and only
    the needed blocks are chosen in between.  READING: key blocks that touch an
    anchor token (index < anchor_frames * S) are anchors; key blocks that touch
    the last recent_frames frames are recent; the rest form the middle range.
    """
    S = tokens_per_frame
    a_end = ceil_div(anchor_frames * S, block)
    r_begin = (n_tokens_k - recent_frames * S) // block
    return a_end, max(r_begin, a_end)


def ar_mask(qbar, kbar, p, scale, n_tokens_k, tokens_per_frame, block, anchor_frames,
            recent_frames):
    """Anchors and recent blocks forced on; NABLA (CDF over the middle range only,
    READING: renormalised over the blocks still to be chosen) decides the rest."""
    a_end, r_begin = ar_block_ranges(n_tokens_k, tokens_per_frame, block, anchor_frames,
                                     recent_frames)
    return nabla_mask(qbar, kbar, p, scale, a_end, r_begin, force_outside=1)


def nabla_sta_mask(qbar, kbar, p, scale, sta_mask):
    """NABLA selection united with a Sliding-Tile window (NABLA explainer,
    sections 1-2: NABLA is combined with STA and other sparse patterns).
    READING: the union of the two block masks, the NABLA cut taken over all key
    blocks as usual; the window mask is shared by every batch and head."""
    m, near = nabla_mask(qbar, kbar, p, scale)
    return (m | (sta_mask[None, None] != 0)).astype(np.uint8), near


# ---------------------------------------------------------------------------
# 6. Compaction of a block mask into per-row kept lists
# ---------------------------------------------------------------------------

def mask_to_csr(mask2d: np.ndarray):
    """CSR of a [rows, KB] 0/1 mask: row_ptr[rows+1], col_idx ascending per row."""
    rows = mask2d.shape[0]
    counts = (mask2d != 0).sum(axis=1)
    row_ptr = np.zeros(rows + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([np.nonzero(mask2d[r])[0] for r in range(rows)]) if rows else \
        np.zeros(0, dtype=np.int64)
    return row_ptr, col_idx.astype(np.int64)


# ---------------------------------------------------------------------------
# 7. Block-sparse attention (the plain definition)
# ---------------------------------------------------------------------------

def dense_masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                           allowed: np.ndarray, scale: float):
    """softmax(q k^T * scale + M) v with M = 0 where allowed, -inf elsewhere.

    q: [Nq, D], k, v: [Nk, D], allowed: [Nq, Nk] bool.  Rows with nothing allowed
    give O = 0 and LSE = -inf.  Returns (O [Nq, D], LSE [Nq]) (natural log).
    """
    s = (q @ k.T) * scale
    s = np.where(allowed, s, NEG_INF)
    mx = s.max(axis=1)
    empty = ~np.isfinite(mx)
    mx_safe = np.where(empty, 0.0, mx)
    e = np.exp(s - mx_safe[:, None])
    l = e.sum(axis=1)
    o = np.where(empty[:, None], 0.0, (e @ v) / np.where(empty, 1.0, l)[:, None])
    lse = np.where(empty, NEG_INF, mx_safe + np.log(np.where(empty, 1.0, l)))
    return o, lse


def token_mask_from_blocks(mask2d: np.ndarray, nq: int, nk: int, block_q: int,
                           block_k: int) -> np.ndarray:
    """Token-level allowed matrix: (i, j) allowed iff block pair (i//bq, j//bk) is kept."""
    qi = np.arange(nq) // block_q
    kj = np.arange(nk) // block_k
    return mask2d[qi][:, kj] != 0


def block_sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                           block_q: int, block_k: int, scale: Optional[float] = None,
                           rows: Optional[Sequence[int]] = None):
    """Attention restricted to kept (query block, key block) pairs.

    STA explainer section 3 / NABLA section 3 / Radial section 3: the method
    computes exactly softmax(QK^T / sqrt(D) + M) V where M is 0 on kept block
    pairs (and keys j < Nk) and -inf elsewhere.  Masked blocks contribute
    exp(-inf) = 0, so only kept blocks are evaluated; the arithmetic per row is
    the plain definition in float64.

    q: [B, Nq, H, D]; k, v: [B, Nk, H, D]; mask: [Hm, QB, KB] with Hm == 1 (same
    mask for every batch and head) or Hm == B * H (index b * H + h).
    ``rows``: optional query rows to evaluate (others are left NaN).
    Returns (O [B, Nq, H, D], LSE [B, H, Nq]).
    """
    Bn, nq, H, D = q.shape
    nk = k.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.full((Bn, nq, H, D), np.nan)
    lse = np.full((Bn, H, nq), np.nan)
    rows = np.arange(nq) if rows is None else np.asarray(rows, dtype=np.int64)
    qbs = rows // block_q
    for b in range(Bn):
        for h in range(H):
            m = mask[0 if mask.shape[0] == 1 else b * H + h]
            for qb in np.unique(qbs):
                sel = rows[qbs == qb]
                kept = np.nonzero(m[qb])[0]
                cols = np.concatenate([np.arange(kb * block_k, min((kb + 1) * block_k, nk))
                                       for kb in kept]) if kept.size else np.zeros(0, np.int64)
                if cols.size == 0:
                    o[b, sel, h] = 0.0
                    lse[b, h, sel] = NEG_INF
                    continue
                s = (q[b, sel, h] @ k[b, cols, h].T) * scale
                mx = s.max(axis=1, keepdims=True)
                e = np.exp(s - mx)
                l = e.sum(axis=1, keepdims=True)
                o[b, sel, h] = (e @ v[b, cols, h]) / l
                lse[b, h, sel] = (mx + np.log(l))[:, 0]
    return o, lse


# ---------------------------------------------------------------------------
# 8. Backward of the block-sparse attention (training)
# ---------------------------------------------------------------------------

def block_sparse_attention_backward(q, k, v, do, mask, block_q, block_k, scale=None, rows=None,
                                    cols=None):
    """Gradients of O = softmax(Q K^T * scale + M) V with respect to Q, K, V.

    The Radial explainer (section 4, training cost), the NABLA explainer
    (section 4, training and inference speed-up) and the Sparse Forcing summary
    (trainable sparse attention) train through the sparse attention; the
    gradients are those of the same masked softmax, written out per row:
        P = softmax(S),  dV = P^T dO,  dP = dO V^T,
        dS = P * (dP - rowsum(dO * O)),  dQ = dS K * scale,  dK = dS^T Q * scale,
    evaluated over each row's kept key blocks only (masked entries have P = 0).
    q: [B, Nq, H, D]; k, v: [B, Nk, H, D]; do: [B, Nq, H, D]; mask: [Hm, QB, KB].
    ``rows`` (optional): evaluate only these query rows -- dq is exact on them (0
    elsewhere) and dk, dv hold only their contributions (for sampled checks at
    full size).
    ``cols`` (optional): key rows whose dk and dv are wanted -- only query blocks
    that keep a block holding one of them are evaluated (each over its whole kept
    row, since P and rowsum(dO * O) need every kept key), so dk and dv are exact
    on these keys; dq, and dk / dv at other keys, hold only the evaluated rows'
    contributions.
    Returns (dq, dk, dv) with the shapes of q, k, v.
    """
    Bn, nq, H, D = q.shape
    nk = k.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    want_kb = None if cols is None else np.unique(np.asarray(cols, dtype=np.int64) // block_k)
    for b in range(Bn):
        for h in range(H):
            m = mask[0 if mask.shape[0] == 1 else b * H + h]
            for qb in range(m.shape[0]):
                rows_b = np.arange(qb * block_q, min((qb + 1) * block_q, nq))
                if rows is not None:
                    rows_b = np.intersect1d(rows_b, np.asarray(rows))
                kept = np.nonzero(m[qb])[0]
                if kept.size == 0 or rows_b.size == 0:
                    continue
                if want_kb is not None and np.intersect1d(kept, want_kb).size == 0:
                    continue
                rows_ = rows_b
                keys = np.concatenate([np.arange(kb * block_k, min((kb + 1) * block_k, nk))
                                       for kb in kept])
                s = (q[b, rows_, h] @ k[b, keys, h].T) * scale
                s = s - s.max(axis=1, keepdims=True)
                p = np.exp(s)
                p /= p.sum(axis=1, keepdims=True)
                o = p @ v[b, keys, h]
                g = do[b, rows_, h]
                dv[b, keys, h] += p.T @ g
                dp = g @ v[b, keys, h].T
                ds = p * (dp - (g * o).sum(axis=1, keepdims=True))
                dq[b, rows_, h] += (ds @ k[b, keys, h]) * scale
                dk[b, keys, h] += (ds.T @ q[b, rows_, h]) * scale
    return dq, dk, dv


# ---------------------------------------------------------------------------
# SPADE: slice-shape menu and SICS scheme generation
# ---------------------------------------------------------------------------

def tile_tokens(grid: Tuple[int, int, int], tile: Tuple[int, int, int], index: int) -> np.ndarray:
    """Raster token indices (ascending) of tile `index`, tiles in raster order over
    the tile grid, ragged at the grid's far edges (the same tiling as tile_order)."""
    T, H, W = grid
    tT, tH, tW = tile
    nT, nH, nW = ceil_div(T, tT), ceil_div(H, tH), ceil_div(W, tW)
    a, rem = divmod(index, nH * nW)
    b, c = divmod(rem, nW)
    ts = np.arange(a * tT, min(T, a * tT + tT))
    hs = np.arange(b * tH, min(H, b * tH + tH))
    ws = np.arange(c * tW, min(W, c * tW + tW))
    return ((ts[:, None, None] * H + hs[None, :, None]) * W + ws[None, None, :]).reshape(-1)


def sics_blocks(x: np.ndarray, grid: Tuple[int, int, int], tile: Tuple[int, int, int]) -> np.ndarray:
    """SICS of every block of one slicing (SPADE summary, solution part 2).

    A block is one tile of shape `tile`; its SICS is the sum over all ordered token
    pairs (i, j) of the block, i == j included, of the cosine similarity of the two
    tokens' vectors, per head.  A zero vector has no direction and contributes 0
    (READING).  x: [B, N, H, D] in raster token order.  Returns [B, H, n_tiles].
    """
    Bn, N, Hh, D = x.shape
    nt = ceil_div(grid[0], tile[0]) * ceil_div(grid[1], tile[1]) * ceil_div(grid[2], tile[2])
    out = np.zeros((Bn, Hh, nt))
    for t in range(nt):
        idx = tile_tokens(grid, tile, t)
        for b in range(Bn):
            for h in range(Hh):
                v = x[b, idx, h, :]
                norm = np.sqrt((v * v).sum(axis=1))
                u = np.where(norm[:, None] > 0, v / np.where(norm > 0, norm, 1.0)[:, None], 0.0)
                out[b, h, t] = (u @ u.T).sum()      # every pairwise cosine, summed
    return out


def sics_scheme(q: np.ndarray, k: np.ndarray, grid: Tuple[int, int, int],
                shapes: Sequence[Tuple[int, int, int]]):
    """Per-head slicing choice from a menu of block shapes (SPADE summary, parts 1-2).

    READING: a slicing is better the more its blocks agree internally.  Its score for
    head h is the mean cosine similarity over the intra-block token pairs of Q and K,
        score = (sum_b SICS_Q(b) + sum_b SICS_K(b)) / (2 * sum_b n_b^2),
    n_b the block's token count; the head takes the highest-scoring shape (ties: the
    earlier menu entry).  Returns (scores [B, H, n_shapes], choice [B, H] int).
    """
    Bn, _, Hh, _ = q.shape
    scores = np.zeros((Bn, Hh, len(shapes)))
    for si, shape in enumerate(shapes):
        nt = ceil_div(grid[0], shape[0]) * ceil_div(grid[1], shape[1]) * ceil_div(grid[2], shape[2])
        pairs = sum(len(tile_tokens(grid, shape, t)) ** 2 for t in range(nt))
        total = sics_blocks(q, grid, shape).sum(axis=2) + sics_blocks(k, grid, shape).sum(axis=2)
        scores[:, :, si] = total / (2.0 * pairs)
    choice = np.zeros((Bn, Hh), dtype=np.int64)
    for b in range(Bn):
        for h in range(Hh):
            best = 0
            for si in range(1, len(shapes)):
                if scores[b, h, si] > scores[b, h, best]:
                    best = si
            choice[b, h] = best
    return scores, choice


# ---------------------------------------------------------------------------
# Paged KV cache with persistent anchors (Sparse Forcing summary, part 2)
# ---------------------------------------------------------------------------
#
# READING: the cache holds K and V in fixed-size pages of a physical pool, one
# page table per batch maps each logical page (page_tokens consecutive tokens of
# the key sequence) to a physical page or to -1 once evicted.  Anchor pages (those
# touching the anchor frames) are persistent, the pages of the most recent frames
# are kept, and of the pages in between only a fixed budget of the most important
# survive, importance being the pooled attention mass the latest queries put on
# the page -- the same pooled distribution NABLA selects from.


def paged_view(pool: np.ndarray, page_table: np.ndarray, page_tokens: int, n_tokens: int):
    """Logical [B, n_tokens, H, D] tensor of a paged cache and its residency.

    pool: [P, page_tokens, H, D]; page_table: [B, n_pages] (physical page or -1).
    Token j of batch b is row j % page_tokens of page page_table[b, j // page_tokens];
    tokens of evicted pages read as 0 and are not resident.
    """
    Bn, n_pages = page_table.shape
    _, _, H, D = pool.shape
    out = np.zeros((Bn, n_tokens, H, D))
    resident = np.zeros((Bn, n_tokens), dtype=bool)
    for b in range(Bn):
        for pg in range(n_pages):
            lo, hi = pg * page_tokens, min((pg + 1) * page_tokens, n_tokens)
            if lo >= hi or page_table[b, pg] < 0:
                continue
            out[b, lo:hi] = pool[page_table[b, pg], :hi - lo]
            resident[b, lo:hi] = True
    return out, resident


def resident_blocks(page_table: np.ndarray, page_tokens: int, block: int, n_tokens: int) -> np.ndarray:
    """[B, KB] bool: key block kb is resident iff the page holding it is (pages hold
    whole blocks: page_tokens is a multiple of the block)."""
    KB = ceil_div(n_tokens, block)
    pages = (np.arange(KB) * block) // page_tokens
    return page_table[:, pages] >= 0


def paged_block_sparse_attention(q, k_pool, v_pool, page_table, page_tokens, nk, mask, block_q,
                                 block_k, scale=None, rows=None):
    """Block-sparse attention over a paged cache: the plain block-sparse attention
    of the logical K/V with every block on an evicted page dropped from the mask.
    mask: [Hm, QB, KB] with Hm == 1 or B * H.  Returns (O, LSE) like
    block_sparse_attention."""
    Bn, _, H, _ = q.shape
    k, _ = paged_view(k_pool, page_table, page_tokens, nk)
    v, _ = paged_view(v_pool, page_table, page_tokens, nk)
    res = resident_blocks(page_table, page_tokens, block_k, nk)            # [B, KB]
    full = np.broadcast_to(mask, (Bn * H,) + mask.shape[1:]) if mask.shape[0] == 1 else mask
    m = np.array(full, dtype=np.uint8).reshape(Bn, H, mask.shape[1], mask.shape[2])
    m = (m * res[:, None, None, :]).reshape(Bn * H, mask.shape[1], mask.shape[2])
    return block_sparse_attention(q, k, v, m.astype(np.uint8), block_q, block_k, scale, rows)


def kv_page_scores(qbar, kbar, scale, kb_begin, kb_end, block, page_tokens, n_pages,
                   key_allowed=None):
    """Importance of each logical page: the pooled attention probability (softmax of
    qbar . kbar * scale over the candidate key blocks of [kb_begin, kb_end), as in
    nabla_mask) summed over heads and query blocks and over the page's blocks.
    Pages without candidate blocks score 0.  Returns [B, n_pages]."""
    Bn, H, QB, _ = qbar.shape
    out = np.zeros((Bn, n_pages))
    for b in range(Bn):
        cand = np.arange(kb_begin, kb_end)
        if key_allowed is not None:
            cand = cand[key_allowed[b, kb_begin:kb_end]]
        if cand.size == 0:
            continue
        for h in range(H):
            z = (qbar[b, h] @ kbar[b, h, cand].T) * scale
            z = z - z.max(axis=1, keepdims=True)
            e = np.exp(z)
            probs = e / e.sum(axis=1, keepdims=True)
            mass = probs.sum(axis=0)                                      # per candidate block
            for i, kb in enumerate(cand):
                out[b, (kb * block) // page_tokens] += mass[i]
    return out


def kv_keep_pages(scores, resident, anchor_pages, recent_begin, budget):
    """Pages the cache keeps: every page below anchor_pages (persistent anchors) and
    from recent_begin on (recent frames), and of the resident pages in between the
    `budget` highest scores (ties: the lower page).  Returns keep [B, n_pages] bool."""
    Bn, n_pages = scores.shape
    keep = np.zeros((Bn, n_pages), dtype=bool)
    keep[:, :anchor_pages] = True
    keep[:, recent_begin:] = True
    for b in range(Bn):
        mid = [pg for pg in range(anchor_pages, recent_begin) if resident[b, pg]]
        mid.sort(key=lambda pg: (-scores[b, pg], pg))
        for pg in mid[:budget]:
            keep[b, pg] = True
    return keep

