"""The block-sparse video attention path, sequenced over the C ABI.

A ``Plan`` owns the device buffers of one workload and runs the whole path with
``step(q, k, v)``: tile permute of Q/K/V, block-mask generation (Sliding-Tile,
radial, NABLA or the autoregressive anchor/recent/NABLA composition), CSR
compaction, the block-sparse attention forward and the inverse permute of O.
The ``spade`` family first picks a slice shape per head by SICS and permutes each
head with its own shape before the NABLA mask.
Every step is a libbsa kernel; this module only allocates and orders calls.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import binding as B
from .configs import Workload, sics_menu


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def ar_block_ranges(n_tokens_k: int, tokens_per_frame: int, block: int, anchor_frames: int,
                    recent_frames: int) -> Tuple[int, int]:
    """Key-block range left to the dynamic selection in the autoregressive mask:
    blocks touching the anchor frames come before it, blocks touching the recent
    frames after it."""
    a_end = ceil_div(anchor_frames * tokens_per_frame, block)
    r_begin = (n_tokens_k - recent_frames * tokens_per_frame) // block
    return a_end, max(r_begin, a_end)


def qblock_range(rank: int, world: int, qblocks: int, granule: int = 1) -> Tuple[int, int]:
    """Query blocks [b0, b1) of rank `rank` when `world` ranks share `qblocks` query
    blocks of every head: the rows of the attention are independent given K and V,
    so a workload with too few heads to split evenly splits its query blocks
    instead, with no exchange.  The blocks go out in units of `granule` (the blocks
    of one 128-row attention q-tile, 128 // block for blocks under 128 tokens), so
    the ranks' q-tiles are the whole call's and the results bit-identical to it.
    Contiguous, every block once, unit counts within one."""
    if world < 1 or not 0 <= rank < world or granule < 1:
        raise ValueError(f"rank {rank} of {world}, granule {granule}")
    units = -(-qblocks // granule)
    u0, u1 = rank * units // world, (rank + 1) * units // world
    return min(qblocks, u0 * granule), min(qblocks, u1 * granule)


def head_range(rank: int, world: int, heads: int) -> Tuple[int, int]:
    """Heads [h0, h1) of rank `rank` when `world` ranks share `heads` heads: every
    (batch, head) row of the attention is independent given Q, K, V and the masks
    are per head, so the heads split with no exchange between ranks.  The ranges
    are contiguous, cover every head once and differ in size by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    return rank * heads // world, (rank + 1) * heads // world


class Plan:
    """Buffers and call sequence for one workload on one device.

    ``heads=(h0, h1)`` restricts the plan to that range of the workload's heads (a
    rank's share when the heads are split over GPUs).  ``step`` then takes either
    the whole-head tensors [B, N, H, D] -- the range is read in place through the
    library's token-row stride -- or tensors holding only the range's heads.

    ``qblocks=(b0, b1)`` (raster-order workloads only) restricts it to those query
    blocks: the plan's queries are rows [b0 * block, min(nq, b1 * block)) of every
    head, against all keys.  ``step`` takes Q with either all of the workload's
    query rows (the range is read in place) or only the range's, and writes O and
    LSE for the range (into the range's rows of a whole-O ``out``)."""

    def __init__(self, w: Workload, device: torch.device = torch.device("cuda"),
                 heads: Optional[Tuple[int, int]] = None,
                 qblocks: Optional[Tuple[int, int]] = None):
        self.w = w
        self.dev = device
        self.h0, self.h1 = (0, w.heads) if heads is None else heads
        if not 0 <= self.h0 < self.h1 <= w.heads:
            raise ValueError(f"head range {heads} of {w.heads} heads")
        Hh, D, Bt = self.h1 - self.h0, w.head_dim, w.batch
        self.heads = Hh
        self.nq, self.nk = w.nq, w.nk
        self.permuted = w.tile is not None or w.mask == "spade"
        qb_all = ceil_div(w.nq, w.block)
        self.qb0, self.qb1 = (0, qb_all) if qblocks is None else qblocks
        if not 0 <= self.qb0 < self.qb1 <= qb_all:
            raise ValueError(f"query-block range {qblocks} of {qb_all} blocks")
        if (self.qb0, self.qb1) != (0, qb_all):
            if self.permuted:
                raise ValueError("a query-block range needs a raster-order workload")
            if w.mask not in ("sta", "radial", "ar"):
                raise ValueError(f"no query-block range for the {w.mask} mask")
        self.q0 = self.qb0 * w.block                      # first query row of the plan
        self.nq = min(w.nq, self.qb1 * w.block) - self.q0
        if self.permuted:
            self.n_pad = ceil_div(w.n_tokens, w.block) * w.block
            self.qp = torch.empty((Bt, self.n_pad, Hh, D), dtype=torch.bfloat16, device=device)
            self.kp = torch.empty_like(self.qp)
            self.vp = torch.empty_like(self.qp)
            self.op = torch.empty_like(self.qp)
        self.QB, self.KB = ceil_div(self.nq, w.block), ceil_div(self.nk, w.block)
        if w.mask in ("sta", "radial"):
            self.list_heads = 1
            # static masks are built whole; the plan's query blocks are a row range
            self.mask_all = torch.empty((qb_all, self.KB), dtype=torch.uint8, device=device)
            self.mask = self.mask_all[self.qb0:self.qb1]
        else:
            self.list_heads = Bt * Hh
            self.mask = torch.empty((Bt, Hh, self.QB, self.KB), dtype=torch.uint8, device=device)
            self.near = torch.zeros(1, dtype=torch.int32, device=device)
        if w.mask == "ar":
            self.nabla_ws = torch.empty(
                B.bsa_nabla_workspace_size(Bt, Hh, self.nq, self.nk, D, w.block),
                dtype=torch.uint8, device=device)
        if w.mask == "spade":
            # per-head slice shapes chosen by SICS from the menu of the block size
            self.menu = sics_menu(w.block)
            self.scores = torch.empty((Bt, Hh, len(self.menu)), dtype=torch.float32, device=device)
            self.choice = torch.empty((Bt, Hh), dtype=torch.int32, device=device)
            self.sics_ws = torch.empty(max(1, B.bsa_sics_workspace_size(Bt, Hh, w.grid, self.menu)),
                                       dtype=torch.uint8, device=device)
            self.scheme_status = torch.zeros(1, dtype=torch.int32, device=device)
        if w.mask in ("nabla", "nabla_sta", "spade"):
            # block means come out of the fused permute of Q and K
            self.qbar = torch.empty((Bt, Hh, self.QB, D), dtype=torch.float32, device=device)
            self.kbar = torch.empty((Bt, Hh, self.KB, D), dtype=torch.float32, device=device)
        rows = self.list_heads * self.QB
        self.row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(rows * self.KB, dtype=torch.int32, device=device)
        self.attn_ws = torch.empty(
            B.bsa_attn_workspace_size(Bt, Hh, self.nq, self.nk, w.block, w.block, self.list_heads),
            dtype=torch.uint8, device=device)
        self.lse = torch.empty((Bt, Hh, self.nq), dtype=torch.float32, device=device)
        self.o = torch.empty((Bt, self.nq, Hh, D), dtype=torch.bfloat16, device=device)
        self.out = self.o
        if w.tile is not None:
            g, t = w.grid, w.tile
            self.tile_grid = (ceil_div(g[0], t[0]), ceil_div(g[1], t[1]), ceil_div(g[2], t[2]))
        if w.mask == "nabla_sta":
            self.base_mask = torch.empty((self.QB, self.KB), dtype=torch.uint8, device=device)
        if w.mask == "ar":
            self.kb_range = ar_block_ranges(self.nk, w.tokens_per_frame, w.block, w.anchor_frames,
                                            w.recent_frames)

    # --- individual stages (each one or a few libbsa launches) ---
    def _mine(self, t: torch.Tensor) -> torch.Tensor:
        """This plan's heads of a token tensor: a strided view of a whole-head
        tensor, or the tensor itself when it holds only the plan's heads."""
        if t.shape[2] == self.heads:
            return t
        if t.shape[2] == self.w.heads:
            return t[:, :, self.h0:self.h1]
        raise ValueError(f"tensor with {t.shape[2]} heads for a plan of heads "
                         f"[{self.h0}, {self.h1}) of {self.w.heads}")

    def _rows(self, t: torch.Tensor) -> torch.Tensor:
        """This plan's query rows of a query-side tensor [B, rows, H, D]: a row view
        of one holding all of the workload's query rows, or the tensor itself when
        it holds only the plan's."""
        if t.shape[1] == self.nq:
            return t
        if t.shape[1] == self.w.nq:
            return t[:, self.q0:self.q0 + self.nq]
        raise ValueError(f"tensor with {t.shape[1]} query rows for a plan of rows "
                         f"[{self.q0}, {self.q0 + self.nq}) of {self.w.nq}")

    def permute_inputs(self, q, k, v):
        w = self.w
        q, k, v = self._mine(q), self._mine(k), self._mine(v)
        if w.mask in ("nabla", "nabla_sta"):
            # NABLA pools Q and K per block while they are permuted
            B.bsa_tile_permute_pool(q, w.grid, w.tile, self.n_pad, w.block, y=self.qp,
                                    pooled=self.qbar)
            B.bsa_tile_permute_pool(k, w.grid, w.tile, self.n_pad, w.block, y=self.kp,
                                    pooled=self.kbar)
            B.bsa_tile_permute(v, w.grid, w.tile, self.n_pad, y=self.vp)
            return
        if w.mask == "spade":
            B.bsa_sics_scheme(q, k, w.grid, self.menu, scores=self.scores, choice=self.choice,
                              ws=self.sics_ws)
            for src, dst, pooled in ((q, self.qp, self.qbar), (k, self.kp, self.kbar),
                                     (v, self.vp, None)):
                B.bsa_scheme_permute(src, w.grid, self.menu, self.choice, self.n_pad, w.block,
                                     y=dst, pooled=pooled, device_status=self.scheme_status)
            return
        for src, dst in ((q, self.qp), (k, self.kp), (v, self.vp)):
            B.bsa_tile_permute(src, w.grid, w.tile, self.n_pad, y=dst)

    def build_mask(self):
        w = self.w
        if w.mask == "sta":
            B.bsa_sta_mask(self.tile_grid, w.window, 0, mask=self.mask_all)
        elif w.mask == "radial":
            B.bsa_radial_mask(self.nk, w.tokens_per_frame, w.block, mask=self.mask_all)
        elif w.mask in ("nabla", "spade"):
            B.bsa_nabla_select(self.qbar, self.kbar, w.p, mask=self.mask, near_count=self.near)
        elif w.mask == "nabla_sta":
            B.bsa_sta_mask(self.tile_grid, w.window, 0, mask=self.base_mask)
            B.bsa_nabla_select(self.qbar, self.kbar, w.p, base_mask=self.base_mask,
                               mask=self.mask, near_count=self.near)
        elif w.mask == "ar":
            a_end, r_begin = self.kb_range
            B.bsa_nabla_mask(self._rows(self._mine(self._q)), self._mine(self._k), w.block, w.p,
                             0.0, a_end,
                             r_begin, 1, nq=self.nq, nk=self.nk, mask=self.mask,
                             near_count=self.near, ws=self.nabla_ws)
        else:
            raise ValueError(w.mask)

    def compact(self):
        B.bsa_mask_compact(self.mask, row_ptr=self.row_ptr, col_idx=self.col_idx)

    def attention(self):
        w = self.w
        if self.permuted:
            q, k, v, out = self.qp, self.kp, self.vp, self.op
        else:
            q, k, v = self._rows(self._mine(self._q)), self._mine(self._k), self._mine(self._v)
            out = self._rows(self._mine(self.out))
        B.bsa_attn_fwd(q, k, v, self.row_ptr, self.col_idx, w.block, w.block, self.list_heads,
                       nq=self.nq, nk=self.nk, o=out, lse=self.lse, ws=self.attn_ws)

    def untile(self):
        if self.w.mask == "spade":
            B.bsa_scheme_untile(self.op, self.w.grid, self.menu, self.choice,
                                x=self._mine(self.out), device_status=self.scheme_status)
            return
        B.bsa_tile_untile(self.op, self.w.grid, self.w.tile, x=self._mine(self.out))

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             out: Optional[torch.Tensor] = None):
        """One pass of the whole path.  Returns (O raster order, LSE in the path's token
        order).  ``out`` (optional): a whole-head [B, nq, H, D] tensor whose heads of
        this plan receive O (in place); by default the plan's own O buffer."""
        self.set_output(out)
        self._q, self._k, self._v = q, k, v
        if self.permuted:
            self.permute_inputs(q, k, v)
        self.build_mask()
        self.compact()
        self.attention()
        if self.permuted:
            self.untile()
        return self.out, self.lse

    def capture(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                out: Optional[torch.Tensor] = None) -> "torch.cuda.CUDAGraph":
        """Records one ``step`` on these tensors into a CUDA graph and returns it.
        ``graph.replay()`` then re-runs the whole path -- every launch of the step,
        with no host work between them -- on whatever the same tensors hold; new
        inputs are copied into q, k, v in place.  One eager step runs first, outside
        the capture, so that every one-time setup of the library (kernel attributes,
        symbol addresses) is done before it."""
        self.step(q, k, v, out=out)
        torch.cuda.synchronize(self.dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.step(q, k, v, out=out)
        return graph

    def set_output(self, out: Optional[torch.Tensor] = None):
        """Where the next steps write O: a whole-head (and, with a query-block range,
        whole-row) tensor -- this plan's heads and rows of it -- or the plan's own
        buffer (None)."""
        self.out = self.o if out is None else out
        self._rows(self._mine(self.out))

    def kernel_launches_per_step(self) -> int:
        """libbsa kernels one step launches (for the benchmark's launch count)."""
        n = 0
        if self.permuted:
            n += 3 + 1                   # permute Q, K, V and untile O
        if self.w.mask == "spade":
            n += 2                       # SICS of every (tensor, shape) tile + the per-head pick
        n += {"nabla": 1, "nabla_sta": 2, "ar": 2}.get(self.w.mask, 1)   # mask kernels
        n += 3                           # compact: count, scan, fill
        n += 2                           # kept-list build + attention
        return n


def effective_flops(mask: torch.Tensor, nq: int, nk: int, block: int, head_dim: int,
                    batch_heads: int) -> float:
    """4 * D * (number of (query, key) token pairs inside kept blocks), all heads."""
    QB, KB = mask.shape[-2], mask.shape[-1]
    vq = torch.full((QB,), float(block), dtype=torch.float64, device=mask.device)
    vq[-1] = nq - (QB - 1) * block
    vk = torch.full((KB,), float(block), dtype=torch.float64, device=mask.device)
    vk[-1] = nk - (KB - 1) * block
    m = mask.reshape(-1, QB, KB).to(torch.float64)
    pairs = torch.einsum("hqk,q,k->", m, vq, vk).item()
    if m.shape[0] == 1:
        pairs *= batch_heads
    return 4.0 * head_dim * pairs


class PagedARCache:
    """Paged K/V cache of an autoregressive run with persistent anchors.

    The key sequence grows a chunk (``chunk_frames`` frames) at a time.  K and V
    live in pools of 128-token pages with one page table per batch; the pools hold
    only ``pool_pages_per_batch`` pages per batch -- anchors, the recent window,
    ``budget`` middle pages and room for the next chunk -- not the whole sequence.
    A chunk step is ``append`` (write the chunk's K/V to free pages), ``attend``
    (mask = anchors + recent forced, NABLA over the resident middle blocks; paged
    attention) and ``evict`` (page importance from the chunk's pooled queries, keep
    the ``budget`` most important middle pages, free the rest).  Every step is a
    libbsa kernel; the free list lives on the host (one small read-back per chunk).
    """

    def __init__(self, w: Workload, max_tokens: int, budget: int, device=torch.device("cuda")):
        self.w, self.dev = w, device
        Bt, Hh, D = w.batch, w.heads, w.head_dim
        self.page = B.KV_PAGE
        self.block = w.block
        self.S = w.tokens_per_frame
        self.budget = budget
        self.max_pages = ceil_div(max_tokens, self.page)
        self.anchor_tokens = w.anchor_frames * self.S
        self.recent_tokens = w.recent_frames * self.S
        chunk_tokens = (w.q_frames or 1) * self.S
        per_batch = (ceil_div(self.anchor_tokens, self.page) + ceil_div(self.recent_tokens, self.page)
                     + budget + ceil_div(chunk_tokens, self.page) + 3)
        self.pool_pages_per_batch = min(per_batch, self.max_pages)
        n_pool = Bt * self.pool_pages_per_batch
        self.k_pool = torch.zeros((n_pool, self.page, Hh, D), dtype=torch.bfloat16, device=device)
        self.v_pool = torch.zeros_like(self.k_pool)
        self.table_host = torch.full((Bt, self.max_pages), -1, dtype=torch.int32)
        self.table = self.table_host.to(device)
        self.free = list(range(n_pool))
        self.freed = torch.empty(Bt * self.max_pages, dtype=torch.int32, device=device)
        self.freed_count = torch.zeros(1, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.n_tokens = 0
        self.attn_ws = None

    def resident_bytes(self) -> int:
        """Bytes of K and V the cache holds now (resident pages only)."""
        pages = int((self.table_host >= 0).sum())
        w = self.w
        return 2 * pages * self.page * w.heads * w.head_dim * 2

    def pool_bytes(self) -> int:
        return 2 * self.k_pool.numel() * self.k_pool.element_size()

    def append(self, k: torch.Tensor, v: torch.Tensor):
        Bt, n_new = k.shape[0], k.shape[1]
        first, last = self.n_tokens, self.n_tokens + n_new
        if ceil_div(last, self.page) > self.max_pages:
            raise ValueError("sequence longer than the cache was sized for")
        for b in range(Bt):
            for lp in range(first // self.page, ceil_div(last, self.page)):
                if self.table_host[b, lp] < 0:
                    if not self.free:
                        raise RuntimeError("KV pool exhausted")
                    self.table_host[b, lp] = self.free.pop()
        self.table.copy_(self.table_host)
        B.bsa_kv_write(k, first, self.table, self.k_pool, self.status)
        B.bsa_kv_write(v, first, self.table, self.v_pool, self.status)
        self.n_tokens = last

    def attend(self, q: torch.Tensor, p: float, scale: float = 0.0):
        """Attention of the chunk's queries q [B, nq, H, D] over the cache.  Returns
        (O, LSE, mask); keeps the pooled means for ``evict``."""
        w = self.w
        Bt, nq, Hh, D = q.shape
        nk, blk = self.n_tokens, self.block
        QB, KB = ceil_div(nq, blk), ceil_div(nk, blk)
        self.qbar = torch.empty((Bt, Hh, QB, D), dtype=torch.float32, device=self.dev)
        self.kbar = torch.empty((Bt, Hh, KB, D), dtype=torch.float32, device=self.dev)
        B.bsa_block_pool(q, nq, blk, 0, QB, self.qbar)
        B.bsa_block_pool(self.k_pool, nk, blk, 0, KB, self.kbar, page_table=self.table, batch=Bt)
        self.allowed = B.bsa_kv_resident_blocks(self.table, blk, KB)
        self.kb_range = ar_block_ranges(nk, self.S, blk, w.anchor_frames, w.recent_frames)
        a_end, r_begin = self.kb_range
        mask, self.near = B.bsa_nabla_select(self.qbar, self.kbar, p, scale, a_end, r_begin, 1,
                                             key_allowed=self.allowed)
        row_ptr, col_idx = B.bsa_mask_compact(mask)
        size = B.bsa_attn_workspace_size(Bt, Hh, nq, nk, blk, blk, Bt * Hh)
        if self.attn_ws is None or self.attn_ws.numel() < size:
            self.attn_ws = torch.empty(size, dtype=torch.uint8, device=self.dev)
        o, lse, _ = B.bsa_attn_fwd_paged(q, self.k_pool, self.v_pool, self.table, nk, row_ptr,
                                         col_idx, blk, blk, Bt * Hh, scale=scale, ws=self.attn_ws)
        return o, lse, mask

    def evict(self, scale: float = 0.0):
        """Keeps the anchors, the recent window and the `budget` most important middle
        pages (importance from the last ``attend``); frees the other pages."""
        nk, blk = self.n_tokens, self.block
        n_pages = ceil_div(nk, self.page)
        a_end, r_begin = self.kb_range
        scores = B.bsa_kv_page_scores(self.qbar, self.kbar, a_end, r_begin, blk, n_pages,
                                      scale=scale, key_allowed=self.allowed)
        anchor_pages = ceil_div(self.anchor_tokens, self.page)
        recent_begin = max(anchor_pages, (nk - self.recent_tokens) // self.page)
        self.freed_count.zero_()
        B.bsa_kv_keep_pages(scores, anchor_pages, recent_begin, self.budget, self.table,
                            self.freed, self.freed_count)
        self.table_host.copy_(self.table.cpu())
        n = int(self.freed_count.item())
        self.free.extend(self.freed[:n].cpu().tolist())
        self.last_scores = scores
        self.last_pages = (anchor_pages, recent_begin)

