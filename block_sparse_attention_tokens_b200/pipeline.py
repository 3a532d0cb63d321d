"""The block-sparse video attention path, sequenced over the C ABI.

A ``Plan`` owns the device buffers of one workload and runs the whole path with
``step(q, k, v)``: tile permute of Q/K/V, block-mask generation (Sliding-Tile,
radial, NABLA or the autoregressive anchor/recent/NABLA composition), CSR
compaction, the block-sparse attention forward and the inverse permute of O.
Every step is a libbsa kernel; this module only allocates and orders calls.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import binding as B
from .configs import Workload


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


class Plan:
    """Buffers and call sequence for one workload on one device."""

    def __init__(self, w: Workload, device: torch.device = torch.device("cuda")):
        self.w = w
        self.dev = device
        Hh, D, Bt = w.heads, w.head_dim, w.batch
        self.nq, self.nk = w.nq, w.nk
        self.permuted = w.tile is not None
        if self.permuted:
            self.n_pad = ceil_div(w.n_tokens, w.block) * w.block
            self.qp = torch.empty((Bt, self.n_pad, Hh, D), dtype=torch.bfloat16, device=device)
            self.kp = torch.empty_like(self.qp)
            self.vp = torch.empty_like(self.qp)
            self.op = torch.empty_like(self.qp)
        self.QB, self.KB = ceil_div(self.nq, w.block), ceil_div(self.nk, w.block)
        if w.mask in ("sta", "radial"):
            self.list_heads = 1
            self.mask = torch.empty((self.QB, self.KB), dtype=torch.uint8, device=device)
        else:
            self.list_heads = Bt * Hh
            self.mask = torch.empty((Bt, Hh, self.QB, self.KB), dtype=torch.uint8, device=device)
            self.near = torch.zeros(1, dtype=torch.int32, device=device)
        if w.mask == "ar":
            self.nabla_ws = torch.empty(
                B.bsa_nabla_workspace_size(Bt, Hh, self.nq, self.nk, D, w.block),
                dtype=torch.uint8, device=device)
        if w.mask in ("nabla", "nabla_sta"):
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
        if w.tile is not None:
            g, t = w.grid, w.tile
            self.tile_grid = (ceil_div(g[0], t[0]), ceil_div(g[1], t[1]), ceil_div(g[2], t[2]))
        if w.mask == "nabla_sta":
            self.base_mask = torch.empty((self.QB, self.KB), dtype=torch.uint8, device=device)
        if w.mask == "ar":
            self.kb_range = ar_block_ranges(self.nk, w.tokens_per_frame, w.block, w.anchor_frames,
                                            w.recent_frames)

    # --- individual stages (each one or a few libbsa launches) ---
    def permute_inputs(self, q, k, v):
        w = self.w
        if w.mask in ("nabla", "nabla_sta"):
            # NABLA pools Q and K per block while they are permuted
            B.bsa_tile_permute_pool(q, w.grid, w.tile, self.n_pad, w.block, y=self.qp,
                                    pooled=self.qbar)
            B.bsa_tile_permute_pool(k, w.grid, w.tile, self.n_pad, w.block, y=self.kp,
                                    pooled=self.kbar)
            B.bsa_tile_permute(v, w.grid, w.tile, self.n_pad, y=self.vp)
            return
        for src, dst in ((q, self.qp), (k, self.kp), (v, self.vp)):
            B.bsa_tile_permute(src, w.grid, w.tile, self.n_pad, y=dst)

    def build_mask(self):
        w = self.w
        if w.mask == "sta":
            B.bsa_sta_mask(self.tile_grid, w.window, 0, mask=self.mask)
        elif w.mask == "radial":
            B.bsa_radial_mask(self.nk, w.tokens_per_frame, w.block, mask=self.mask)
        elif w.mask == "nabla":
            B.bsa_nabla_select(self.qbar, self.kbar, w.p, mask=self.mask, near_count=self.near)
        elif w.mask == "nabla_sta":
            B.bsa_sta_mask(self.tile_grid, w.window, 0, mask=self.base_mask)
            B.bsa_nabla_select(self.qbar, self.kbar, w.p, base_mask=self.base_mask,
                               mask=self.mask, near_count=self.near)
        elif w.mask == "ar":
            a_end, r_begin = self.kb_range
            B.bsa_nabla_mask(self._q, self._k, w.block, w.p, 0.0, a_end, r_begin, 1, nq=self.nq,
                             nk=self.nk, mask=self.mask, near_count=self.near, ws=self.nabla_ws)
        else:
            raise ValueError(w.mask)

    def compact(self):
        B.bsa_mask_compact(self.mask, row_ptr=self.row_ptr, col_idx=self.col_idx)

    def attention(self):
        w = self.w
        q, k, v = (self.qp, self.kp, self.vp) if self.permuted else (self._q, self._k, self._v)
        out = self.op if self.permuted else self.o
        B.bsa_attn_fwd(q, k, v, self.row_ptr, self.col_idx, w.block, w.block, self.list_heads,
                       nq=self.nq, nk=self.nk, o=out, lse=self.lse, ws=self.attn_ws)

    def untile(self):
        B.bsa_tile_untile(self.op, self.w.grid, self.w.tile, x=self.o)

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
        """One pass of the whole path.  Returns (O raster order, LSE in the path's token order)."""
        self._q, self._k, self._v = q, k, v
        if self.permuted:
            self.permute_inputs(q, k, v)
        self.build_mask()
        self.compact()
        self.attention()
        if self.permuted:
            self.untile()
        return self.o, self.lse

    def kernel_launches_per_step(self) -> int:
        """libbsa kernels one step launches (for the benchmark's launch count)."""
        n = 0
        if self.permuted:
            n += 3 + 1                   # permute Q, K, V and untile O
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
