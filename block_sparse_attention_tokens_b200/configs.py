"""Synthetic video-DiT attention workloads (shapes only, no arithmetic of the method).

Each workload is a token grid of ``frames x height x width`` latent tokens, a head
count and a head dimension, the block / tile geometry and the mask family that the
block-sparse attention path uses on it.  The shapes follow the video-DiT settings
the sparse-attention pages talk about (720p Sliding-Tile, 480p NABLA, 500-frame
720p radial, chunked autoregressive decode with anchor frames).

The generator recipe that fills these shapes with numbers lives in ``synth.py``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                      # position in the workload list (seed = 1000 + index)
    batch: int
    heads: int
    head_dim: int
    grid: Tuple[int, int, int]      # token grid (T, H, W) of the key/value sequence
    block: int                      # block size in tokens (q and k)
    mask: str                       # "sta" | "nabla" | "radial" | "ar"
    tile: Optional[Tuple[int, int, int]] = None     # 3D tile for the permute (None: raster order)
    window: Optional[Tuple[int, int, int]] = None   # STA window in tiles
    p: Optional[float] = None                       # NABLA cumulative-mass threshold
    strength: Optional[float] = None                # Fourier-locality strength (fixed)
    strength_range: Optional[Tuple[float, float]] = None  # per-head strength U(lo, hi)
    iid: bool = False                               # Q,K,V iid N(0,1), no locality
    q_frames: Optional[int] = None                  # AR: query chunk = last q_frames frames
    anchor_frames: Optional[int] = None             # AR: persistent anchor frames at the start
    recent_frames: Optional[int] = None             # AR: trailing frames kept dense
    extra: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def tokens_per_frame(self) -> int:
        return self.grid[1] * self.grid[2]

    @property
    def nk(self) -> int:
        return self.n_tokens

    @property
    def nq(self) -> int:
        if self.q_frames is not None:
            return self.q_frames * self.tokens_per_frame
        return self.n_tokens

    @property
    def seed(self) -> int:
        return 1000 + self.index


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def padded(n: int, block: int) -> int:
    return _ceil_div(n, block) * block


WORKLOADS = [
    # Tiny Sliding-Tile case: 4 blocks of 64 tokens, window covers every tile -> all ones.
    Workload(name="sta_tiny", index=0, batch=1, heads=2, head_dim=64, grid=(4, 8, 8),
             block=64, mask="sta", tile=(4, 4, 4), window=(1, 3, 3), iid=True),
    # Sliding-Tile attention on a 720p DiT latent grid.
    Workload(name="sta_720p", index=1, batch=1, heads=24, head_dim=128, grid=(30, 48, 80),
             block=384, mask="sta", tile=(6, 8, 8), window=(3, 3, 5), strength=1.5),
    # Dynamic NABLA mask on a 480p DiT latent grid, per-head locality strength.
    Workload(name="nabla_480p", index=2, batch=1, heads=40, head_dim=128, grid=(21, 30, 52),
             block=64, mask="nabla", tile=(4, 4, 4), p=0.9, strength_range=(0.5, 3.0)),
    # Radial energy-decay mask at 500 frames 720p (126 latent frames), raster token order.
    Workload(name="radial_long", index=3, batch=1, heads=12, head_dim=128, grid=(126, 45, 80),
             block=128, mask="radial", strength=2.0),
    # Autoregressive chunked decode: last 3 frames against a 60-frame cache,
    # anchors (first 3 frames) + last 6 frames dense + NABLA p=0.85 elsewhere.
    Workload(name="ar_decode", index=4, batch=1, heads=16, head_dim=128, grid=(60, 30, 52),
             block=64, mask="ar", p=0.85, strength=1.5, q_frames=3, anchor_frames=3,
             recent_frames=6),
]

# Extra parity cases (not benchmark lines).
EXTRA = [
    # NABLA united with a Sliding-Tile window on a 480p-like grid whose 4x4x4 tiles
    # coincide with the 64-token blocks (20x32x52 = 520 blocks).
    Workload(name="nabla_sta_480p", index=5, batch=1, heads=40, head_dim=128,
             grid=(20, 32, 52), block=64, mask="nabla_sta", tile=(4, 4, 4), window=(3, 3, 5),
             p=0.9, strength_range=(0.5, 3.0)),
    # SPADE-style per-head slicing on the 480p grid: SICS picks one of the 64-token
    # slice shapes per head, Q/K/V are permuted head by head with it, then the
    # NABLA mask over those slices.  Per-head axis stretches make the heads'
    # features vary along different axes, so the choices differ between heads.
    Workload(name="spade_480p", index=6, batch=1, heads=40, head_dim=128, grid=(21, 30, 52),
             block=64, mask="spade", p=0.9, strength_range=(1.0, 3.0),
             extra={"axis_stretch": 6.0}),
]

BY_NAME = {w.name: w for w in WORKLOADS + EXTRA}


def get(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    return BY_NAME[name_or_index]


# Slice-shape menus for SPADE scheme generation, one per block size: every shape
# holds `block` tokens -- a cube, a wide flat slab (one or two frames), a mixed
# slab and a tall thin column (many frames, a small spatial patch).
SICS_MENUS = {
    64: ((4, 4, 4), (1, 8, 8), (2, 4, 8), (16, 2, 2)),
    128: ((2, 8, 8), (1, 8, 16), (4, 4, 8), (32, 2, 2)),
    384: ((6, 8, 8), (1, 16, 24), (2, 12, 16), (24, 4, 4)),
}


def sics_menu(block: int):
    return SICS_MENUS[block]

