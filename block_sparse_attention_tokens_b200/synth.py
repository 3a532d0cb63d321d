"""Seeded synthetic inputs for the block-sparse video attention path.

This module only draws numbers; it holds none of the attention, mask or permute
arithmetic.  Both the CUDA path (through tests and the benchmark) and the CPU
oracle take their inputs from here.

Recipe (one call per workload, ``numpy.random.default_rng(seed)``, seed = 1000 + index):

1. ``omega``  (16, 3)  ~ N(0, 4^2)         frequencies of 16 random Fourier features
2. ``phi``    (16,)    ~ U[0, 2*pi)         their phases
3. per-head strength s_h: fixed, or U(lo, hi) drawn in head order
4. ``W_q[h]`` (16, D)  ~ N(0, 1/16) for h = 0..H-1, then ``W_k[h]`` likewise
4b. only with an axis stretch r: ``a[h]`` (H, 3) = exp(U(-ln r, ln r)), per-head
    scales of the (t, h, w) coordinates (heads whose features vary fastest along
    different axes)
5. noise for Q, then K, then V: standard normal float32 of shape (B, N, H, D)

Position features: token i of a T x H x W grid in raster order sits at
x = (t/(T-1), h/(H-1), w/(W-1)) (0 on an axis of length 1) and F(x) = cos(omega x + phi)
(with a stretch: F_h(x) = cos(omega (a[h] * x) + phi)).
Q = noise + s_h * F(x) W_q[h], K = noise + s_h * F(x) W_k[h], V = noise (iid N(0,1)).
The float32 values are rounded to bfloat16 (round to nearest even).  Tokens are
returned in raster order, layout [B, N, H, D].
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import configs as _configs

N_FEATURES = 16


def raster_positions(grid: Tuple[int, int, int], token_ids: np.ndarray) -> np.ndarray:
    """Normalised (t, h, w) coordinates of raster-order token indices, shape (n, 3)."""
    T, H, W = grid
    t = token_ids // (H * W)
    h = (token_ids // W) % H
    w = token_ids % W
    out = np.empty((token_ids.shape[0], 3), dtype=np.float64)
    for j, (c, n) in enumerate(((t, T), (h, H), (w, W))):
        out[:, j] = c / (n - 1) if n > 1 else 0.0
    return out


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def generate(batch: int, heads: int, head_dim: int, grid: Tuple[int, int, int], seed: int,
             strength: Optional[float] = None,
             strength_range: Optional[Tuple[float, float]] = None,
             iid: bool = False,
             q_token_ids: Optional[np.ndarray] = None,
             axis_stretch: Optional[float] = None):
    """Draw (Q, K, V) as bfloat16 CPU tensors [B, N, H, D] following the module recipe.

    ``q_token_ids`` selects the raster positions of the query tokens (default: all
    tokens of the grid); keys and values always cover the whole grid.
    Returns (q, k, v, meta) with meta holding the strengths actually used.
    """
    rng = np.random.default_rng(seed)
    T, Hh, Ww = grid
    n = T * Hh * Ww
    k_ids = np.arange(n, dtype=np.int64)
    q_ids = k_ids if q_token_ids is None else np.asarray(q_token_ids, dtype=np.int64)
    nq = q_ids.shape[0]

    omega = rng.normal(0.0, 4.0, size=(N_FEATURES, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=N_FEATURES)
    if strength_range is not None:
        s = rng.uniform(strength_range[0], strength_range[1], size=heads)
    elif strength is not None:
        s = np.full(heads, float(strength))
    else:
        s = np.zeros(heads)
    wq = np.stack([rng.normal(0.0, 0.25, size=(N_FEATURES, head_dim)) for _ in range(heads)])
    wk = np.stack([rng.normal(0.0, 0.25, size=(N_FEATURES, head_dim)) for _ in range(heads)])
    stretch = None
    if axis_stretch is not None:
        lr = math.log(axis_stretch)
        stretch = np.exp(rng.uniform(-lr, lr, size=(heads, 3)))

    def with_features(noise: np.ndarray, ids: np.ndarray, w: np.ndarray) -> np.ndarray:
        if iid:
            return noise
        pos = raster_positions(grid, ids)
        feats = np.cos(pos @ omega.T + phi)                                 # (n, 16)
        for h in range(heads):
            if stretch is not None:
                feats = np.cos((pos * stretch[h]) @ omega.T + phi)
            add = (feats @ (s[h] * w[h])).astype(np.float32)               # (n, D)
            noise[:, :, h, :] += add[None, :, :]
        return noise

    q = with_features(rng.standard_normal((batch, nq, heads, head_dim), dtype=np.float32), q_ids, wq)
    qt = _to_bf16(q)
    del q
    k = with_features(rng.standard_normal((batch, n, heads, head_dim), dtype=np.float32), k_ids, wk)
    kt = _to_bf16(k)
    del k
    v = rng.standard_normal((batch, n, heads, head_dim), dtype=np.float32)
    vt = _to_bf16(v)
    del v
    return qt, kt, vt, {"strength": s, "omega": omega, "phi": phi, "stretch": stretch}


def workload_inputs(w: "_configs.Workload"):
    """Q, K, V for a named workload (raster token order, [B, N, H, D] bfloat16)."""
    q_ids = None
    if w.q_frames is not None:
        n = w.n_tokens
        q_ids = np.arange(n - w.nq, n, dtype=np.int64)
    return generate(w.batch, w.heads, w.head_dim, w.grid, w.seed, strength=w.strength,
                    strength_range=w.strength_range, iid=w.iid, q_token_ids=q_ids,
                    axis_stretch=w.extra.get("axis_stretch"))


def grad_output(w: "_configs.Workload", seed_offset: int = 500) -> torch.Tensor:
    """dL/dO for a workload's backward pass: i.i.d. N(0, 1) in bfloat16, shaped like O
    ([B, nq, H, D]) in the path's token order."""
    rng = np.random.default_rng(w.seed + seed_offset)
    a = rng.standard_normal((w.batch, w.nq, w.heads, w.head_dim), dtype=np.float32)
    return _to_bf16(a)


def random_mask(rows: int, cols: int, density: float, seed: int) -> np.ndarray:
    """Uniform random 0/1 block mask (uint8) used by parity tests of the attention kernel."""
    rng = np.random.default_rng(seed)
    return (rng.random((rows, cols)) < density).astype(np.uint8)


def sample_rows(n: int, count: int, seed: int, must: Sequence[int] = ()) -> np.ndarray:
    """Sorted distinct row indices in [0, n): ``must`` plus a seeded uniform draw."""
    rng = np.random.default_rng(seed)
    base = set(int(m) for m in must if 0 <= m < n)
    extra = rng.choice(n, size=min(n, count), replace=False)
    base.update(int(e) for e in extra)
    return np.array(sorted(base), dtype=np.int64)
