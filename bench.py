#!/usr/bin/env python3
"""Benchmark of the block-sparse video attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over one batch of synthetic input already
resident in HBM: tile permute of Q, K, V -> block mask -> CSR compaction ->
block-sparse attention forward -> inverse permute of O.  The default workload is
the largest single-GPU one: the radial (energy-decay) mask at 500 frames of
720p video (1 x 12 heads x 128, 126x45x80 = 453,600 tokens in raster order,
128-token blocks); ``--workload sta_720p`` is the Sliding-Tile 720p DiT shape
(1 x 24 heads x 128, 30x48x80 tokens, 6x8x8 tiles of 384 tokens, 3x3x5-tile
window), ``nabla_480p`` and ``ar_decode`` the dynamic-mask ones.  Metric: effective TFLOP/s =
4 * head_dim * (query, key) pairs inside kept blocks / time.

``--pass sics`` times SPADE scheme generation (SICS of Q and K under every shape
of the workload's slice-shape menu, per-head choice), metric: GB/s of Q and K read
(one pass per shape), with its time as a fraction of the workload's attention.

``--pass ar_paged`` runs the autoregressive workload's decode through the paged,
persistent-anchor KV cache (one chunk of frames at a time: append, attend,
evict) and times the last chunk's attention step over the cache; the line also
reports the cache's memory against a plain cache of the whole sequence.

``--pass bwd`` times the block-sparse attention backward instead (dQ, dK, dV from
Q, K, V, O, LSE and dO in the path's token order, over the kept lists of the
workload's mask), metric: effective TFLOP/s = 10 * head_dim * kept pairs / time
(five matrix products of 2 * head_dim flops per pair: the recomputed scores, dP,
dV, dQ and dK).

Under torchrun (N > 1) the forward path splits the workload's heads over the
ranks (each rank holds and computes its own range of heads; masks are per head,
so nothing is exchanged): strong scaling, value = the whole workload's work
divided by the slowest rank's time; ``--pass bwd`` splits the heads the same
way.  The SICS and paged passes run one copy of the workload per rank (weak
scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (dense bf16 tensor, HBM3e on HGX boards), for the
# fraction of nominal reported beside the fraction of the measured peak.
NOMINAL_PEAKS = {"TFLOP/s": 2250.0, "GB/s": 7700.0}


def with_nominal(roofline: dict) -> dict:
    roofline["frac_of_nominal"] = roofline["achieved"] / NOMINAL_PEAKS[roofline["unit"]]
    return roofline


def choose_tensor_peak(peaks: dict, clocks: dict, timed_s: float):
    """The bf16 peak a kernel timed in this run is held to: the burst figure (a GEMM
    timed alone, at the maximum clock) when the median SM clock over the timed
    region stayed within 3 % of the maximum, else the sustained figure (a
    seconds-long GEMM loop under the power cap): a kernel that itself drove the
    clock down under the power cap is compared with the GEMM under the same cap,
    however short the region.  Without clock samples the burst figure is used."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if not (mhz and mx):
        return peaks["bf16_tflops"], "burst", "no clock samples"
    if mhz >= 0.97 * mx:
        return peaks["bf16_tflops"], "burst", \
            f"median SM clock {mhz:.0f} of {mx:.0f} MHz over {timed_s:.1f} s"
    return peaks["bf16_tflops_sustained"], "sustained", \
        f"median SM clock {mhz:.0f} of {mx:.0f} MHz over {timed_s:.1f} s (power cap)"


def tensor_roofline(achieved: float, kernel_ms: float, peaks: dict, peak_kind: str,
                    clocks: dict, timed_s: float, **extra) -> dict:
    """Roofline object of a tensor-bound kernel: frac against the peak that
    choose_tensor_peak picks, the fractions of both measured figures, and the
    kernel's mean time times the median SM clock (ms x MHz = thousands of SM
    cycles), which compares runs taken at different clocks."""
    peak, kind, why = choose_tensor_peak(peaks, clocks, timed_s)
    mhz = clocks.get("sm_mhz")
    r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
         "frac": achieved / peak,
         "peak_note": f"{peak_kind} {kind} bf16 ({why})",
         "frac_of_burst": achieved / peaks["bf16_tflops"],
         "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
         "kernel_ms_x_sm_mhz": kernel_ms * mhz if mhz else None}
    r.update(extra)
    return with_nominal(r)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


KERNEL_SOURCES = {
    "attn_fwd": ("attn_fwd.cu", "attn_common.cuh", "bsa_common.cuh", "tmem_io.cuh"),
    "attn_bwd": ("attn_bwd.cu", "attn_common.cuh", "bsa_common.cuh", "tmem_io.cuh"),
    "sics": ("sics.cu", "bsa_common.cuh"),
}


def attn_source_hash(kind: str = "attn_fwd") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "block_sparse_attention_tokens_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kind: str = "attn_fwd"):
    """DRAM bytes per launch from the committed ncu summary of `kind` on the
    workload, if that summary was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kind}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != attn_source_hash(kind):
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self.samples = []
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def summary(self):
        if not getattr(self, "samples", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for n, val in zip(names, s[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(self.samples)}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_head_perms(w, q, k):
    """Token order of every head in the path, by the oracle: None (raster order),
    the workload's tile order, or (per-head slicing) the tile order of the shape the
    oracle's SICS scheme picks for the head."""
    import oracle as O
    if w.mask == "spade":
        from block_sparse_attention_tokens_b200.configs import sics_menu
        menu = sics_menu(w.block)
        _, choice = O.sics_scheme(q.double().numpy(), k.double().numpy(), w.grid, menu)
        return [O.tile_order(w.grid, menu[int(choice[0, h])]) for h in range(w.heads)]
    if w.tile is not None:
        return [O.tile_order(w.grid, w.tile)] * w.heads
    return [None] * w.heads


def oracle_workload_mask(w, q, k, perms=None):
    """The oracle's own block mask of the workload, [Hm, QB, KB] uint8 (Hm = 1 for
    the static masks, batch * heads otherwise), from the raster-order bf16 inputs:
    the Sliding-Tile window, the radial rule, NABLA (per-head pooled means of the
    tile-ordered Q and K), NABLA united with the window, NABLA over per-head slices,
    or the autoregressive composition.  perms: oracle_head_perms (computed if None)."""
    import numpy as np
    import oracle as O
    QB, KB = math.ceil(w.nq / w.block), math.ceil(w.nk / w.block)
    if w.tile is not None:
        tg = tuple(math.ceil(g / t) for g, t in zip(w.grid, w.tile))
    if w.mask == "sta":
        return O.sta_tile_mask(tg, w.window)[None]
    if w.mask == "radial":
        return O.radial_block_mask_fast(w.nk, w.tokens_per_frame, w.block)[None]
    D = w.head_dim
    scale = 1.0 / math.sqrt(D)
    if perms is None:
        perms = oracle_head_perms(w, q, k)
    n_pad = QB * w.block
    qbar = np.zeros((w.batch, w.heads, QB, D))
    kbar = np.zeros((w.batch, w.heads, KB, D))
    for h in range(w.heads):
        qh = q[:, :, h:h + 1].double().numpy()
        kh = k[:, :, h:h + 1].double().numpy()
        if perms[h] is not None:
            qh, kh = O.tile_permute(qh, perms[h], n_pad), O.tile_permute(kh, perms[h], n_pad)
        else:
            qh = np.concatenate([qh, np.zeros((w.batch, QB * w.block - w.nq, 1, D))], axis=1)
            kh = np.concatenate([kh, np.zeros((w.batch, KB * w.block - w.nk, 1, D))], axis=1)
        qbar[:, h] = O.nabla_pool(qh, w.block, w.nq)[:, 0]
        kbar[:, h] = O.nabla_pool(kh, w.block, w.nk)[:, 0]
    if w.mask in ("nabla", "spade"):
        m, _ = O.nabla_mask(qbar, kbar, w.p, scale)
    elif w.mask == "nabla_sta":
        m, _ = O.nabla_sta_mask(qbar, kbar, w.p, scale, O.sta_tile_mask(tg, w.window))
    elif w.mask == "ar":
        m, _ = O.ar_mask(qbar, kbar, w.p, scale, w.nk, w.tokens_per_frame, w.block,
                         w.anchor_frames, w.recent_frames)
    else:
        raise ValueError(w.mask)
    return m.reshape(-1, QB, KB).astype(np.uint8)


class OracleSample:
    """The CPU oracle on whole query blocks of the workload (all heads).

    Setup (untimed): the oracle's own mask of the workload (for NABLA and the
    autoregressive mask this runs the oracle's pooling and top-p selection) and,
    for tiled workloads, the oracle's tile order.  ``run(budget_s)`` evaluates
    random query blocks until about budget_s seconds of oracle work: per block and
    head, the block's query rows and the keys of its kept blocks are gathered from
    the bf16 inputs in the path's token order and upcast to float64 (untimed), and
    the oracle's attention is timed on them -- the same rows over the same kept
    keys as a call on the whole sequence, without holding float64 copies of it.
    Returns (effective TFLOP/s, sample text).
    """

    def __init__(self, w, q, k, v):
        import numpy as np
        import oracle as O
        self.w, self.O, self.np = w, O, np
        t0 = time.perf_counter()
        self.q, self.k, self.v = q, k, v
        self.perms = oracle_head_perms(w, q, k)
        self.mask = oracle_workload_mask(w, q, k, self.perms)
        self.setup_s = time.perf_counter() - t0
        self.rng = np.random.default_rng(7)

    def path_rows(self, t, rows, h):
        """float64 [B, len(rows), 1, D] of tensor t at path-order rows, head h."""
        idx = rows if self.perms[h] is None else self.perms[h][rows]
        return t[:, self.np.asarray(idx), h:h + 1].double().numpy()

    def gather(self, qb, h):
        """(rows, keys, kept blocks) of query block qb under head h's mask row."""
        w, np = self.w, self.np
        hm = 0 if self.mask.shape[0] == 1 else h
        rows = np.arange(qb * w.block, min((qb + 1) * w.block, w.nq))
        kept = np.nonzero(self.mask[hm, qb])[0]
        keys = np.concatenate([np.arange(kb * w.block, min((kb + 1) * w.block, w.nk))
                               for kb in kept]) if kept.size else np.zeros(0, np.int64)
        return rows, keys, kept

    def run(self, budget_s: float):
        w, O, np = self.w, self.O, self.np
        QB = math.ceil(w.nq / w.block)
        flops, done, timed = 0.0, 0, 0.0
        for qb in self.rng.permutation(QB):
            for h in range(w.heads):
                rows, keys, kept = self.gather(qb, h)
                if keys.size == 0:
                    continue
                qh, kh, vh = (self.path_rows(t, r, h) for t, r in
                              ((self.q, rows), (self.k, keys), (self.v, keys)))
                ones = np.ones((1, 1, kept.size), np.uint8)   # the gathered kept blocks
                t1 = time.perf_counter()
                O.block_sparse_attention(qh, kh, vh, ones, w.block, w.block)
                timed += time.perf_counter() - t1
                flops += 4.0 * w.head_dim * rows.size * keys.size
            done += 1
            if timed > budget_s:
                break
        sample = (f"{done} random query blocks x {w.heads} heads of {w.name} "
                  f"({flops / 1e12:.4f} effective TFLOP), float64 oracle, {timed:.1f} s "
                  f"(+{self.setup_s:.1f} s untimed setup: the oracle's own mask; rows and kept "
                  f"keys gathered and upcast outside the timing)")
        return flops / timed / 1e12, sample


class BackwardOracleSample(OracleSample):
    """The CPU oracle's backward on whole query blocks of the workload (all heads):
    each sampled block and head runs the oracle's block-sparse backward on the
    block's query rows and its kept keys (dO of those rows), which is the backward
    work of those queries: 10 * head_dim flops per kept pair."""

    def __init__(self, w, q, k, v, do):
        super().__init__(w, q, k, v)
        self.do = do                     # already in the path's token order

    def run(self, budget_s: float):
        w, O, np = self.w, self.O, self.np
        QB = math.ceil(w.nq / w.block)
        flops, done, timed = 0.0, 0, 0.0
        for qb in self.rng.permutation(QB):
            for h in range(w.heads):
                rows, keys, kept = self.gather(qb, h)
                if keys.size == 0:
                    continue
                qh, kh, vh = (self.path_rows(t, r, h) for t, r in
                              ((self.q, rows), (self.k, keys), (self.v, keys)))
                dh = self.do[:, rows, h:h + 1].double().numpy()
                ones = np.ones((1, 1, kept.size), np.uint8)
                t1 = time.perf_counter()
                O.block_sparse_attention_backward(qh, kh, vh, dh, ones, w.block, w.block)
                timed += time.perf_counter() - t1
                flops += 10.0 * w.head_dim * rows.size * keys.size
            done += 1
            if timed > budget_s:
                break
        sample = (f"{done} random query blocks x {w.heads} heads of {w.name} "
                  f"({flops / 1e12:.4f} effective TFLOP), float64 oracle backward, {timed:.1f} s "
                  f"(+{self.setup_s:.1f} s untimed setup: the oracle's own mask; rows and kept "
                  f"keys gathered and upcast outside the timing)")
        return flops / timed / 1e12, sample


BWD_METRIC = "block-sparse attention backward effective TFLOP/s"
SICS_METRIC = "SPADE SICS scheme generation GB/s (Q and K read once per menu shape)"
AR_PAGED_METRIC = "paged AR chunk attention effective TFLOP/s (persistent-anchor KV cache)"
AR_KEEP_FRACTION = 0.58   # pages kept at the end of the run: the Sparse Forcing summary's 42 % saving


def ar_budget(w, keep_fraction=AR_KEEP_FRACTION):
    """Middle pages the cache keeps so that anchors + recent + middle make up
    keep_fraction of the pages of the whole sequence."""
    page = 128
    S = w.tokens_per_frame
    n_pages = math.ceil(w.n_tokens / page)
    anchor_pages = math.ceil(w.anchor_frames * S / page)
    recent_begin = (w.n_tokens - w.recent_frames * S) // page
    return max(0, round(keep_fraction * n_pages) - anchor_pages - (n_pages - recent_begin))


def ar_all_queries(w):
    """Q for every token of the AR workload (each chunk's queries), K and V."""
    import numpy as np
    from block_sparse_attention_tokens_b200 import synth
    q, k, v, _ = synth.generate(w.batch, w.heads, w.head_dim, w.grid, w.seed, strength=w.strength,
                                strength_range=w.strength_range, iid=w.iid,
                                q_token_ids=np.arange(w.n_tokens))
    return q, k, v


class PagedAROracleSample:
    """The oracle on the last chunk of the paged AR run: the cache's residency is
    simulated with the oracle's own policy over every earlier chunk (untimed
    setup); the timed part is the oracle's attention over the resident pages for
    random query blocks of the last chunk (all heads)."""

    def __init__(self, w, q, k, v):
        import numpy as np
        import oracle as O
        self.w, self.O, self.np = w, O, np
        t0 = time.perf_counter()
        S, blk, page = w.tokens_per_frame, w.block, 128
        chunk = w.q_frames * S
        scale = 1.0 / math.sqrt(w.head_dim)
        n_chunks = w.n_tokens // chunk
        budget = ar_budget(w)
        k64 = k.double().numpy()
        KBmax = math.ceil(w.n_tokens / blk)
        kpad = np.zeros((w.batch, KBmax * blk, w.heads, w.head_dim))
        kpad[:, :w.n_tokens] = k64
        kbar_all = O.nabla_pool(kpad, blk, w.n_tokens)     # every block's mean (causal per block)
        resident = np.zeros((w.batch, math.ceil(w.n_tokens / page)), dtype=bool)
        for c in range(n_chunks):
            lo, hi = c * chunk, (c + 1) * chunk
            resident[:, lo // page: math.ceil(hi / page)] = True
            n_pages, KB = math.ceil(hi / page), math.ceil(hi / blk)
            table = np.where(resident[:, :n_pages], 0, -1)
            allowed = O.resident_blocks(table, page, blk, hi)
            QB = math.ceil(chunk / blk)
            qpad = np.zeros((w.batch, QB * blk, w.heads, w.head_dim))
            qpad[:, :chunk] = q[:, lo:hi].double().numpy()
            qbar = O.nabla_pool(qpad, blk, chunk)
            kbar = kbar_all[:, :, :KB].copy()
            if KB * blk > hi:                                # the last block is partial now
                kbar[:, :, KB - 1] = k64[:, (KB - 1) * blk:hi].mean(axis=1)
            a_end, r_begin = O.ar_block_ranges(hi, S, blk, w.anchor_frames, w.recent_frames)
            if c == n_chunks - 1:
                m, _ = O.nabla_mask(qbar, kbar, w.p, scale, a_end, r_begin, 1, key_allowed=allowed)
                self.mask = (m * allowed[:, None, None, :]).reshape(-1, QB, KB).astype(np.uint8)
                break
            sc = O.kv_page_scores(qbar, kbar, scale, a_end, r_begin, blk, page, n_pages,
                                  key_allowed=allowed)
            anchor_pages = math.ceil(w.anchor_frames * S / page)
            recent_begin = max(anchor_pages, (hi - w.recent_frames * S) // page)
            resident[:, :n_pages] &= O.kv_keep_pages(sc, resident[:, :n_pages], anchor_pages,
                                                     recent_begin, budget)
        self.lo, self.hi, self.chunk = (n_chunks - 1) * chunk, n_chunks * chunk, chunk
        self.heads64 = [(q[:, self.lo:self.hi, h:h + 1].double().numpy(),
                         k64[:, :self.hi, h:h + 1], v[:, :self.hi, h:h + 1].double().numpy())
                        for h in range(w.heads)]
        self.setup_s = time.perf_counter() - t0
        self.rng = np.random.default_rng(5)

    def run(self, budget_s: float):
        w, O, np = self.w, self.O, self.np
        blk = w.block
        QB = math.ceil(self.chunk / blk)
        flops, done = 0.0, 0
        t1 = time.perf_counter()
        for qb in self.rng.permutation(QB):
            rows = np.arange(qb * blk, min((qb + 1) * blk, self.chunk))
            for h, (qh, kh, vh) in enumerate(self.heads64):
                O.block_sparse_attention(qh, kh, vh, self.mask[h:h + 1], blk, blk, rows=rows)
                kept = np.nonzero(self.mask[h, qb])[0]
                nkeys = sum(min((kb + 1) * blk, self.hi) - kb * blk for kb in kept)
                flops += 4.0 * w.head_dim * len(rows) * nkeys
            done += 1
            if time.perf_counter() - t1 > budget_s:
                break
        el = time.perf_counter() - t1
        sample = (f"{done} random query blocks x {w.heads} heads of the last chunk of {w.name} "
                  f"over the resident pages ({flops / 1e12:.4f} effective TFLOP), float64 oracle, "
                  f"{el:.1f} s (+{self.setup_s:.1f} s untimed setup: the oracle's cache policy over "
                  f"the earlier chunks)")
        return flops / el / 1e12, sample


class SicsOracleSample:
    """The oracle's SICS scheme generation on whole heads of the workload: each
    sampled head runs the full menu over that head's Q and K."""

    def __init__(self, w, q, k):
        import numpy as np
        import oracle as O
        from block_sparse_attention_tokens_b200 import configs
        self.w, self.O, self.np = w, O, np
        self.q, self.k = q, k
        self.menu = configs.sics_menu(w.block)
        self.rng = np.random.default_rng(11)

    def run(self, budget_s: float):
        w, O = self.w, self.O
        done, nbytes = 0, 0.0
        t1 = time.perf_counter()
        for h in self.rng.permutation(w.heads):
            qh = self.q[:, :, h:h + 1].double().numpy()
            kh = self.k[:, :, h:h + 1].double().numpy()
            O.sics_scheme(qh, kh, w.grid, self.menu)
            nbytes += len(self.menu) * 2 * w.batch * w.nq * w.head_dim * 2
            done += 1
            if time.perf_counter() - t1 > budget_s:
                break
        el = time.perf_counter() - t1
        sample = (f"{done} random heads of {w.name}, full menu of {len(self.menu)} shapes, "
                  f"float64 oracle, {el:.1f} s (bytes counted as the bf16 Q and K rows read)")
        return nbytes / el / 1e9, sample
FWD_METRIC = "block-sparse attention effective TFLOP/s (path step)"


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_sparse_attention_tokens_b200 import synth
    q, k, v, _ = synth.workload_inputs(w)
    if args.pass_ == "bwd":
        sampler = BackwardOracleSample(w, q, k, v, path_order_grad(w))
    elif args.pass_ == "ar_paged":
        sampler = PagedAROracleSample(w, *ar_all_queries(w))
    elif args.pass_ == "sics":
        sampler = SicsOracleSample(w, q, k)
    else:
        sampler = OracleSample(w, q, k, v)
    n = max(1, args.steps + args.warmup)
    budget = max(0.5, min(10.0, 90.0 / n, args.cpu_budget))
    vals = []
    sample = ""
    for i in range(n):
        val, sample = sampler.run(budget)
        if i >= args.warmup:
            vals.append(val)
    value = statistics.median(vals) if vals else val
    metric = {"bwd": BWD_METRIC, "sics": SICS_METRIC,
              "ar_paged": AR_PAGED_METRIC}.get(args.pass_, FWD_METRIC)
    unit = "GB/s" if args.pass_ == "sics" else "TFLOP/s"
    line = {"impl": "reference", "metric": metric,
            "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args.pass_),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_cores(),
                             "kind": "oracle", "sample": f"per step: {sample}"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity when not
    distributed).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device=None):
    """Element-wise sum of a float (or list of floats) over all ranks (identity
    when not distributed).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist
    scalar = not isinstance(values, (list, tuple))
    t = torch.tensor([values] if scalar else list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.item() if scalar else t.tolist()


def job_value(flops_all_ranks, ms_per_step):
    """Whole-job throughput (TFLOP/s): the work of all ranks in the slowest rank's
    step time."""
    return flops_all_ranks / (ms_per_step * 1e-3) / 1e12


def weak_scaling_value(flops_per_rank, world, ms_per_step):
    """Whole-job throughput (TFLOP/s): every rank processes its own batch of the
    same shape, the slowest rank's time bounds the step."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def path_order_grad(w):
    """The seeded dL/dO of the workload, [B, nq, H, D] bf16 in the path's token order."""
    from block_sparse_attention_tokens_b200 import synth
    return synth.grad_output(w)


def mask_stats(flops: float, w, nq: int, nk: int, attn_times_ms, near=None) -> dict:
    """Kept share of the (query, key) token pairs, spread of the attention call times
    over the timed steps, and the NABLA rows whose cut lies within 1e-5 of p (or on
    a tie), counted by the selection kernel of the last step."""
    t = sorted(attn_times_ms)
    pct = lambda f: t[min(len(t) - 1, int(round(f * (len(t) - 1))))]
    out = {"kept_pair_fraction": flops / (4.0 * w.head_dim * nq * nk * w.batch * w.heads),
           "attn_ms_p10": pct(0.1), "attn_ms_median": pct(0.5), "attn_ms_p90": pct(0.9)}
    if near is not None:
        out["near_threshold_rows"] = int(near)
    return out


def permute_bandwidth(w, plan, stage_ms: dict, hbm_peak: float):
    """Algorithmic GB/s of the tile permute (Q, K, V: N rows read, n_pad rows
    written, the zero tail included) and of the untile (O: N rows read and
    written), with the fraction of the HBM peak; None without a tile order."""
    if not plan.permuted:
        return None
    row = w.heads * w.head_dim * 2
    n, n_pad = w.n_tokens, plan.n_pad
    permute_bytes = 3 * w.batch * (n + n_pad) * row
    if w.mask == "spade":
        # the stage also runs the SICS scheme: Q and K read once per menu shape
        permute_bytes += 2 * len(plan.menu) * w.batch * n * row
    out = {}
    for name, nbytes in (("permute", permute_bytes), ("untile", 2 * w.batch * n * row)):
        ms = stage_ms[name]
        gbs = nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
        out[name] = {"bytes": nbytes, "gb_s": gbs,
                     "frac_of_hbm": gbs / hbm_peak if gbs else None}
    if w.mask == "spade":
        out["permute"]["stage"] = "SICS scheme + per-head permute of Q, K (pooled), V"
    return out


def workload_config(w, pass_: str = "fwd"):
    cfg = {"workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
           "grid_thw": list(w.grid), "block": w.block, "mask": w.mask}
    if pass_ == "bwd":
        cfg["pass"] = "backward (dQ, dK, dV)"
    if pass_ == "ar_paged":
        cfg["pass"] = "paged persistent-anchor KV cache, last chunk of the decode"
        cfg["kv_page_tokens"] = 128
        cfg["kv_keep_fraction"] = AR_KEEP_FRACTION
        cfg["kv_middle_budget_pages"] = ar_budget(w)
    if pass_ == "sics":
        from block_sparse_attention_tokens_b200 import configs
        cfg["pass"] = "SPADE scheme generation (SICS)"
        cfg["menu"] = [list(sh) for sh in configs.sics_menu(w.block)]
    if w.tile:
        cfg["tile"] = list(w.tile)
    if w.window:
        cfg["window_tiles"] = list(w.window)
    if w.p is not None:
        cfg["p"] = w.p
    cfg["l2"] = "inputs larger than L2 (no flush between steps)"
    return cfg


def setup_ranks():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, torch.device("cuda", torch.cuda.current_device())


def run_backward(args, w):
    """Times bsa_attn_bwd at the workload's full size.  The forward path runs once
    (untimed) to give O, LSE and the kept lists; each timed step is one backward
    call (list transposition, LSE/Delta preparation and the two tcgen05 passes)."""
    import torch
    import torch.distributed as dist
    from block_sparse_attention_tokens_b200 import binding as B
    from block_sparse_attention_tokens_b200 import synth
    from block_sparse_attention_tokens_b200.pipeline import Plan, effective_flops, head_range

    world, rank, dev = setup_ranks()
    q_h, k_h, v_h, _ = synth.workload_inputs(w)
    do_h = path_order_grad(w)
    # with N ranks each rank takes its range of heads, as in the forward
    h0, h1 = head_range(rank, world, w.heads)
    q_h, k_h, v_h, do_h = (t_[:, :, h0:h1].contiguous() for t_ in (q_h, k_h, v_h, do_h))
    plan = Plan(w, dev, heads=(h0, h1))
    plan.step(q_h.to(dev), k_h.to(dev), v_h.to(dev))
    qq, kk, vv = (plan.qp, plan.kp, plan.vp) if plan.permuted else (plan._q, plan._k, plan._v)
    oo = plan.op if plan.permuted else plan.o
    do = do_h.to(dev)
    dq, dk, dv = torch.empty_like(qq), torch.empty_like(kk), torch.empty_like(vv)
    ws = torch.empty(B.bsa_attn_bwd_workspace_size(w.batch, plan.heads, plan.nq, plan.nk, w.block,
                                                   w.block, plan.list_heads),
                     dtype=torch.uint8, device=dev)

    def bwd(q_, k_, v_, o_, do_, lse_, rp_, ci_, outs=None):
        dq_, dk_, dv_ = (dq, dk, dv) if outs is None else outs
        B.bsa_attn_bwd(q_, k_, v_, o_, do_, lse_, rp_, ci_, w.block, w.block, plan.list_heads,
                       nq=plan.nq, nk=plan.nk, dq=dq_, dk=dk_, dv=dv_, ws=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    args_dev = (qq, kk, vv, oo, do, plan.lse, plan.row_ptr, plan.col_idx)
    for _ in range(max(3, args.warmup)):
        bwd(*args_dev)
    barrier()
    if B.bsa_read_status(ws) != 0:
        raise RuntimeError("backward kernel reported a device-side error")
    flops = 2.5 * effective_flops(plan.mask, plan.nq, plan.nk, w.block, w.head_dim,
                                  w.batch * plan.heads)
    flops_all = sum_over_ranks(flops, dev)

    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier()
    with sampler:
        time.sleep(0.5)
        for i in range(args.steps):
            ev[i][0].record(stream)
            bwd(*args_dev)
            ev[i][1].record(stream)
        barrier()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_total = sum(a.elapsed_time(b) for a, b in ev)
    ms, ms_total = max_over_ranks([ms, ms_total], dev)
    value = job_value(flops_all, ms)

    # end to end through the public API: every step copies its inputs from pinned
    # host memory (Q, K, V, O, dO in the path's token order, LSE, the kept lists),
    # runs the backward and copies dQ, dK, dV back.  Steps are pipelined as a
    # training loop would run them: the input copy of step i+1 (copy stream) and the
    # output copy of step i-1 (out stream) overlap the backward of step i; inputs
    # and outputs are double-buffered.
    e2e = None
    if not args.no_e2e:
        host_in = [t_.detach().to("cpu").pin_memory() for t_ in args_dev]
        dev_in = [[torch.empty_like(t_) for t_ in args_dev] for _ in range(2)]
        dev_out = [tuple(torch.empty_like(t_) for t_ in (dq, dk, dv)) for _ in range(2)]
        host_out = [torch.empty(t_.shape, dtype=t_.dtype).pin_memory() for t_ in (dq, dk, dv)]
        e_steps = max(3, args.steps // 2)
        total = 2 + e_steps
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(total)]
        ev_done = [torch.cuda.Event() for _ in range(total)]
        ev_out = [torch.cuda.Event() for _ in range(total)]

        def h2d(i):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i - 2])      # inputs of step i-2 consumed
                for dst, src in zip(dev_in[i % 2], host_in):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)

        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h2d(0)
        for i in range(total):
            if i == 2:
                e0.record(stream)
            if i + 1 < total:
                h2d(i + 1)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])         # these outputs copied out (step i-2)
            bwd(*dev_in[i % 2], outs=dev_out[i % 2])
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                for dst, src in zip(host_out, dev_out[i % 2]):
                    dst.copy_(src, non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_event(ev_out[total - 1])
        e1.record(stream)
        barrier()
        # time from the start of step 2 to the end of the last output copy, per step
        e_ms = max_over_ranks([e0.elapsed_time(e1) / e_steps], dev)[0]
        h2d, d2h = sum_over_ranks(
            [sum(t_.numel() * t_.element_size() for t_ in host_in),
             sum(t_.numel() * t_.element_size() for t_ in host_out)], dev)
        e2e = {"value": job_value(flops_all, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "note": "pinned host buffers; copies of neighbouring steps overlap the backward"}

    peaks, peak_kind = load_peaks()
    achieved = flops_all / world / (ms * 1e-3) / 1e12
    clocks = sampler.summary()
    roofline = tensor_roofline(
        achieved, ms, peaks, peak_kind, clocks, ms_total * 1e-3,
        traffic=profiled_traffic(w.name, "attn_bwd"),
        kernel="attn_bwd_kernel<128> (dK/dV pass + dQ pass) and list preparation", bwd_ms=ms)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, sample = BackwardOracleSample(w, q_h, k_h, v_h, do_h).run(args.cpu_budget)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample}
    if rank == 0:
        cfg = workload_config(w, "bwd")
        cfg["parallelism"] = f"heads split over {world} GPU(s), no data-path collective"
        line = {"metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": cfg,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "clocks": clocks, "gpu_launches": 6 * args.steps,
                "effective_tflop_per_step": flops_all / 1e12}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_sics(args, w):
    """Times bsa_sics_scheme over the workload's Q and K (raster order, resident in
    HBM) with the workload's slice-shape menu; also times the workload's attention
    kernel to state scheme generation as a fraction of it."""
    import torch
    import torch.distributed as dist
    from block_sparse_attention_tokens_b200 import binding as B
    from block_sparse_attention_tokens_b200 import configs, synth
    from block_sparse_attention_tokens_b200.pipeline import Plan

    world, rank, dev = setup_ranks()
    q_h, k_h, v_h, _ = synth.workload_inputs(w)
    q, k = q_h.to(dev), k_h.to(dev)
    menu = configs.sics_menu(w.block)
    scores = torch.empty((w.batch, w.heads, len(menu)), dtype=torch.float32, device=dev)
    choice = torch.empty((w.batch, w.heads), dtype=torch.int32, device=dev)
    ws = torch.empty(B.bsa_sics_workspace_size(w.batch, w.heads, w.grid, menu),
                     dtype=torch.uint8, device=dev)

    def scheme(q_, k_):
        B.bsa_sics_scheme(q_, k_, w.grid, menu, scores=scores, choice=choice, ws=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        scheme(q, k)
    barrier()
    nbytes = len(menu) * 2 * q.numel() * q.element_size()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier()
    with sampler:
        time.sleep(0.5)
        for i in range(args.steps):
            ev[i][0].record(stream)
            scheme(q, k)
            ev[i][1].record(stream)
        barrier()
    ms = max_over_ranks([statistics.mean(a.elapsed_time(b) for a, b in ev)], dev)[0]
    value = nbytes * world / (ms * 1e-3) / 1e9

    # the workload's attention kernel, for the fraction of attention time
    plan = Plan(w, dev)
    plan.step(q, k, v_h.to(dev))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    a0.record(stream)
    for _ in range(5):
        plan.attention()
    a1.record(stream)
    barrier()
    attn_ms = a0.elapsed_time(a1) / 5
    del plan

    e2e = None
    if not args.no_e2e:
        hq, hk = q_h.pin_memory(), k_h.pin_memory()
        dq_, dk_ = torch.empty_like(q), torch.empty_like(k)
        hs = torch.empty(scores.shape, dtype=scores.dtype).pin_memory()
        hc = torch.empty(choice.shape, dtype=choice.dtype).pin_memory()
        e_steps = max(3, args.steps // 2)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            dq_.copy_(hq, non_blocking=True)
            dk_.copy_(hk, non_blocking=True)
            scheme(dq_, dk_)
            hs.copy_(scores, non_blocking=True)
            hc.copy_(choice, non_blocking=True)
        e1.record(stream)
        barrier()
        e_ms = max_over_ranks([e0.elapsed_time(e1) / e_steps], dev)[0]
        e2e = {"value": nbytes * world / (e_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": 2 * q_h.numel() * q_h.element_size(),
               "d2h_bytes_per_step": hs.numel() * 4 + hc.numel() * 4,
               "note": "pinned host buffers; copies and the scheme serialised on one stream"}

    peaks, peak_kind = load_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(w.name, "sics"),
                "kernel": "sics_kernel<128> (one launch per tensor and menu shape)",
                "peak_note": f"{peak_kind} HBM copy bandwidth"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, sample = SicsOracleSample(w, q_h, k_h).run(args.cpu_budget)
        cpu = {"value": val, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample}
    if rank == 0:
        line = {"metric": SICS_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic", "config": workload_config(w, "sics"),
                "roofline": with_nominal(roofline), "cpu_baseline": cpu, "e2e": e2e,
                "clocks": sampler.summary(),
                "gpu_launches": 2 * args.steps,   # one SICS launch for every shape + the choice
                "attention_ms": attn_ms, "fraction_of_attention_time": ms / attn_ms,
                "choice_histogram": torch.bincount(choice.flatten().long(),
                                                   minlength=len(menu)).tolist()}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_ar_paged(args, w):
    """The AR workload decoded chunk by chunk through PagedARCache; the timed step
    is the last chunk's attention over the cache (block means, residency, NABLA
    over the resident middle blocks, compaction, paged attention)."""
    import torch
    import torch.distributed as dist
    from block_sparse_attention_tokens_b200.pipeline import PagedARCache, Plan, effective_flops

    if w.mask != "ar":
        raise ValueError("--pass ar_paged needs an autoregressive workload")
    world, rank, dev = setup_ranks()
    q_h, k_h, v_h = ar_all_queries(w)
    S = w.tokens_per_frame
    chunk = w.q_frames * S
    n_chunks = w.n_tokens // chunk
    budget = ar_budget(w)
    cache = PagedARCache(w, w.n_tokens, budget, dev)
    qd, kd, vd = q_h.to(dev), k_h.to(dev), v_h.to(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for c in range(n_chunks - 1):
        lo, hi = c * chunk, (c + 1) * chunk
        cache.append(kd[:, lo:hi], vd[:, lo:hi])
        cache.attend(qd[:, lo:hi], w.p)
        cache.evict()
    lo, hi = (n_chunks - 1) * chunk, n_chunks * chunk
    cache.append(kd[:, lo:hi], vd[:, lo:hi])
    q_last = qd[:, lo:hi].contiguous()
    for _ in range(max(3, args.warmup)):
        o, lse, mask = cache.attend(q_last, w.p)
    barrier()
    if cache.status.item() != 0 or device_status(cache.attn_ws) != 0:
        raise RuntimeError("paged cache kernels reported a device-side error")
    flops = effective_flops(mask, chunk, hi, w.block, w.head_dim, w.batch * w.heads)
    resident_before = cache.resident_bytes()

    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier()
    with sampler:
        time.sleep(0.5)
        for i in range(args.steps):
            ev[i][0].record(stream)
            cache.attend(q_last, w.p)
            ev[i][1].record(stream)
        barrier()
    ms = max_over_ranks([statistics.mean(a.elapsed_time(b) for a, b in ev)], dev)[0]
    value = weak_scaling_value(flops, world, ms)

    # the same chunk through the plain (contiguous, never evicting) AR path
    plan = Plan(w, dev)
    plan.step(q_last, kd, vd)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    a0.record(stream)
    for _ in range(5):
        plan.build_mask()
        plan.compact()
        plan.attention()
    a1.record(stream)
    barrier()
    plain_ms = a0.elapsed_time(a1) / 5
    del plan

    e2e = None
    if not args.no_e2e:
        hq = q_h[:, lo:hi].contiguous().pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        dq_ = torch.empty_like(q_last)
        e_steps = max(3, args.steps // 2)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            dq_.copy_(hq, non_blocking=True)
            o_, _, _ = cache.attend(dq_, w.p)
            ho.copy_(o_, non_blocking=True)
        e1.record(stream)
        barrier()
        e_ms = max_over_ranks([e0.elapsed_time(e1) / e_steps], dev)[0]
        e2e = {"value": weak_scaling_value(flops, world, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size(),
               "note": "the chunk's queries from pinned host memory, O back; K/V stay in the "
                       "device cache (that is the cache's job)"}

    cache.evict()
    barrier()
    plain_bytes = 2 * w.batch * w.n_tokens * w.heads * w.head_dim * 2
    kv = {"plain_cache_bytes": plain_bytes, "resident_bytes_before_evict": resident_before,
          "resident_bytes_after_evict": cache.resident_bytes(), "pool_bytes": cache.pool_bytes(),
          "saving_vs_plain": 1.0 - cache.resident_bytes() / plain_bytes,
          "pool_saving_vs_plain": 1.0 - cache.pool_bytes() / plain_bytes}
    peaks, peak_kind = load_peaks()
    clocks = sampler.summary()
    roofline = tensor_roofline(
        value / world, ms, peaks, peak_kind, clocks, ms * args.steps * 1e-3, traffic=None,
        kernel="attn_fwd_kernel<128> through the page table, with the chunk's mask kernels "
               "(the whole attend step is timed)")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, sample = PagedAROracleSample(w, q_h, k_h, v_h).run(args.cpu_budget)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample}
    if rank == 0:
        line = {"metric": AR_PAGED_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": workload_config(w, "ar_paged"),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                # per attend step: 2 block means, residency, selection, 3 compaction,
                # kept-list build, attention
                "clocks": clocks, "gpu_launches": 9 * args.steps,
                "kv_cache": kv, "plain_path_attend_ms": plain_ms,
                "effective_tflop_per_step": flops / 1e12}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def device_status(ws):
    """The device-side status word of a libbsa workspace (0 = no error)."""
    from block_sparse_attention_tokens_b200 import binding as B
    return B.bsa_read_status(ws)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="radial_long",
                    help="workload name (default: the largest, 453,600-token radial one)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline field")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller cases for profiler captures)")
    ap.add_argument("--pass", dest="pass_", default="fwd",
                    choices=["fwd", "bwd", "sics", "ar_paged"],
                    help="fwd: the whole forward path (default); bwd: the attention "
                         "backward; sics: SPADE scheme generation; ar_paged: the AR decode "
                         "through the paged persistent-anchor KV cache")
    args = ap.parse_args()

    from block_sparse_attention_tokens_b200 import configs
    import dataclasses
    if args.pass_ == "ar_paged" and args.workload == "radial_long":
        args.workload = "ar_decode"
    w = configs.get(args.workload)
    if args.pass_ == "ar_paged" and w.mask != "ar":
        ap.error(f"--pass ar_paged decodes an autoregressive workload (mask 'ar'); "
                 f"{w.name} has mask '{w.mask}'")
    if args.heads > 0:
        w = dataclasses.replace(w, heads=args.heads)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.pass_ == "bwd":
        return run_backward(args, w)
    if args.pass_ == "sics":
        return run_sics(args, w)
    if args.pass_ == "ar_paged":
        return run_ar_paged(args, w)

    import torch
    import torch.distributed as dist
    from block_sparse_attention_tokens_b200 import binding as B
    from block_sparse_attention_tokens_b200 import synth
    from block_sparse_attention_tokens_b200.pipeline import (Plan, effective_flops, head_range,
                                                             qblock_range)

    world, rank, dev = setup_ranks()

    # inputs: the workload's seeded Q, K, V; with N ranks each rank takes its range
    # of heads (masks are per head and every head is independent, so nothing is
    # exchanged) and holds only those heads, as after a head-parallel projection.
    # A raster-order workload whose heads do not split evenly (12 radial heads over
    # 8 GPUs) splits its query blocks instead: each rank takes every head of its
    # query rows, against all keys -- again with no exchange.
    q_all, k_all, v_all, _ = synth.workload_inputs(w)
    split_q = (world > 1 and w.heads % world != 0 and w.tile is None
               and w.mask in ("sta", "radial", "ar"))
    if split_q:
        qb0, qb1 = qblock_range(rank, world, math.ceil(w.nq / w.block),
                                granule=max(1, 128 // w.block))
        q_h = q_all[:, qb0 * w.block:min(w.nq, qb1 * w.block)].contiguous()
        k_h, v_h = k_all, v_all
        plan_kw = {"qblocks": (qb0, qb1)}
        split_text = f"query blocks split over {world} GPU(s), no data-path collective"
    else:
        h0, h1 = head_range(rank, world, w.heads)
        q_h, k_h, v_h = (t_[:, :, h0:h1].contiguous() for t_ in (q_all, k_all, v_all))
        plan_kw = {"heads": (h0, h1)}
        split_text = f"heads split over {world} GPU(s), no data-path collective"
    del q_all, k_all, v_all
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    plan = Plan(w, dev, **plan_kw)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        plan.step(q, k, v)
    barrier()
    flops = effective_flops(plan.mask, plan.nq, plan.nk, w.block, w.head_dim,
                            w.batch * plan.heads)
    flops_all = sum_over_ranks(flops, dev)
    if B.bsa_read_status(plan.attn_ws) != 0:
        raise RuntimeError("attention kernel reported a device-side error")

    # ---- timed region: K whole-path steps, attention launches bracketed by events
    stream = torch.cuda.current_stream()
    ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    # stage boundaries: step start, after the permute, after the mask, step end
    ev_s = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier()
    with sampler:
        time.sleep(0.5)          # let nvidia-smi start sampling before the timed region
        start.record(stream)
        for i in range(args.steps):
            ev_s[i][0].record(stream)
            plan._q, plan._k, plan._v = q, k, v
            if plan.permuted:
                plan.permute_inputs(q, k, v)
            ev_s[i][1].record(stream)
            plan.build_mask()
            ev_s[i][2].record(stream)
            plan.compact()
            ev_a[i][0].record(stream)
            plan.attention()
            ev_a[i][1].record(stream)
            if plan.permuted:
                plan.untile()
            ev_s[i][3].record(stream)
        end.record(stream)
        barrier()
    ms_total = start.elapsed_time(end)
    attn_times = [a.elapsed_time(b) for a, b in ev_a]
    attn_ms = statistics.mean(attn_times)
    stage_ms = {
        "permute": statistics.mean(e[0].elapsed_time(e[1]) for e in ev_s),
        "mask": statistics.mean(e[1].elapsed_time(e[2]) for e in ev_s),
        "compact": statistics.mean(e[2].elapsed_time(a[0]) for e, a in zip(ev_s, ev_a)),
        "attention": attn_ms,
        "untile": statistics.mean(a[1].elapsed_time(e[3]) for e, a in zip(ev_s, ev_a)),
    }
    ms_total, attn_ms = max_over_ranks([ms_total, attn_ms], dev)
    ms_per_step = ms_total / args.steps
    value = job_value(flops_all, ms_per_step)

    # ---- end to end through the public API: pinned host inputs in, O back to host.
    # Steps are pipelined the way a serving loop would run them: the host->device
    # copy of step i+1 (copy stream) and the device->host copy of O of step i-1
    # (out stream) overlap the path of step i (compute stream); device inputs and O
    # are double-buffered.  Every step still moves all of its inputs and its output.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = (t_.pin_memory() for t_ in (q_h, k_h, v_h))
        o_host = torch.empty(plan.o.shape, dtype=plan.o.dtype).pin_memory()
        bufs = [tuple(torch.empty_like(t_) for t_ in (q, k, v)) for _ in range(2)]
        o_bufs = [plan.o, torch.empty_like(plan.o)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        e2e_steps = max(3, args.steps // 2)
        total = 2 + e2e_steps
        ev_in = [torch.cuda.Event() for _ in range(total)]
        ev_done = [torch.cuda.Event() for _ in range(total)]
        ev_out = [torch.cuda.Event() for _ in range(total)]

        def h2d(i):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i - 2])      # buffer free once step i-2 finished
                for dst, src in zip(bufs[i % 2], (qp, kp, vp)):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)

        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h2d(0)
        for i in range(total):
            if i == 2:
                e0.record(stream)
            if i + 1 < total:
                h2d(i + 1)
            stream.wait_event(ev_in[i])
            qd, kd, vd = bufs[i % 2]
            plan._q, plan._k, plan._v = qd, kd, vd
            plan.set_output(o_bufs[i % 2])
            if plan.permuted:
                plan.permute_inputs(qd, kd, vd)
            plan.build_mask()
            plan.compact()
            if i >= 2 and not plan.permuted:
                stream.wait_event(ev_out[i - 2])         # this O buffer copied out (step i-2)
            plan.attention()
            if plan.permuted:
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])     # this O buffer copied out (step i-2)
                plan.untile()
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                o_host.copy_(o_bufs[i % 2], non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_event(ev_out[total - 1])
        plan.set_output(None)
        e1.record(stream)
        barrier()
        # time from the start of step 2 to the end of the last output copy, per step
        e_ms = torch.tensor(max_over_ranks([e0.elapsed_time(e1) / e2e_steps], dev),
                            dtype=torch.float64)
        h2d_bytes = sum(t_.numel() * t_.element_size() for t_ in (q_h, k_h, v_h))
        d2h_bytes = o_host.numel() * o_host.element_size()
        h2d_bytes, d2h_bytes = (int(x) for x in sum_over_ranks([h2d_bytes, d2h_bytes], dev))
        e2e = {"value": job_value(flops_all, e_ms.item()), "unit": "TFLOP/s",
               "ms_per_step": e_ms.item(), "h2d_bytes_per_step": h2d_bytes,
               "d2h_bytes_per_step": d2h_bytes,
               "note": "pinned host buffers (each rank its share of Q, K, V); copies of neighbouring steps "
                       "overlap compute"}

    peaks, peak_kind = load_peaks()
    # the slowest rank's attention time, for that rank's share of the work
    achieved = flops_all / world / (attn_ms * 1e-3) / 1e12
    clocks = sampler.summary()
    gathered = w.block == 64
    roofline = tensor_roofline(
        achieved, attn_ms, peaks, peak_kind, clocks, ms_total * 1e-3,
        traffic=profiled_traffic(w.name),
        kernel=f"attn_fwd_kernel<{w.head_dim}, {'gathered' if gathered else 'adjacent'} key tiles>",
        attn_ms=attn_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, sample = OracleSample(w, q_h, k_h, v_h).run(args.cpu_budget)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample}

    if rank == 0:
        cfg = workload_config(w)
        cfg["parallelism"] = split_text
        line = {"metric": FWD_METRIC,
                "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": cfg,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "clocks": clocks,
                "gpu_launches": plan.kernel_launches_per_step() * args.steps,
                "effective_tflop_per_step": flops_all / 1e12,
                "mask_stats": mask_stats(flops, w, plan.nq, plan.nk, attn_times,
                                         plan.near.item() if hasattr(plan, "near") else None),
                # mean device time of each stage of a timed step (this rank, CUDA events)
                "stage_ms": stage_ms,
                "stage_gbs": permute_bandwidth(w, plan, stage_ms, peaks["hbm_gbs"])}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
