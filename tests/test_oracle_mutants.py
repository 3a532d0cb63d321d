"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case takes the source of one oracle function, turns one expression into a
plausible slip -- a dropped term, an off-by-one, a wrong axis, index or sign, a
swapped operand, an ignored argument -- installs the changed function in place
of the original for the length of the test, and runs the pins that should
notice.  At least one of them must fail with an assertion.  A planted mistake
that every pin lets through marks a property of the oracle that nothing outside
the oracle checks, so each case here is also a statement of what its pins are
for.  The mistakes are planted in the oracle, on the CPU; nothing here touches
the CUDA library.
"""
import inspect
import textwrap
from dataclasses import dataclass, field
from typing import Callable, List, Tuple

import numpy as np
import pytest

import oracle
from oracle import bsa_oracle as M
from tests import test_oracle_masks as TM
from tests import test_oracle_nabla_attention as TN
from tests import test_oracle_paged as TP
from tests import test_oracle_scheme as TSC
from tests import test_oracle_sics as TS


@dataclass
class Mutant:
    id: str
    func: str            # oracle function whose source is changed
    old: str             # exact text in that source (must occur once)
    new: str             # the slip
    pins: List[Tuple[Callable, dict]] = field(default_factory=list)


def pin(fn, **kw):
    return fn, kw


def install(monkeypatch, func, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(M, func)))
    assert src.count(old) == 1, f"{func}: {old!r} occurs {src.count(old)} times"
    ns = dict(vars(M))
    exec(compile(src.replace(old, new), f"<planted mistake in {func}>", "exec"), ns)
    monkeypatch.setattr(M, func, ns[func])
    if hasattr(oracle, func):
        monkeypatch.setattr(oracle, func, ns[func])


MUTANTS = [
    # ------------------------------------------------------------ tile permutation
    Mutant("tile_order/inner-raster-reversed", "tile_order",
           "inner = ((t % tT) * tH + (h % tH)) * tW + (w % tW)",
           "inner = ((w % tW) * tH + (h % tH)) * tT + (t % tT)",
           [pin(TM.test_tile_order_golden_ragged),
            pin(TM.test_tile_order_matches_reshape_transpose_when_divisible,
                grid=(6, 4, 10), tile=(2, 2, 5))]),
    Mutant("tile_order/tile-raster-w-major", "tile_order",
           "tile_id = ((t // tT) * nH + (h // tH)) * nW + (w // tW)",
           "tile_id = ((w // tW) * nH + (h // tH)) * ceil_div(T, tT) + (t // tT)",
           [pin(TM.test_tile_order_matches_reshape_transpose_when_divisible,
                grid=(6, 4, 10), tile=(2, 2, 5)),
            pin(TM.test_tile_order_bijection_and_tile_contiguity, grid=(5, 7, 3), tile=(2, 3, 2))]),
    Mutant("tile_order/floor-tile-count", "tile_order",
           "nH, nW = ceil_div(H, tH), ceil_div(W, tW)",
           "nH, nW = H // tH, W // tW",
           [pin(TM.test_tile_order_golden_ragged),
            pin(TM.test_tile_order_bijection_and_tile_contiguity, grid=(5, 7, 3), tile=(2, 3, 2))]),
    Mutant("tile_permute/inverse-permutation", "tile_permute",
           "y[:, :n] = x[:, perm]", "y[:, perm] = x",
           [pin(TM.test_permute_untile_roundtrip_and_zero_tail)]),
    Mutant("tile_untile/forward-permutation", "tile_untile",
           "x[:, perm] = y[:, :n]", "x[:] = y[:, perm]",
           [pin(TM.test_permute_untile_roundtrip_and_zero_tail)]),
    Mutant("scheme_permute/choice-transposed", "scheme_permute",
           "perm = tile_order(grid, tuple(shapes[int(choice[b, h])]))",
           "perm = tile_order(grid, tuple(shapes[int(choice.reshape(-1)[h * Bt + b])]))",
           [pin(TSC.test_scheme_permute_golden_mixed_choices)]),
    Mutant("scheme_permute/first-head-shape-for-all", "scheme_permute",
           "perm = tile_order(grid, tuple(shapes[int(choice[b, h])]))",
           "perm = tile_order(grid, tuple(shapes[int(choice[b, 0])]))",
           [pin(TSC.test_scheme_permute_golden_mixed_choices)]),
    Mutant("scheme_permute/inverse-permutation", "scheme_permute",
           "y[b, :n, h] = x[b, perm, h]", "y[b, perm, h] = x[b, :, h]",
           [pin(TSC.test_scheme_permute_golden_mixed_choices),
            pin(TSC.test_scheme_roundtrip_random_choices)]),
    Mutant("scheme_untile/forward-permutation", "scheme_untile",
           "x[b, perm, h] = y[b, :n, h]", "x[b, :, h] = y[b, perm, h]",
           [pin(TSC.test_scheme_untile_golden_mixed_choices),
            pin(TSC.test_scheme_roundtrip_random_choices)]),
    Mutant("scheme_untile/batch-0-choice", "scheme_untile",
           "perm = tile_order(grid, tuple(shapes[int(choice[b, h])]))",
           "perm = tile_order(grid, tuple(shapes[int(choice[0, h])]))",
           [pin(TSC.test_scheme_untile_golden_mixed_choices)]),

    # ------------------------------------------------------------ Sliding-Tile window
    Mutant("sta/exclusive-upper-edge", "sta_axis_keep",
           "keep[a, lo:hi + 1] = True", "keep[a, lo:hi] = True",
           [pin(TM.test_sta_golden_band), pin(TM.test_sta_kept_count_closed_form_720p, shift=False)]),
    Mutant("sta/width-as-half-width", "sta_axis_keep",
           "lo_off, hi_off = (w - 1) // 2, w // 2", "lo_off, hi_off = w - 1, w - 1",
           [pin(TM.test_sta_golden_band), pin(TM.test_sta_kept_count_closed_form_720p, shift=False)]),
    Mutant("sta/shifted-window-not-clamped", "sta_axis_keep",
           "start = min(max(a - lo_off, 0), max(n - w, 0))", "start = max(a - lo_off, 0)",
           [pin(TM.test_sta_kept_count_closed_form_720p, shift=True),
            pin(TM.test_sta_matches_token_level_enumeration, shift=True)]),
    Mutant("sta/shifted-window-one-too-wide", "sta_axis_keep",
           "lo, hi = start, min(start + w, n) - 1", "lo, hi = start, min(start + w, n)",
           [pin(TM.test_sta_kept_count_closed_form_720p, shift=True)]),
    Mutant("sta/window-axes-reversed", "sta_tile_mask",
           "zip(tile_grid, window)", "zip(tile_grid, window[::-1])",
           [pin(TM.test_sta_kept_count_closed_form_720p, shift=False)]),
    Mutant("sta/query-tile-index-transposed", "sta_tile_mask",
           "q = (a * nH + b) * nW + c", "q = (c * nH + b) * nT + a",
           [pin(TM.test_sta_symmetric_and_tiny_all_ones),
            pin(TM.test_sta_matches_token_level_enumeration, shift=False)]),

    # ------------------------------------------------------------ radial
    Mutant("radial/full-width-window", "_radial_params",
           "return True, S, 1 << r", "return True, S, 1 << max(r - 1, 0)",
           [pin(TM.test_radial_token_rule_golden)]),
    Mutant("radial/subsampling-inverted", "_radial_params",
           "if dist % (1 << c) != 0:", "if dist % (1 << c) == 0:",
           [pin(TM.test_radial_token_rule_golden)]),
    Mutant("radial/dense-only-same-frame", "radial_token_keep",
           "if dist <= 1:", "if dist < 1:",
           [pin(TM.test_radial_token_rule_golden)]),
    Mutant("radial/window-edge-inclusive", "radial_token_keep",
           "2 * abs(sq - sk) * den < num", "2 * abs(sq - sk) * den <= num",
           [pin(TM.test_radial_token_rule_golden)]),
    Mutant("radial/segment-start-distance", "radial_block_mask",
           "gap = max(0, b0 - a1, a0 - b1)", "gap = abs(b0 - a0)",
           [pin(TM.test_radial_block_mask_equals_token_enumeration, frames=12, S=16, B=4, n=None),
            pin(TM.test_radial_block_mask_equals_token_enumeration, frames=9, S=6, B=8, n=50)]),
    Mutant("radial_fast/missing-straddle-segment", "radial_block_mask_fast",
           "max_segs = ceil_div(block, S) + 1", "max_segs = ceil_div(block, S)",
           [pin(TM.test_radial_block_mask_equals_token_enumeration, frames=11, S=5, B=8, n=None)]),
    Mutant("radial_fast/segment-start-distance", "radial_block_mask_fast",
           "gap = np.maximum(0, np.maximum(seg_a[j] - a1, a0 - seg_b[j]))",
           "gap = np.abs(seg_a[j] - a0)",
           [pin(TM.test_radial_block_mask_equals_token_enumeration, frames=12, S=16, B=4, n=None),
            pin(TM.test_radial_block_mask_equals_token_enumeration, frames=9, S=6, B=8, n=50)]),

    # ------------------------------------------------------------ NABLA
    Mutant("nabla_pool/padding-in-the-mean", "nabla_pool",
           "lo, hi = b * block, min((b + 1) * block, n_valid)",
           "lo, hi = b * block, (b + 1) * block",
           [pin(TN.test_pool_mean_over_valid_tokens_only)]),
    Mutant("nabla_select/crossing-block-dropped", "nabla_select_row",
           "k_star = int(hit[0]) + 1 if hit.size else n",
           "k_star = int(hit[0]) if hit.size else n",
           [pin(TN.test_select_is_minimal_and_covers_p_brute_force, seed=0, p=0.7),
            pin(TN.test_select_uniform_keeps_ceil_p_lowest_indices)]),
    Mutant("nabla_select/ties-to-higher-index", "nabla_select_row",
           'order = np.argsort(-probs, kind="stable")',
           'order = np.argsort(probs, kind="stable")[::-1]',
           [pin(TN.test_select_uniform_keeps_ceil_p_lowest_indices)]),
    Mutant("nabla_select/strict-threshold", "nabla_select_row",
           "hit = np.nonzero(cum >= p)[0]", "hit = np.nonzero(cum > p)[0]",
           [pin(TN.test_select_uniform_keeps_ceil_p_lowest_indices),
            pin(TN.test_select_reaching_p_exactly_covers_it)]),
    Mutant("nabla_mask/logit-scale-dropped", "nabla_mask",
           "z = (qbar[b, h] @ kbar[b, h, cand].T) * scale",
           "z = (qbar[b, h] @ kbar[b, h, cand].T)",
           [pin(TN.test_nabla_mask_range_and_forced_outside)]),
    Mutant("nabla_mask/softmax-over-queries", "nabla_mask",
           "probs = e / e.sum(axis=1, keepdims=True)", "probs = e / e.sum(axis=0, keepdims=True)",
           [pin(TN.test_nabla_mask_range_and_forced_outside)]),
    Mutant("nabla_mask/range-offset-forgotten", "nabla_mask",
           "mask[b, h, qb, cand[kept]] = 1", "mask[b, h, qb, kept] = 1",
           [pin(TN.test_nabla_mask_range_and_forced_outside)]),
    Mutant("nabla_mask/near-flag-ignores-the-previous-prefix", "nabla_mask",
           "flag = abs(c_last - p) < near_tol or abs(c_prev - p) < near_tol",
           "flag = abs(c_last - p) < near_tol",
           [pin(TN.test_near_threshold_flag)]),
    Mutant("nabla_mask/near-flag-ignores-ties", "nabla_mask",
           "flag = flag or abs(a - bb) <= tie_tol * max(a, bb)", "flag = flag",
           [pin(TN.test_near_threshold_flag)]),
    Mutant("nabla_mask/allowed-blocks-ignored", "nabla_mask",
           "cand = cand[key_allowed[b, kb_begin:kb_end]]", "cand = cand",
           [pin(TP.test_nabla_with_allowed_blocks_equals_nabla_on_the_allowed_subset)]),
    Mutant("ar/anchor-blocks-floored", "ar_block_ranges",
           "a_end = ceil_div(anchor_frames * S, block)", "a_end = (anchor_frames * S) // block",
           [pin(TN.test_ar_ranges_match_the_decode_workload)]),
    Mutant("ar/recent-blocks-ceiled", "ar_block_ranges",
           "r_begin = (n_tokens_k - recent_frames * S) // block",
           "r_begin = ceil_div(n_tokens_k - recent_frames * S, block)",
           [pin(TN.test_ar_ranges_match_the_decode_workload)]),
    Mutant("ar_mask/outside-range-not-forced", "ar_mask",
           "force_outside=1", "force_outside=0",
           [pin(TN.test_ar_mask_forces_anchors_and_recent_and_selects_the_middle)]),
    Mutant("ar_mask/anchor-and-recent-counts-swapped", "ar_mask",
           "anchor_frames,\n                                     recent_frames)",
           "recent_frames,\n                                     anchor_frames)",
           [pin(TN.test_ar_mask_forces_anchors_and_recent_and_selects_the_middle)]),
    Mutant("nabla_sta/intersection", "nabla_sta_mask",
           "m | (sta_mask[None, None] != 0)", "m & (sta_mask[None, None] != 0)",
           [pin(TN.test_nabla_sta_union_contains_both_masks)]),

    # ------------------------------------------------------------ compaction
    Mutant("csr/row-pointer-shifted", "mask_to_csr",
           "row_ptr[1:] = np.cumsum(counts)", "row_ptr[:-1] = np.cumsum(counts)",
           [pin(TM.test_mask_to_csr_matches_scipy)]),

    # ------------------------------------------------------------ attention
    Mutant("dense/lse-in-log2", "dense_masked_attention",
           "lse = np.where(empty, NEG_INF, mx_safe + np.log(np.where(empty, 1.0, l)))",
           "lse = np.where(empty, NEG_INF, mx_safe + np.log2(np.where(empty, 1.0, l)))",
           [pin(TN.test_attention_golden_two_keys)]),
    Mutant("token_mask/query-blocks-of-key-size", "token_mask_from_blocks",
           "qi = np.arange(nq) // block_q", "qi = np.arange(nq) // block_k",
           [pin(TN.test_block_mask_equals_token_level_definition, bq=64, bk=128)]),
    Mutant("dense/empty-rows-divide-by-zero", "dense_masked_attention",
           "o = np.where(empty[:, None], 0.0, (e @ v) / np.where(empty, 1.0, l)[:, None])",
           "o = (e @ v) / np.where(empty, 1.0, l)[:, None] + np.where(empty, np.nan, 0.0)[:, None]",
           [pin(TN.test_block_mask_equals_token_level_definition, bq=64, bk=64)]),
    Mutant("attn/scale-1-over-d", "block_sparse_attention",
           "scale = 1.0 / math.sqrt(D) if scale is None else scale",
           "scale = 1.0 / D if scale is None else scale",
           [pin(TN.test_all_ones_mask_equals_sdpa_float64)]),
    Mutant("attn/mask-head-index-transposed", "block_sparse_attention",
           "m = mask[0 if mask.shape[0] == 1 else b * H + h]",
           "m = mask[0 if mask.shape[0] == 1 else h * Bn + b]",
           [pin(TN.test_per_batch_head_masks_index_b_times_h_plus_h)]),
    Mutant("attn/last-key-dropped", "block_sparse_attention",
           "min((kb + 1) * block_k, nk)", "min((kb + 1) * block_k, nk - 1)",
           [pin(TN.test_block_mask_equals_token_level_definition, bq=64, bk=64)]),
    Mutant("attn/lse-max-term-dropped", "block_sparse_attention",
           "lse[b, h, sel] = (mx + np.log(l))[:, 0]", "lse[b, h, sel] = (np.log(l))[:, 0]",
           [pin(TN.test_all_ones_mask_equals_sdpa_float64),
            pin(TN.test_single_kept_block_is_softmax_over_that_block_and_lse_normalises)]),
    Mutant("attn/empty-row-nonzero", "block_sparse_attention",
           "o[b, sel, h] = 0.0", "o[b, sel, h] = v[b, :, h].mean(axis=0)",
           [pin(TN.test_block_mask_equals_token_level_definition, bq=64, bk=64)]),

    # ------------------------------------------------------------ backward
    Mutant("bwd/softmax-jacobian-term-dropped", "block_sparse_attention_backward",
           "ds = p * (dp - (g * o).sum(axis=1, keepdims=True))", "ds = p * dp",
           [pin(TN.test_backward_matches_autograd_float64, bq=64, bk=64)]),
    Mutant("bwd/dk-scale-dropped", "block_sparse_attention_backward",
           "dk[b, keys, h] += (ds.T @ q[b, rows_, h]) * scale",
           "dk[b, keys, h] += (ds.T @ q[b, rows_, h])",
           [pin(TN.test_backward_matches_autograd_float64, bq=64, bk=64)]),
    Mutant("bwd/dv-from-output", "block_sparse_attention_backward",
           "dv[b, keys, h] += p.T @ g", "dv[b, keys, h] += p.T @ o",
           [pin(TN.test_backward_matches_autograd_float64, bq=64, bk=64)]),
    Mutant("bwd/dq-with-v", "block_sparse_attention_backward",
           "dq[b, rows_, h] += (ds @ k[b, keys, h]) * scale",
           "dq[b, rows_, h] += (ds @ v[b, keys, h]) * scale",
           [pin(TN.test_backward_matches_autograd_float64, bq=64, bk=64)]),
    Mutant("bwd/default-scale-1-over-d", "block_sparse_attention_backward",
           "scale = 1.0 / math.sqrt(D) if scale is None else scale",
           "scale = 1.0 / D if scale is None else scale",
           [pin(TN.test_backward_matches_autograd_float64, bq=64, bk=64)]),
    Mutant("bwd/row-sample-ignored", "block_sparse_attention_backward",
           "rows_b = np.intersect1d(rows_b, np.asarray(rows))", "rows_b = rows_b",
           [pin(TN.test_backward_row_sampling_is_exact_on_dq_and_additive_on_dk_dv)]),
    Mutant("bwd/col-sample-in-query-blocks", "block_sparse_attention_backward",
           "np.asarray(cols, dtype=np.int64) // block_k", "np.asarray(cols, dtype=np.int64) // block_q",
           [pin(TN.test_backward_column_sampling_is_exact_on_dk_dv)]),
    Mutant("bwd/col-sample-softmax-over-wanted-blocks-only", "block_sparse_attention_backward",
           "                                       for kb in kept])\n                s = (q",
           "                                       for kb in (kept if want_kb is None else np.intersect1d(kept, want_kb))])\n                s = (q",
           [pin(TN.test_backward_column_sampling_is_exact_on_dk_dv)]),

    # ------------------------------------------------------------ SICS
    Mutant("tile_tokens/ragged-edge-overrun", "tile_tokens",
           "hs = np.arange(b * tH, min(H, b * tH + tH))", "hs = np.arange(b * tH, b * tH + tH)",
           [pin(TS.test_tile_tokens_partition_and_match_tile_order)]),
    Mutant("sics/raw-dot-products", "sics_blocks",
           "out[b, h, t] = (u @ u.T).sum()", "out[b, h, t] = (v @ v.T).sum()",
           [pin(TS.test_sics_equals_squared_norm_of_summed_unit_vectors),
            pin(TS.test_scale_invariance)]),
    Mutant("sics/diagonal-excluded", "sics_blocks",
           "out[b, h, t] = (u @ u.T).sum()", "out[b, h, t] = (u @ u.T).sum() - len(idx)",
           [pin(TS.test_identical_orthogonal_and_opposite_vectors)]),
    Mutant("sics/zero-vector-normalised", "sics_blocks",
           "u = np.where(norm[:, None] > 0, v / np.where(norm > 0, norm, 1.0)[:, None], 0.0)",
           "u = v / np.where(norm > 0, norm, 0.0)[:, None]",
           [pin(TS.test_identical_orthogonal_and_opposite_vectors)]),
    Mutant("scheme/ties-to-later-entry", "sics_scheme",
           "if scores[b, h, si] > scores[b, h, best]:", "if scores[b, h, si] >= scores[b, h, best]:",
           [pin(TS.test_scheme_ties_take_the_first_menu_entry)]),
    Mutant("scheme/not-normalised-by-pairs", "sics_scheme",
           "scores[:, :, si] = total / (2.0 * pairs)", "scores[:, :, si] = total / 2.0",
           [pin(TS.test_scheme_picks_the_slicing_the_field_is_constant_along)]),
    Mutant("scheme/keys-ignored", "sics_scheme",
           "+ sics_blocks(k, grid, shape).sum(axis=2)", "+ sics_blocks(q, grid, shape).sum(axis=2)",
           [pin(TS.test_scheme_scores_queries_and_keys_alike)]),
    Mutant("scheme/argmin", "sics_scheme",
           "if scores[b, h, si] > scores[b, h, best]:", "if scores[b, h, si] < scores[b, h, best]:",
           [pin(TS.test_scheme_picks_the_slicing_the_field_is_constant_along)]),

    # ------------------------------------------------------------ paged KV cache
    Mutant("paged_view/page-table-ignored", "paged_view",
           "out[b, lo:hi] = pool[page_table[b, pg], :hi - lo]",
           "out[b, lo:hi] = pool[b * n_pages + pg, :hi - lo]",
           [pin(TP.test_paged_view_identity_shuffled_and_evicted)]),
    Mutant("resident/block-index-as-token", "resident_blocks",
           "pages = (np.arange(KB) * block) // page_tokens", "pages = np.arange(KB) // page_tokens",
           [pin(TP.test_paged_attention_equals_plain_and_drops_evicted_pages)]),
    Mutant("paged_attn/evicted-blocks-kept", "paged_block_sparse_attention",
           "m = (m * res[:, None, None, :])", "m = (m * 1)",
           [pin(TP.test_paged_attention_equals_plain_and_drops_evicted_pages)]),
    Mutant("page_scores/max-not-sum", "kv_page_scores",
           "mass = probs.sum(axis=0)", "mass = probs.max(axis=0)",
           [pin(TP.test_page_scores_sum_to_rows_and_follow_a_dominant_block)]),
    Mutant("page_scores/allowed-blocks-ignored", "kv_page_scores",
           "cand = cand[key_allowed[b, kb_begin:kb_end]]", "cand = cand",
           [pin(TP.test_page_scores_sum_to_rows_and_follow_a_dominant_block)]),
    Mutant("keep_pages/least-important-kept", "kv_keep_pages",
           "mid.sort(key=lambda pg: (-scores[b, pg], pg))", "mid.sort(key=lambda pg: (scores[b, pg], pg))",
           [pin(TP.test_keep_pages_anchors_recent_and_budget)]),
    Mutant("keep_pages/evicted-pages-revived", "kv_keep_pages",
           "mid = [pg for pg in range(anchor_pages, recent_begin) if resident[b, pg]]",
           "mid = list(range(anchor_pages, recent_begin))",
           [pin(TP.test_keep_pages_anchors_recent_and_budget)]),
    Mutant("keep_pages/last-anchor-page-dropped", "kv_keep_pages",
           "keep[:, :anchor_pages] = True", "keep[:, :anchor_pages - 1] = True",
           [pin(TP.test_keep_pages_anchors_recent_and_budget)]),
    Mutant("keep_pages/first-recent-page-dropped", "kv_keep_pages",
           "keep[:, recent_begin:] = True", "keep[:, recent_begin + 1:] = True",
           [pin(TP.test_keep_pages_anchors_recent_and_budget)]),
    Mutant("keep_pages/tie-to-higher-page", "kv_keep_pages",
           "mid.sort(key=lambda pg: (-scores[b, pg], pg))", "mid.sort(key=lambda pg: (-scores[b, pg], -pg))",
           [pin(TP.test_keep_pages_anchors_recent_and_budget)]),
]


@pytest.mark.parametrize("case", MUTANTS, ids=[c.id for c in MUTANTS])
def test_planted_mistake_fails_a_pin(case, monkeypatch):
    install(monkeypatch, case.func, case.old, case.new)
    caught = []
    for fn, kw in case.pins:
        try:
            with np.errstate(all="ignore"):      # a planted slip may divide by zero
                fn(**kw)
        except AssertionError:
            caught.append(fn.__name__)
    assert caught, f"no pin notices the planted mistake {case.id}"


def test_every_public_oracle_function_has_a_planted_mistake():
    covered = {c.func for c in MUTANTS}
    helpers = {"ceil_div"}
    public = {n for n, f in vars(M).items()
              if inspect.isfunction(f) and f.__module__ == M.__name__ and not n.startswith("_")}
    assert public - helpers <= covered, sorted(public - helpers - covered)


def test_pins_pass_on_the_unchanged_oracle():
    for case in MUTANTS:
        for fn, kw in case.pins:
            fn(**kw)
