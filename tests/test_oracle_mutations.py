"""Plant plausible mistakes in the oracle (CPU only) and check that the pins catch them.

Each mutant replaces one oracle function with a subtly wrong copy (a dropped term,
a wrong sign, a transposed operand, a non-strict comparison, a wrong tie-break);
the test passes only if at least one pin then fails.
"""
import dataclasses
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle.attention as OA
import oracle.flashblock as OF
import oracle.sparse as OS
import oracle.transition as OT
import oracle.similarity as OSim
import oracle.losa as OL

from tests import test_oracle_attention as TA
from tests import test_oracle_flashblock as TF
from tests import test_oracle_sparse as TS
from tests import test_oracle_transition as TT
from tests import test_oracle_similarity as TSim
from tests import test_oracle_losa as TL

_orig_attend = OA.attend
_orig_merge = OA.merge


def _merge_den_drop(a1, l1, a2, l2):
    m = np.maximum(l1, l2)
    w1, w2 = np.exp(l1 - m), np.exp(l2 - m)
    return (w1[..., None] * a1 + w2[..., None] * a2) / np.maximum(w1, 1e-300)[..., None], m + np.log(w1 + w2)


def _merge_L_drop(a1, l1, a2, l2):
    A, L = _orig_merge(a1, l1, a2, l2)
    m = np.maximum(l1, l2)
    return A, np.where(np.isneginf(m), m, m)


def _merge_sign(a1, l1, a2, l2):
    m = np.maximum(l1, l2)
    w1, w2 = np.exp(m - l1), np.exp(m - l2)
    return (w1[..., None] * a1 + w2[..., None] * a2) / (w1 + w2)[..., None], m + np.log(w1 + w2)


def _attend_no_scale(q, k, v, scale):
    return _orig_attend(q, k, v, 1.0)


def _attend_kv_swapped(q, k, v, scale):
    if k.shape == v.shape:
        return _orig_attend(q, k, k, scale)
    return _orig_attend(q, k, v, scale)


def _attend_L_no_max(q, k, v, scale):
    A, L = _orig_attend(q, k, v, scale)
    if k.shape[0] == 0:
        return A, L
    s = scale * (np.asarray(q) @ np.asarray(k).T)
    return A, np.log(np.exp(s - s.max(1, keepdims=True)).sum(1))


def _attend_values_rolled(q, k, v, scale):
    # each key paired with the next key's value
    v = np.asarray(v)
    return _orig_attend(q, k, np.roll(v, 1, axis=0) if v.shape[0] > 1 else v, scale)


def _tau_le(M, tau, first_step):
    return np.zeros(M.shape, bool) if first_step else M <= tau


def _gamma_ge(sim, gamma, first_step, shape):
    if first_step:
        return np.zeros(shape, bool)
    if sim is None:
        return np.ones(shape, bool)
    return np.asarray(sim, np.float32) >= np.float32(gamma)


def _est_min(q_rows, kmin, kmax):
    q_rows = np.asarray(q_rows, np.float64)
    est = np.zeros((q_rows.shape[0], kmin.shape[0]))
    for d in range(q_rows.shape[1]):
        qd = q_rows[:, d:d + 1]
        est = est + np.minimum(qd * kmin[None, :, d], qd * kmax[None, :, d])
    return est


def _select_high_tie(est, k_sel):
    out = np.zeros((est.shape[0], k_sel), dtype=np.int64)
    for r in range(est.shape[0]):
        order = sorted(range(est.shape[1]), key=lambda p: (-est[r, p], -p))
        out[r] = np.sort(order[:k_sel])
    return out


_orig_update = OT.update_page_minmax
_orig_append = OT.append_block


def _update_skips_partial_page(kmin, kmax, k_grown, n_old, page):
    # starts at the first page after the old rows, leaving a partial page stale
    return _orig_update(kmin, kmax, k_grown, -(-n_old // page) * page, page) if n_old % page else \
        _orig_update(kmin, kmax, k_grown, n_old, page)


def _append_block_first(k_cache, v_cache, k_blk, v_blk):
    # block placed before the prefix instead of after it
    return _orig_append(k_blk, v_blk, k_cache, v_cache)


_orig_ordered_sum = OSim._ordered_sum


def _sum_pairwise(row_terms):
    # rows added as a pairwise tree (neighbours first) instead of one after another
    x = list(np.asarray(row_terms, np.float64))
    while len(x) > 1:
        x = [x[i] + x[i + 1] if i + 1 < len(x) else x[i] for i in range(0, len(x), 2)]
    return float(x[0]) if x else 0.0


_orig_row_dots = OSim._row_dots


def _row_dots_descending(a, b):
    # channels added from the last to the first
    return _orig_row_dots(np.asarray(a)[:, ::-1], np.asarray(b)[:, ::-1])


def _sim_no_sqrt(q, q_ref):
    q = np.asarray(q, np.float64)
    r = np.asarray(q_ref, np.float64)
    out = np.zeros(q.shape[:2], np.float32)
    for bi in range(q.shape[0]):
        for h in range(q.shape[1]):
            a = _orig_ordered_sum(OSim._row_dots(q[bi, h], r[bi, h]))
            n = _orig_ordered_sum(OSim._row_dots(q[bi, h], q[bi, h])) * _orig_ordered_sum(
                OSim._row_dots(r[bi, h], r[bi, h]))
            out[bi, h] = np.float32(a / n) if n > 0 else np.float32(0.0)
    return out


_orig_token_mse = OL.token_mse
_orig_union = OL.union_bitmap


def _mse_no_mean(q, q_prev):
    # the squared differences summed but not divided by H_q * D
    return (_orig_token_mse(q, q_prev).astype(np.float64) * (np.asarray(q).shape[1] * np.asarray(q).shape[3])
            ).astype(np.float32)


def _union_with_stable_rows(sel_rows, n_pages_):
    # stable rows' -1 entries folded in as page 0 (the union taken over every row)
    s = np.asarray(sel_rows)
    return _orig_union(np.concatenate([s, np.zeros(1, np.int64)]), n_pages_)


def _n_selected_floor(n_prefix, page, density):
    # k rounded down instead of up
    P = OS.n_pages(n_prefix, page)
    return min(P, max(1 if P else 0, math.floor(Fraction(str(density)) * P)))


def _page_minmax_zero_padded(k, page):
    # the partial last page padded with zero rows that enter its bounds
    N, D = k.shape
    P = -(-N // page)
    pad = np.zeros((P * page, D))
    pad[:N] = k
    blk = pad.reshape(P, page, D)
    return blk.min(axis=1), blk.max(axis=1)


_orig_key_mask = OS.key_mask_from_pages


def _key_mask_complement(sel_rows, n_prefix, page):
    # selected and residual key sets swapped
    return ~_orig_key_mask(sel_rows, n_prefix, page)


def _updated_count_complement(mask):
    # counts the tokens that were not updated
    m = np.asarray(mask)
    return (m == 0).reshape(m.shape[0], -1).sum(axis=1).astype(np.int64)


_orig_step = OF.CachedBlockAttention.step


def _step_refreshes_cache(self, q, k_blk, v_blk, mask, first_step, tau, sim=None, gamma=0.0):
    # every step recomputes the cache (a reuse step refreshes it with the new queries)
    if self.a_out is None:
        return _orig_step(self, q, k_blk, v_blk, mask, first_step, tau, sim, gamma)
    r = _orig_step(self, q, k_blk, v_blk, mask, True, tau, sim, gamma)
    M, reuse = OF.decisions(np.asarray(mask), first_step, tau, sim, gamma, np.asarray(q).shape[1])
    return dataclasses.replace(r, M=M, reuse=reuse)


def _active_ge(mse, delta):
    # a token whose score equals delta counted as active
    return np.asarray(mse, np.float32) >= np.float32(delta)


_orig_refresh = OSim.refresh_reference


def _refresh_reusing_heads(q, q_ref, reuse):
    # the reusing heads take the new queries instead of the recomputing ones
    return _orig_refresh(q, q_ref, ~np.asarray(reuse, bool))


PINS_ATTN = [
    lambda: TA.test_attend_matches_torch_sdpa_and_logsumexp(3, 7, 16, 0.25),
    lambda: TA.test_key_order_does_not_matter(),
    lambda: TA.test_common_score_shift_moves_L_only(),
    lambda: TA.test_golden_attention_cases(),
    lambda: TA.test_golden_merge_cases(),
    lambda: TA.test_merge_of_partition_equals_dense_over_union(0),
]
PINS_GATE = [lambda: TF.test_golden_gate_cases(),
             lambda: TF.test_updated_count_and_decision_per_step(),
             lambda: TF.test_updated_count_counts_nonzero_entries()]
PINS_STEP = [lambda: TF.test_tau_above_block_reuses_after_first_step(),
             lambda: TF.test_reuse_rows_with_unchanged_query_equal_dense()]
PINS_SPARSE = [lambda: TS.test_page_estimate_bounds_every_score_in_page(),
               lambda: TS.test_select_pages_matches_full_lexsort(0),
               lambda: TS.test_select_ties_prefer_lower_page(),
               lambda: TS.test_n_selected(),
               lambda: TS.test_page_minmax_partial_last_page(),
               lambda: TS.test_page_minmax_partial_page_ignores_missing_rows(),
               lambda: TS.test_density_one_leaves_empty_residual_and_equals_dense(),
               lambda: TS.test_selected_part_is_attention_over_selected_pages()]

PINS_TRANSITION = [lambda: TT.test_incremental_page_bounds_equal_recomputed(17, 4),
                   lambda: TT.test_appended_prefix_is_old_prefix_then_block(37, 5),
                   lambda: TT.test_generation_first_steps_are_dense_over_all_earlier_blocks()]

PINS_SIM = [lambda: TSim.test_matches_library_cosine(300),
            lambda: TSim.test_closed_forms(),
            lambda: TSim.test_rows_added_in_ascending_order(),
            lambda: TSim.test_channels_added_in_ascending_order(),
            lambda: TSim.test_sum_error_within_the_sequential_bound(),
            lambda: TSim.test_refresh_reference_takes_recomputing_heads()]

PINS_LOSA = [lambda: TL.test_token_mse_matches_library_mean(),
             lambda: TL.test_union_is_over_active_rows_only(),
             lambda: TL.test_delta_zero_keeps_unmoved_tokens_stable()]

MUTANTS = [
    ("merge: denominator drops w_in", [(OA, "merge"), (OF, "merge"), (OS, "merge")], _merge_den_drop, PINS_ATTN),
    ("merge: L drops ln(w1+w2)", [(OA, "merge"), (OF, "merge"), (OS, "merge")], _merge_L_drop, PINS_ATTN),
    ("merge: exponent sign flipped", [(OA, "merge"), (OF, "merge"), (OS, "merge")], _merge_sign, PINS_ATTN),
    ("attend: softmax scale dropped", [(OA, "attend"), (OF, "attend"), (OS, "attend")], _attend_no_scale, PINS_ATTN),
    ("attend: K used in place of V", [(OA, "attend"), (OF, "attend"), (OS, "attend")], _attend_kv_swapped, PINS_ATTN),
    ("attend: values paired with the wrong keys", [(OA, "attend"), (OF, "attend"), (OS, "attend")],
     _attend_values_rolled, PINS_ATTN),
    ("attend: L drops the max term", [(OA, "attend"), (OF, "attend"), (OS, "attend")], _attend_L_no_max, PINS_ATTN),
    ("tau gate: <= instead of <", [(OF, "tau_reuse")], _tau_le, PINS_GATE),
    ("gamma gate: >= instead of >", [(OF, "gamma_reuse")], _gamma_ge, PINS_GATE),
    ("page bound: min instead of max", [(OS, "page_estimates")], _est_min, PINS_SPARSE),
    ("top-k: ties to the higher page", [(OS, "select_pages")], _select_high_tie, PINS_SPARSE),
    ("transition: partial page left stale", [(OT, "update_page_minmax")], _update_skips_partial_page,
     PINS_TRANSITION),
    ("transition: block before the prefix", [(OT, "append_block")], _append_block_first, PINS_TRANSITION),
    ("similarity: rows summed as a pairwise tree", [(OSim, "_ordered_sum")], _sum_pairwise, PINS_SIM),
    ("similarity: channels summed in descending order", [(OSim, "_row_dots")], _row_dots_descending, PINS_SIM),
    ("similarity: norm without the square root", [(OSim, "head_similarity")], _sim_no_sqrt, PINS_SIM),
    ("LoSA: score summed, not averaged", [(OL, "token_mse")], _mse_no_mean, PINS_LOSA),
    ("LoSA: union over every row", [(OL, "union_bitmap")], _union_with_stable_rows, PINS_LOSA),
    ("LoSA: score equal to delta counted active", [(OL, "active_tokens")], _active_ge, PINS_LOSA),
    ("top-k size: floor instead of ceil", [(OS, "n_selected"), (OL, "n_selected")], _n_selected_floor, PINS_SPARSE),
    ("page bounds: partial page padded with zeros", [(OS, "page_minmax"), (OL, "page_minmax")],
     _page_minmax_zero_padded, PINS_SPARSE),
    ("sparse: selected and residual keys swapped", [(OS, "key_mask_from_pages"), (OL, "key_mask_from_pages")],
     _key_mask_complement, PINS_SPARSE),
    ("M: counts the tokens not updated", [(OF, "updated_count")], _updated_count_complement, PINS_GATE),
    ("cached step: reuse refreshes the cache", [(OF.CachedBlockAttention, "step")], _step_refreshes_cache,
     PINS_STEP),
    ("similarity: reusing heads refresh their reference", [(OSim, "refresh_reference")], _refresh_reusing_heads,
     PINS_SIM),
]


@pytest.mark.parametrize("name,targets,mutant,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, targets, mutant, pins):
    for mod, attr in targets:
        if hasattr(mod, attr):
            monkeypatch.setattr(mod, attr, mutant)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake: {name}"


def test_pins_pass_on_unmutated_oracle():
    for pin in PINS_ATTN + PINS_GATE + PINS_STEP + PINS_SPARSE + PINS_TRANSITION + PINS_SIM + PINS_LOSA:
        pin()
