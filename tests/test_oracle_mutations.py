"""Each plausible mistake planted in the oracle must make at least one pin fail.

The mistakes are planted on the CPU, in the oracle only, through monkeypatching; the
pins are the functions of test_oracle_pins.py.
"""

import numpy as np
import pytest

import oracle
import oracle.longspark_oracle as M
import tests.test_oracle_pins as P


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(M, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _scan_off_by_one(draft, target):
    a, _ = ORIG["accept_scan"](draft, target)
    a = min(a + 1, len(draft))
    return a, int(target[a])


def _retain_wrong_slot(sh, v, k_row, v_row):
    # finalised segment written one slot too far
    p = v.length
    v.ring_k[:, :, p % sh.window, :] = k_row
    v.ring_v[:, :, p % sh.window, :] = v_row
    for k, s in enumerate(sh.scales):
        v.part_k[k] += k_row
        v.part_v[k] += v_row
        v.part_count[k] += 1
        if v.part_count[k] == s:
            j = v.n_seg[k]
            v.seg_k[k][:, :, (j + 1) % sh.slots, :] = v.part_k[k] / s
            v.seg_v[k][:, :, (j + 1) % sh.slots, :] = v.part_v[k] / s
            v.n_seg[k] += 1
            v.part_k[k] = np.zeros_like(v.part_k[k])
            v.part_v[k] = np.zeros_like(v.part_v[k])
            v.part_count[k] = 0
    v.glob_k += k_row
    v.glob_v += v_row
    v.length = p + 1


def _scratch_relative_alignment(sh, full_k, full_v, n, boundary=None):
    # segments aligned to the end of the cache instead of absolute position 0
    v = ORIG["views_from_scratch"](sh, full_k, full_v, n, boundary)
    for k, s in enumerate(sh.scales):
        off = n % s
        n_c = n // s
        for j in range(max(0, n_c - sh.slots), n_c):
            lo = off + j * s
            v.seg_k[k][:, :, j % sh.slots, :] = full_k[:, :, lo:lo + s, :].mean(axis=2)
            v.seg_v[k][:, :, j % sh.slots, :] = full_v[:, :, lo:lo + s, :].mean(axis=2)
    return v


def _slots_without_partials(sh, v, l, g, bk, bv):
    K, V, ok = ORIG["attention_slots"](sh, v, l, g, bk, bv)
    ok = ok.copy()
    for k in range(len(sh.scales)):
        ok[1 + sh.window + k * (sh.slots + 1) + sh.slots] = False
    return K, V, ok


def _attend_wrong_group(sh, v, q, bk, bv, scale):
    out = np.zeros_like(q)
    for l in range(sh.n_layers):
        for qh in range(sh.n_q_heads):
            K, V, ok = M.attention_slots(sh, v, l, qh % sh.n_kv_heads, bk, bv)
            lg = q[l, :, qh] @ K.T * scale
            lg[:, ~ok] = -np.inf
            w = np.exp(lg - lg.max(axis=1, keepdims=True))
            out[l, :, qh] = (w / w.sum(axis=1, keepdims=True)) @ V
    return out


def _slots_window_mask_off_by_one(sh, v, l, g, bk, bv):
    K, V, ok = ORIG["attention_slots"](sh, v, l, g, bk, bv)
    ok = ok.copy()
    for r in range(sh.window):
        ok[1 + r] = r <= v.length
    return K, V, ok


def _retain_global_skips(sh, v, k_row, v_row):
    ORIG["retain_row"](sh, v, k_row, v_row)
    if v.length == 1:  # first row never reaches the global sum
        v.glob_k -= k_row
        v.glob_v -= v_row


def _views_global_in_window(sh):
    # the global-mean slot (the last one) attributed to the window view
    vs = ORIG["view_of_slots"](sh).copy()
    vs[-1] = M.VIEW_WINDOW
    return vs


def _views_boundary_in_summary(sh):
    vs = ORIG["view_of_slots"](sh).copy()
    vs[0] = M.VIEW_SUMMARY
    return vs


def _residual_swapped(q_rows, p_rows, a):
    # max(0, q - p) instead of max(0, p - q) after a rejection
    if a < q_rows.shape[0]:
        return np.maximum(0.0, q_rows[a].astype(np.float64) - p_rows[a].astype(np.float64))
    return p_rows[-1].astype(np.float64)


def _accept_ratio_inverted(draft_ids, q_rows, p_rows, u):
    # keep when u * p < q
    return ORIG["accept_decisions"](draft_ids, p_rows[:len(draft_ids)], q_rows, u)


def _paged_offset_from_page_end(pages, block_table, page_size, b, positions):
    # offset counted from the end of the page instead of its start
    pages = np.asarray(pages)
    out = ORIG["paged_rows"](pages, block_table, page_size, b, positions)
    for i, pos in enumerate(positions):
        out[:, i] = pages[:, int(block_table[b][pos // page_size]), page_size - 1 - pos % page_size]
    return out


def _paged_commit_from_position_zero(sh, v, draft_ids, target_ids, k_pages, v_pages, block_table, page_size, b,
                                     verify_hidden):
    # verify rows read from the start of the sequence instead of its current length
    pos = range(sh.block + 1)
    return M.commit_round(sh, v, draft_ids, target_ids, M.paged_rows(k_pages, block_table, page_size, b, pos),
                          M.paged_rows(v_pages, block_table, page_size, b, pos), verify_hidden)


def _inverse_cdf_side_left(w, v):
    # the first token whose running sum reaches (instead of passes) the threshold
    c = np.cumsum(w)
    t = int(np.searchsorted(c, v * c[-1], side="left"))
    return min(t, len(w) - 1)


def _paged_rows_first_sequence(pages, block_table, page_size, b, positions):
    # every sequence read through sequence 0's row of the block table
    return ORIG["paged_rows"](pages, block_table, page_size, 0, positions)


def _residual_from_next_position(q_rows, p_rows, a):
    # the residual built from the target's row after the rejected position
    B = q_rows.shape[0]
    if a < B:
        return np.maximum(0.0, p_rows[a + 1].astype(np.float64) - q_rows[a].astype(np.float64))
    return p_rows[B].astype(np.float64)


def _zero_mass_emits_rejected_draft(draft_ids, q_rows, p_rows, u, v):
    # a residual without mass answered with the rejected draft token itself
    a, _ = M.accept_decisions(draft_ids, q_rows, p_rows, u)
    w = M.sampling_weights(q_rows, p_rows, a)
    if not (w > 0).any():
        return a, int(draft_ids[a]) if a < len(draft_ids) else 0
    return a, M.inverse_cdf(w, v)


def _inverse_cdf_one_past(w, v):
    # the index after the one whose running sum passes the threshold (clamped)
    return min(ORIG["inverse_cdf"](w, v) + 1, len(w) - 1)


def _prologue_layer0_weights(w_kv, w_q, boundary, x):
    # every layer projected with layer 0's weights
    w_kv, w_q = np.asarray(w_kv), np.asarray(w_q)
    return ORIG["draft_prologue"](np.broadcast_to(w_kv[:1], w_kv.shape), np.broadcast_to(w_q[:1], w_q.shape),
                                  boundary, x)


ORIG = {n: getattr(M, n) for n in ("accept_scan", "retain_row", "views_from_scratch",
                                   "attention_slots", "draft_attend", "view_of_slots",
                                   "accept_decisions", "sampling_weights", "draft_prologue", "paged_rows",
                                   "inverse_cdf", "accept_sampled")}

CASES = [
    ("accept_scan", _scan_off_by_one, [P.test_scan_golden_examples]),
    ("retain_row", _retain_wrong_slot, [lambda: P.test_ramp_closed_forms(513)]),
    ("views_from_scratch", _scratch_relative_alignment, [lambda: P.test_incremental_equals_recompute(123)]),
    ("attention_slots", _slots_without_partials, [P.test_golden_worked_example]),
    ("draft_attend", _attend_wrong_group, [P.test_attend_matches_torch_sdpa]),
    ("attention_slots", _slots_window_mask_off_by_one, [P.test_mask_counts]),
    ("retain_row", _retain_global_skips, [lambda: P.test_ramp_closed_forms(200)]),
    ("view_of_slots", _views_global_in_window, [P.test_views_constant_values_per_view]),
    ("view_of_slots", _views_boundary_in_summary, [P.test_views_boundary_alone_is_its_value]),
    ("sampling_weights", _residual_swapped, [P.test_sampled_emits_target_distribution]),
    ("accept_decisions", _accept_ratio_inverted, [P.test_sampled_emits_target_distribution]),
    ("draft_prologue", _prologue_layer0_weights, [P.test_prologue_orientation_and_layers]),
    ("paged_rows", _paged_offset_from_page_end, [P.test_paged_rows_hand_worked]),
    ("paged_rows", _paged_rows_first_sequence, [P.test_paged_rows_hand_worked]),
    ("inverse_cdf", _inverse_cdf_side_left, [P.test_inverse_cdf_boundaries]),
    ("sampling_weights", _residual_from_next_position, [P.test_sampled_emits_target_distribution]),
    ("commit_round_paged", _paged_commit_from_position_zero, [lambda: P.test_paged_commit_equals_dense(3)]),
    ("accept_sampled", _zero_mass_emits_rejected_draft, [P.test_sampled_residual_without_mass_draws_from_target_row]),
    ("inverse_cdf", _inverse_cdf_one_past, [P.test_inverse_cdf_exact_brute_force]),
]


@pytest.mark.parametrize("name,fn,pins", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, fn, pins):
    _patch(monkeypatch, name, fn)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()
