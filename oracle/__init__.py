"""CPU oracle of the LongSpark drafting round (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` and
``--impl reference`` legs may import this package; the CUDA library never does.
"""
from .longspark_oracle import (  # noqa: F401
    BF16, F32, VIEW_ALL, VIEW_BOUNDARY, VIEW_SUMMARY, VIEW_WINDOW, Shapes, Views, accept_decisions,
    accept_sampled, accept_scan, draw_weights, inverse_cdf, sampling_weights,
    attention_slots, commit_round, commit_round_paged, draft_attend, draft_prologue, empty_views, paged_rows, prefill, prefill_paged, retain_row, segment_count,
    softmax_scale_for, state_bytes, to_f64, view_of_slots, views_from_scratch,
)
