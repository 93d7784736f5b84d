"""The roofline numerators: the bench's algorithmic bytes per launch, against the count
worked out by hand from the shapes (Qwen3-8B: batch 16, 4 tapped layers, 8 KV / 32 query
heads, head_dim 128, B 16, W 512, scales 64/512/4096 x 32 slots, bf16 rows, fp32 sums)."""

import bench
from fixed_cost_drafter_b200 import workloads as WL


def test_attention_bytes_by_hand():
    wl = WL.CONFIGS["qwen3_8b_64k"]
    tiles = 16 * 4 * 8
    q_and_o = 2 * (16 * 4 * 16 * 32 * 128 * 2)          # 8.39 MB each way
    window = tiles * 512 * 2 * 128 * 2                   # 512 ring rows, K and V
    summary = tiles * (3 * 33 + 1) * 2 * 128 * 2         # 100 mean rows, K and V
    boundary = tiles * 2 * 128 * 2                       # the boundary key and value rows
    counters = 16 * 4 * 4 * 8
    assert bench.attend_bytes(wl) == q_and_o + window + summary + boundary + counters == 177_473_536
    # the view ablations drop exactly their rows
    assert bench.attend_bytes(wl, bench.VIEW_ALL & ~bench.VIEW_WINDOW) == 177_473_536 - window
    assert bench.attend_bytes(wl, bench.VIEW_ALL & ~bench.VIEW_SUMMARY) == 177_473_536 - summary
    assert bench.attend_bytes(wl, bench.VIEW_ALL & ~bench.VIEW_BOUNDARY) == 177_473_536 - boundary


def test_commit_bytes_by_hand():
    wl = WL.CONFIGS["qwen3_8b_64k"]
    delta = 6.0  # a = 5 accepted drafts, plus the bonus row
    tiles = 16 * 4 * 8
    rows = 2 * (16 * delta * 4 * 8 * 2 * 128 * 2)        # retained rows read, ring rows written
    sums = 2 * tiles * 4 * 2 * 128 * 4                   # fp32 partial (3 scales) + global sums, RMW
    finished = tiles * 2 * 128 * (4 + 2) * (delta / 64 + delta / 512 + delta / 4096)
    mean_rows = tiles * 4 * 2 * 128 * 2                  # partial and global mean rows refreshed
    boundary = 2 * 16 * 4 * 4096 * 2                     # hidden row gathered and written
    ids = 16 * 33 * 4 + 8 * 16
    counters = 2 * 16 * 4 * 4 * 8
    want = int(rows + sums + finished + mean_rows + boundary + ids + counters)
    assert bench.commit_bytes(wl, delta) == want == 9_527_616
