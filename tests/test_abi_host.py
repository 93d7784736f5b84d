"""CPU checks of the C ABI: the library loads without a GPU, exports every declared entry
point, validates configurations and lays out a fixed-size state arena."""

import ctypes
import os
import re

import pytest

import fixed_cost_drafter_b200 as F

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "longspark.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LS_API\s+[\w\s\*]+?\b(ls_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(F.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(F.EXPORTED) == names


def _cfg(**kw):
    base = dict(batch=16, n_layers=4, n_kv_heads=8, n_q_heads=32, head_dim=128, hidden=4096, block=16,
                window=512, scales=[64, 512, 4096], slots_per_scale=32, dtype=F.LS_BF16)
    base.update(kw)
    return F.make_config(**base)


def test_layout_sizes():
    c = _cfg()
    y = F.ls_get_layout(c)
    b, L, H, D, nsc, sl = 16, 4, 8, 128, 3, 32
    R = 512 + nsc * (sl + 1) + 1
    assert y.kv_rows == R == 612 and y.elem_bytes == 2
    assert y.off_seg_mean - y.off_kv >= b * L * H * 2 * R * D * 2
    assert y.off_part_sum - y.off_seg_mean >= b * L * H * nsc * sl * 2 * D * 4
    assert y.off_glob_sum - y.off_part_sum >= b * L * H * nsc * 2 * D * 4
    assert y.off_boundary - y.off_glob_sum >= b * L * H * 2 * D * 4
    assert y.off_sample - y.off_boundary >= b * L * 4096 * 2 and y.off_prologue - y.off_sample >= b * 65 * 4
    # the projections' scratch: 320 split-tile slots of 128 x 16 fp32 partial sums, 160 counts
    assert y.total_bytes - y.off_prologue == 320 * 128 * 16 * 4 + 160 * 4 + 256 - (320 * 128 * 16 * 4 + 160 * 4) % 256
    for off in (y.off_counters, y.off_error, y.off_sync, y.off_kv, y.off_seg_mean, y.off_part_sum, y.off_glob_sum,
                y.off_boundary, y.off_sample, y.off_prologue, y.total_bytes):
        assert off % 256 == 0
    assert F.ls_state_bytes(c) == y.total_bytes
    # about 13.3 MB per sequence of views at Qwen3-8B shapes, whatever the prefix, plus the
    # 2.6 MB scratch of the projections for the whole batch
    assert 13.2e6 < y.off_prologue / 16 < 13.4e6 and y.total_bytes - y.off_prologue < 2.7e6
    # no scratch where the projections do not run (fp32 state)
    y32 = F.ls_get_layout(_cfg(dtype=F.LS_F32))
    assert y32.total_bytes == y32.off_prologue


def test_view_state_bytes():
    """Per-view state sizes at Qwen3-8B shapes (the state side of Table 5's ablations):
    per sequence the window is 4 layers x 8 heads x 512 rows x (K, V) x 128 x 2 B
    = 8.39 MB, the summary 100 rows x (fp32 + the bf16 copy) = 4.92 MB and the boundary
    4 x 4096 x 2 B = 32 KB; the counters are always kept."""
    c = _cfg()
    b, L, H, D = 16, 4, 8, 128
    counters = b * L * 4 * 8
    win = b * L * H * 512 * 2 * D * 2
    summ = b * L * H * 2 * 100 * D * (4 + 2)
    bnd = b * L * 4096 * 2
    assert win / b == 8388608 and summ / b == 4915200 and bnd / b == 32768
    want = {F.LS_VIEW_WINDOW: win, F.LS_VIEW_SUMMARY: summ, F.LS_VIEW_BOUNDARY: bnd}
    for views in range(1, 8):
        n = counters + sum(v for bit, v in want.items() if views & bit)
        assert F.ls_view_state_bytes(c, views) == n, views
    everything = F.ls_view_state_bytes(c, F.LS_VIEW_ALL)
    # the arena adds the error word, the commit's arrival counts, the sampler's scratch
    # (counts, 64 chunk sums and 64 x 64 segment sums per sequence), the projections'
    # scratch and the 256-byte alignment of its 11 regions
    extra = 16 + b * L * 4 + b * (1 + 64 + 64 * 64) * 4 + 320 * 128 * 16 * 4 + 160 * 4
    assert everything + extra <= F.ls_state_bytes(c) < everything + extra + 11 * 256
    assert F.ls_view_state_bytes(c, 8) == 0 and F.ls_view_state_bytes(_cfg(batch=0), 1) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), F.LS_ERR_INVALID_ARG),
    (dict(n_q_heads=30), F.LS_ERR_SHAPE),
    (dict(window=16), F.LS_ERR_SHAPE),             # W < B + 1
    (dict(scales=[64, 64, 4096]), F.LS_ERR_SHAPE),  # not ascending
    (dict(scales=[16, 512, 4096]), F.LS_ERR_UNSUPPORTED),  # smallest scale < B + 1
    (dict(scales=[64, 500, 4096]), F.LS_ERR_UNSUPPORTED),  # does not divide the next
    (dict(head_dim=96), F.LS_ERR_UNSUPPORTED),
    (dict(dtype=7), F.LS_ERR_INVALID_ARG),
    (dict(n_kv_heads=16, n_q_heads=64), F.LS_ERR_UNSUPPORTED),
    (dict(block=33, window=64), F.LS_ERR_UNSUPPORTED),        # more drafts than two ballots
    (dict(hidden=4100), F.LS_ERR_UNSUPPORTED),                # hidden not whole 16-byte pieces
    (dict(slots_per_scale=0), F.LS_ERR_INVALID_ARG),
    (dict(flags=0x100), F.LS_ERR_INVALID_ARG),                # unknown flag bit
])
def test_config_validation(kw, status):
    c = _cfg(**kw)
    assert F.ls_state_bytes(c) == 0
    with pytest.raises(F.LsError) as e:
        F.ls_get_layout(c)
    assert e.value.status == status


def test_init_rejects_null_and_misaligned_arena():
    c = _cfg(batch=1)
    with pytest.raises(F.LsError) as e:
        F.ls_init_state(c, None, 1 << 30, 0)
    assert e.value.status == F.LS_ERR_INVALID_ARG
    with pytest.raises(F.LsError) as e:
        F.ls_init_state(c, 0x1000 + 8, 1 << 30, 0)
    assert e.value.status == F.LS_ERR_INVALID_ARG
    with pytest.raises(F.LsError) as e:
        F.ls_init_state(c, 0x10000, 16, 0)
    assert e.value.status == F.LS_ERR_SHAPE


def test_prefill_workspace_bytes():
    c = _cfg()
    # one fp32 sum per (sequence, layer, 512-row unit, K/V column)
    assert F.ls_prefill_workspace_bytes(c, 0, 65536) >= 16 * 4 * 128 * 2 * 8 * 128 * 4
    assert F.ls_prefill_workspace_bytes(c, 10, 5) == 0


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert F.ls_status_string(s) != "unknown status"


def test_make_paged_kv_descriptor():
    """The binding's paged-cache descriptor: per-layer bases in order, the rest of the
    fields as given; more layers than LS_MAX_PAGED_LAYERS, or unequal key/value lists, are
    refused before any call."""
    kv = F.make_paged_kv([0x1000, 0x2000], [0x3000, 0x4000], 4096, 256, 0x5000, 7, 16, 99, verify_slots=0x6000)
    assert list(kv.k_layers[:2]) == [0x1000, 0x2000] and list(kv.v_layers[:2]) == [0x3000, 0x4000]
    assert kv.k_layers[2] is None and kv.v_layers[2] is None
    assert (kv.page_stride, kv.slot_stride, kv.block_table) == (4096, 256, 0x5000)
    assert (kv.max_blocks, kv.page_size, kv.num_pages, kv.verify_slots) == (7, 16, 99, 0x6000)
    assert F.make_paged_kv([0x1000], [0x2000], 256, 256, 0x5000, 1, 1, 1).verify_slots is None
    with pytest.raises(ValueError):
        F.make_paged_kv([0x10] * (F.LS_MAX_PAGED_LAYERS + 1), [0x10] * (F.LS_MAX_PAGED_LAYERS + 1), 0, 256, 1, 1, 1, 1)
    with pytest.raises(ValueError):
        F.make_paged_kv([0x10, 0x20], [0x10], 0, 256, 1, 1, 1, 1)


def test_binding_constants_match_the_header():
    """Every LS_* integer constant the binding defines has the header's value."""
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "include", "longspark.h")) as f:
        text = f.read()
    found = 0
    for name, val in re.findall(r"^#define\s+(LS_[A-Z0-9_]+)\s+\(?(-?(?:0x[0-9a-fA-F]+|\d+))\)?", text, re.M):
        if hasattr(F, name):
            assert getattr(F, name) == int(val, 0), name
            found += 1
    assert found >= 20 and F.LS_ATTEND_INPUTS_READY == 0x100
