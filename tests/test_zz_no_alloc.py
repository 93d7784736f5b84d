"""The prefill entry point for callers that cannot allocate device memory.

Some callers cannot allocate GPU memory when they prefill: an inference engine that keeps
nearly all of the device's memory in a pool it reserved at start-up, or a C program that
links only this library and has no device allocator. ``ls_prefill_summary_noalloc`` runs
the same prefill as ``ls_prefill_summary`` but keeps its scratch in a fixed 16 MiB array
inside the library instead of a caller workspace.

Through the C ABI, two calls in a row (two prefix chunks) must leave exactly the state
the regular entry point leaves: both run the same kernels in the same order on the same
inputs, so every byte of the arena (counters, ring window, boundary, summary sums and
means) is compared bit for bit. After the second call, sampled tiles are checked against
the CPU oracle's views of the same prefix as well. A chunk that needs more scratch than
the array holds is refused with LS_ERR_SCRATCH_LIMIT.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


def _chunk(run, rb, re_):
    """Device prefix rows [rb, re_) of every sequence, as the regular prefill reads them."""
    import synth as S
    wl = run.wl
    rowel = wl.n_kv_heads * wl.head_dim
    n = re_ - rb
    k = torch.empty((wl.batch, wl.n_layers, n, rowel), dtype=run.tdtype, device=run.dev)
    v = torch.empty_like(k)
    run._fill(k, S.PREFIX_K, (1, wl.batch, wl.n_layers, n, rowel), wl.head_dim, p0=rb, scaled=True)
    run._fill(v, S.PREFIX_V, (1, wl.batch, wl.n_layers, n, rowel), wl.head_dim, p0=rb, scaled=True)
    return k, v, n * rowel, rowel


def _same_state(sa, sb):
    for key in sa:
        assert np.array_equal(sa[key], sb[key]), key


def _two_chunk_case(wl, cut):
    regular = WL.DeviceRun(wl, rounds=1)
    noalloc = WL.DeviceRun(wl, rounds=1)
    P = regular.prefix_len
    plen = torch.from_numpy(P).to(regular.dev)
    pmax = int(P.max())
    last_hidden = torch.empty((wl.batch, wl.n_layers, wl.hidden), dtype=regular.tdtype, device=regular.dev)
    import synth as S
    regular._fill(last_hidden, S.LAST_HIDDEN, (1, wl.batch, wl.n_layers, 1, wl.hidden), 0)
    for rb, re_ in ((0, cut), (cut, pmax)):  # two calls in a row
        k, v, plane, rowel = _chunk(regular, rb, re_)
        lh = last_hidden if re_ == pmax else None
        wsb = F.ls_prefill_workspace_bytes(regular.cfg, rb, re_)
        ws = torch.empty(wsb, dtype=torch.uint8, device=regular.dev)
        F.ls_prefill_summary(regular.state, k, v, plane, rowel, plen, rb, re_, lh, ws, wsb, regular.stream)
        F.ls_prefill_summary_noalloc(noalloc.state, k, v, plane, rowel, plen, rb, re_, lh, noalloc.stream)
        torch.cuda.synchronize()
        _same_state(regular.read_state(), noalloc.read_state())
        assert regular.error() == (F.LS_OK, 0) and noalloc.error() == (F.LS_OK, 0)
    # the finished prefill against the oracle's views of the same rows (first and last tile)
    from tests import oracle_side as OS
    st = noalloc.read_state()
    for b, l, h in ((0, 0, 0), (wl.batch - 1, wl.n_layers - 1, wl.n_kv_heads - 1)):
        _, views = OS.tile_views(wl, b, l, h, int(P[b]), [], noalloc.scale_host)
        OS.check_tile_state(wl, st, b, l, h, views)
        assert np.array_equal(st["boundary"][b, l], OS.boundary_hidden(wl, b, l, -1, 0))


def test_noalloc_prefill_matches_regular_ragged():
    wl = WL.Workload("noalloc_mid", 5, 3, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16", (300, 1400),
                     1, None, 1000, head_scale=True)
    _two_chunk_case(wl, 768)


def test_noalloc_prefill_matches_regular_qwen3_8b_shapes():
    from dataclasses import replace
    wl = replace(WL.CONFIGS["qwen3_8b_64k"], prefix=8192, rounds=1)
    _two_chunk_case(wl, 4096)


def test_noalloc_rejects_chunks_beyond_its_scratch():
    wl = WL.CONFIGS["qwen3_8b_64k"]
    run = WL.DeviceRun(wl, rounds=1)
    assert F.ls_prefill_workspace_bytes(run.cfg, 0, 65536) > (16 << 20)
    plen = torch.full((wl.batch,), 65536, dtype=torch.int64, device=run.dev)
    dummy = torch.empty(256, dtype=torch.uint8, device=run.dev)
    with pytest.raises(F.LsError) as e:
        F.ls_prefill_summary_noalloc(run.state, dummy, dummy, 65536 * 1024, 1024, plen, 0, 65536, None)
    assert e.value.status == F.LS_ERR_SCRATCH_LIMIT
    assert "16 MiB" in F.ls_status_string(F.LS_ERR_SCRATCH_LIMIT)
