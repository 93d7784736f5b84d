"""Parity at the full workload sizes, on sampled tiles the oracle computes one by one.

Each run uses the same launch sequence the bench times (one ls_commit_round and one
ls_draft_attend over all tapped layers per round, batch 16). The sampled tiles cover
first/last sequences, layers and KV heads; the oracle rebuilds their whole K/V cache
(prefix + retained verify rows) from the generator and recomputes the views by their
definition. Properties that hold at any size are checked on every tile.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from tests import oracle_side as OS  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


EARLY_ROUND = 3  # an early round whose attention output is kept and checked as well


def _run_full(wl, rounds=None, prefill_chunk=None):
    """Prefill, then every round's commit and attention; returns the run, the last round's
    output and a copy of round EARLY_ROUND's output."""
    run = WL.DeviceRun(wl, rounds=rounds, prefill_chunk=prefill_chunk)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    early = None
    for r in range(run.rounds):
        run.commit(inp, r)
        run.attend(inp, r, out)
        if r == EARLY_ROUND:
            early = out.clone()
    torch.cuda.synchronize()
    return run, out, early


def _check_attend_at(run, wl, out, tiles, r, acc, view_set=None):
    """Attention output of round r on the sampled tiles against the oracle's attention over
    the views as they stood after round r's commit."""
    P = run.prefix_len
    for b, l, h in tiles:
        sh, views = OS.tile_views(wl, b, l, h, int(P[b]), acc[:r + 1, b], run.scale_host)
        hid = OS.boundary_hidden(wl, b, l, r, int(acc[r, b]))
        ref = OS.tile_attend(wl, sh, views, b, l, h, r, hid, OS.O.VIEW_ALL if view_set is None else view_set)
        o = out[b, l].view(wl.block, wl.n_q_heads, wl.head_dim)[:, h * wl.group:(h + 1) * wl.group]
        got = o.float().cpu().numpy().astype(np.float64)
        exc = OS.attend_error_excess(got, ref)
        assert exc <= 0, ("attend", r, b, l, h, float(np.abs(got - ref).max()), exc)


def _sampled_check(run, wl, out, tiles, view_set=None, early=None):
    st = run.read_state()
    R = run.rounds
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    acc = OS.accepts_from_ids(draft, target)
    if early is not None:
        _check_attend_at(run, wl, early, tiles, EARLY_ROUND, acc, view_set)
    assert np.array_equal(acc, run.accept_host), "generator accepts vs oracle scan"
    # any-size properties on every tile: len and counters consistent, all layers equal
    P = run.prefix_len
    want_len = P + (acc + 1).sum(axis=0)
    assert np.array_equal(st["counters"][:, :, 0], np.repeat(want_len[:, None], wl.n_layers, 1))
    for k, s in enumerate(wl.scales):
        assert np.array_equal(st["counters"][:, :, 1 + k], st["counters"][:, :, 0] // s)
    assert np.all(np.isfinite(out.float().cpu().numpy()))
    for b, l, h in tiles:
        sh, views = OS.tile_views(wl, b, l, h, int(P[b]), acc[:, b], run.scale_host)
        OS.check_tile_state(wl, st, b, l, h, views)
        hid = OS.boundary_hidden(wl, b, l, R - 1, int(acc[R - 1, b]))
        assert np.array_equal(st["boundary"][b, l], hid)
        ref = OS.tile_attend(wl, sh, views, b, l, h, R - 1, hid,
                             OS.O.VIEW_ALL if view_set is None else view_set)
        o = out[b, l].view(wl.block, wl.n_q_heads, wl.head_dim)[:, h * wl.group:(h + 1) * wl.group]
        got = o.float().cpu().numpy().astype(np.float64)
        exc = OS.attend_error_excess(got, ref)
        assert exc <= 0, ("attend", b, l, h, float(np.abs(got - ref).max()), exc)


# At batch 16 the attention runs 512 tiles t = (b L + l) Hkv + h on 128 CTAs, tiles
# c, c + 128, c + 256, c + 384 on CTA c: these tiles (t = 0, 245, 331, 511) sit in each of
# the four places of a CTA's schedule.
TILES = [(0, 0, 0), (7, 2, 5), (10, 1, 3), (15, 3, 7)]


@pytest.mark.parametrize("name", ["qwen3_4b_32k", "qwen3_8b_64k", "qwen3_8b_64k_f32out", "qwen3_8b_128k_ragged"])
def test_full_config(name):
    from dataclasses import replace
    wl = (replace(WL.CONFIGS["qwen3_8b_64k"], flags=F.LS_FLAG_OUT_F32) if name.endswith("_f32out")
          else WL.CONFIGS[name])
    run, out, early = _run_full(wl)
    assert run.error() == (F.LS_OK, 0)
    _sampled_check(run, wl, out, TILES, early=early)


def test_full_config_view_ablations():
    """Table 5's three ablations at the bench workload (4 tiles per CTA, W = 512: the four
    ring chunks skipped without the window, the 100 summary rows not loaded without the
    summary), on the sampled tiles."""
    wl = WL.CONFIGS["qwen3_8b_64k"]
    run, out, _ = _run_full(wl)
    inp = run.make_round_inputs(run.rounds - 1, 1)
    for view_set in (F.LS_VIEW_WINDOW | F.LS_VIEW_BOUNDARY, F.LS_VIEW_WINDOW | F.LS_VIEW_SUMMARY,
                     F.LS_VIEW_SUMMARY | F.LS_VIEW_BOUNDARY):
        out.fill_(float("nan"))
        run.attend(inp, run.rounds - 1, out, views=view_set)
        torch.cuda.synchronize()
        assert run.error() == (F.LS_OK, 0)
        _sampled_check(run, wl, out, TILES, view_set)


def test_full_config_per_layer_calls():
    """The bench workload's attention as per-layer calls (128 tiles each), with and without
    LS_ATTEND_INPUTS_READY (with it, each call runs on half of the SMs, two tiles per CTA,
    beside the next call), back to back: the bits of one call over the four layers."""
    wl = WL.CONFIGS["qwen3_8b_64k"]
    run, out, _ = _run_full(wl, rounds=8)
    inp = run.make_round_inputs(run.rounds - 1, 1)
    r = run.rounds - 1
    qs = [inp["q"][0][:, l:l + 1].contiguous() for l in range(wl.n_layers)]
    for views in (F.LS_VIEW_ALL | F.LS_ATTEND_INPUTS_READY, F.LS_VIEW_ALL):
        ones = [run.new_out(1).fill_(float("nan")) for _ in range(wl.n_layers)]
        for rep in range(2):
            for l in range(wl.n_layers):
                F.ls_draft_attend_views(run.state, l, 1, qs[l], run.boundary_k, run.boundary_v, wl.hidden,
                                        run.softmax_scale, views, ones[l], run.stream)
        torch.cuda.synchronize()
        for l in range(wl.n_layers):
            assert torch.equal(ones[l][:, 0], out[:, l]), (views, l)
    # a view subset with the hint: the same bits as one call over that subset
    sub = F.LS_VIEW_WINDOW | F.LS_VIEW_SUMMARY
    full_sub = run.new_out()
    F.ls_draft_attend_views(run.state, 0, wl.n_layers, inp["q"][0], run.boundary_k, run.boundary_v, wl.hidden,
                            run.softmax_scale, sub, full_sub, run.stream)
    ones = [run.new_out(1).fill_(float("nan")) for _ in range(wl.n_layers)]
    for l in range(wl.n_layers):
        F.ls_draft_attend_views(run.state, l, 1, qs[l], run.boundary_k, run.boundary_v, wl.hidden,
                                run.softmax_scale, sub | F.LS_ATTEND_INPUTS_READY, ones[l], run.stream)
    torch.cuda.synchronize()
    for l in range(wl.n_layers):
        assert torch.equal(ones[l][:, 0], full_sub[:, l]), ("subset", l)
    assert run.error() == (F.LS_OK, 0) and r >= 0


@pytest.mark.parametrize("prefix,batch,mean", [(4096, 1, 2.5), (16384, 4, 4.0), (131072, 64, 6.0)])
def test_sweep_points(prefix, batch, mean):
    wl = WL.sweep_point(prefix, batch, mean)
    chunk = 32768 if prefix * batch > 4 * 1024 * 1024 else None
    run, out, _ = _run_full(wl, prefill_chunk=chunk)
    assert run.error() == (F.LS_OK, 0)
    _sampled_check(run, wl, out, [(0, 0, 0), (batch - 1, 3, 7)])


def test_state_bytes_fixed_across_sweep():
    """Drafter state bytes depend on batch and shapes only, never on the prefix."""
    for batch in WL.SWEEP_BATCHES:
        sizes = {F.ls_state_bytes(WL.sweep_point(p, batch, 4.0).config()) for p in WL.SWEEP_PREFIXES}
        assert len(sizes) == 1


def test_full_config_paged():
    """The bench workload with the prefix and every round's verify rows in a paged cache
    (page size 16, pages scattered over a 70K-page pool, 18 GB): ls_prefill_paged, then
    commits reading the pages in place (block table on even rounds, the engine's slot
    mapping on odd ones) and the attention; sampled tiles against the oracle."""
    wl = WL.CONFIGS["qwen3_8b_64k"]
    run = WL.DeviceRun(wl)
    cache = WL.PagedCache(run, 16, run.prefix_len + (run.rounds + 1) * (wl.block + 1), seed=2)
    run.fill_pages(cache)
    run.prefill_paged(cache)
    inp = run.make_round_inputs()
    for r in range(run.rounds):
        run.write_verify_pages(cache, inp, r)
    out = run.new_out()
    for r in range(run.rounds):
        run.commit_paged(cache, inp, r, with_slots=bool(r & 1))
        run.attend(inp, r, out)
    torch.cuda.synchronize()
    assert run.error() == (F.LS_OK, 0)
    del cache
    torch.cuda.empty_cache()
    _sampled_check(run, wl, out, TILES)
