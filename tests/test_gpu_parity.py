"""Parity of the CUDA path with the oracle at sizes the oracle finishes in seconds.

Integers (accept length, next token, len, per-scale segment counts, ring contents and
mean-row roundings) are compared bit for bit; summary means within 1e-3 normwise
relative error per slot vector; attention outputs within 1e-2 max absolute error.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
import synth as S  # noqa: E402
from tests import oracle_side as OS  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


MID = dict(seed=5, batch=3, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128, hidden=512, block=16,
           window=128, scales=(32, 64, 256), slots=4, dtype="bf16", prefix=(300, 1400), rounds=40,
           accept_mean=None, vocab=1000, head_scale=True)


def _mid(**kw):
    return WL.Workload(name="mid", **{**MID, **kw})


def _out_tile(out, wl, b, l, g):
    """GPU output [B][grp][D] of tile (b, l, g) from out [b][L][B][Hq*D]."""
    o = out[b, l].view(wl.block, wl.n_q_heads, wl.head_dim)[:, g * wl.group:(g + 1) * wl.group]
    return o.float().cpu().numpy().astype(np.float64)


def _check_run_against_oracle(run, wl, rounds_done, out, r_last, tiles=None, view_set=None):
    """Every (or the given) tile's state and attention output vs oracle recompute
    (attention over the views in view_set, all views when None)."""
    st = run.read_state()
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    acc = (OS.accepts_from_ids(draft[:rounds_done], target[:rounds_done]) if rounds_done
           else np.zeros((0, wl.batch), dtype=np.int64))
    tiles = tiles or [(b, l, h) for b in range(wl.batch) for l in range(wl.n_layers)
                      for h in range(wl.n_kv_heads)]
    for b, l, h in tiles:
        P = int(run.prefix_len[b])
        sh, views = OS.tile_views(wl, b, l, h, P, acc[:, b], run.scale_host)
        OS.check_tile_state(wl, st, b, l, h, views)
        hid = OS.boundary_hidden(wl, b, l, rounds_done - 1, int(acc[rounds_done - 1, b]) if rounds_done else 0)
        assert np.array_equal(st["boundary"][b, l], hid), ("boundary", b, l)
        if out is not None:
            ref = OS.tile_attend(wl, sh, views, b, l, h, r_last, hid,
                                 O.VIEW_ALL if view_set is None else view_set)
            got = _out_tile(out, wl, b, l, h)
            exc = OS.attend_error_excess(got, ref)
            assert exc <= 0, ("attend", b, l, h, float(np.abs(got - ref).max()), exc)
    return acc


def test_tiny_round_by_round():
    """Config 1 (fp32): every round against the incremental oracle (Figure 3's form)."""
    wl = WL.CONFIGS["tiny"]
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    sh = O.Shapes(n_layers=wl.n_layers, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads,
                  head_dim=wl.head_dim, hidden=wl.hidden, block=wl.block, window=wl.window,
                  scales=tuple(wl.scales), slots=wl.slots)
    L, H, D, P = wl.n_layers, wl.n_kv_heads, wl.head_dim, int(run.prefix_len[0])
    pk = S.fill_normal(wl.seed, S.PREFIX_K, (1, 1, L, P, H * D), head_dim=D, dtype="f32")[0, 0]
    pv = S.fill_normal(wl.seed, S.PREFIX_V, (1, 1, L, P, H * D), head_dim=D, dtype="f32")[0, 0]
    hid = S.fill_normal(wl.seed, S.LAST_HIDDEN, (1, 1, L, 1, wl.hidden), dtype="f32")[0, 0, :, 0]
    views = O.prefill(sh, O.to_f64(pk, "f32").reshape(L, P, H, D), O.to_f64(pv, "f32").reshape(L, P, H, D), P,
                      O.to_f64(hid, "f32"))
    st = run.read_state()
    for l in range(L):
        for h in range(H):
            OS.check_tile_state(wl, st, 0, l, h, OS.slice_views(views, l, h))
    out = run.new_out()
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    vk_all, vv_all, vh_all, q_all = (inp[k].cpu().numpy() for k in ("vk", "vv", "vh", "q"))
    for r in range(wl.rounds):
        run.commit(inp, r)
        run.attend(inp, r, out)
        torch.cuda.synchronize()
        a, nxt = O.commit_round(sh, views, draft[r, 0], target[r, 0],
                                O.to_f64(vk_all[r, 0], "f32").reshape(L, wl.block + 1, H, D),
                                O.to_f64(vv_all[r, 0], "f32").reshape(L, wl.block + 1, H, D),
                                O.to_f64(vh_all[r, 0], "f32"))
        assert int(run.accept_len[0]) == a and int(run.next_token[0]) == nxt
        st = run.read_state()
        for l in range(L):
            for h in range(H):
                OS.check_tile_state(wl, st, 0, l, h, OS.slice_views(views, l, h))
        assert np.array_equal(st["boundary"][0], O.to_f64(vh_all[r, 0, :, a], "f32"))
        bk = views.boundary[:, :H * D].reshape(L, H, D)
        bv = views.boundary[:, H * D:2 * H * D].reshape(L, H, D)
        ref = O.draft_attend(sh, views, O.to_f64(q_all[r, 0], "f32").reshape(L, wl.block, wl.n_q_heads, D),
                             bk, bv, 1.0 / np.sqrt(D))
        got = out[0].view(L, wl.block, wl.n_q_heads, D).double().cpu().numpy()
        assert OS.attend_error_excess(got, ref) <= 0
    assert run.error() == (F.LS_OK, 0)


@pytest.mark.parametrize("force_simt,out_f32", [(False, True), (False, False), (True, True), (True, False)],
                         ids=["tensor_cores_f32out", "tensor_cores_bf16out", "cuda_cores_f32out",
                              "cuda_cores_bf16out"])
def test_mid_ragged_all_tiles(force_simt, out_f32):
    """Ragged prefixes, several tiles; bf16; GQA group 4 x B 16 = a 64-row tile."""
    wl = _mid(flags=(F.LS_FLAG_FORCE_SIMT if force_simt else 0) | (F.LS_FLAG_OUT_F32 if out_f32 else 0))
    run = WL.DeviceRun(wl)
    assert F.ls_attend_uses_tensor_cores(run.state) == (not force_simt)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    _check_run_against_oracle(run, wl, 0, None, -1)
    for r in range(wl.rounds):
        run.commit(inp, r)
        run.attend(inp, r, out)
        if r in (0, 7, wl.rounds - 1):
            torch.cuda.synchronize()
            _check_run_against_oracle(run, wl, r + 1, out, r)
    assert run.error() == (F.LS_OK, 0)


VIEW_SETS = list(range(1, 8))


@pytest.mark.parametrize("force_simt", [False, True], ids=["tensor_cores", "cuda_cores"])
@pytest.mark.parametrize("view_set", VIEW_SETS, ids=[f"views{v}" for v in VIEW_SETS])
def test_view_ablations(force_simt, view_set):
    """ls_draft_attend_views (Table 5's component ablations) on every non-empty subset of the
    views. W = 128 and R = 144: without the window the kernel skips the ring chunk, without
    the summary it loads none of the last chunk's arena rows."""
    wl = _mid(rounds=3, flags=F.LS_FLAG_FORCE_SIMT if force_simt else 0)
    run = WL.DeviceRun(wl)
    assert F.ls_attend_uses_tensor_cores(run.state) == (not force_simt)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    for r in range(wl.rounds):
        run.commit(inp, r)
    out.fill_(float("nan"))
    run.attend(inp, wl.rounds - 1, out, views=view_set)
    torch.cuda.synchronize()
    _check_run_against_oracle(run, wl, wl.rounds, out, wl.rounds - 1, view_set=view_set)
    assert run.error() == (F.LS_OK, 0)


@pytest.mark.parametrize("force_simt", [False, True], ids=["tensor_cores", "cuda_cores"])
def test_view_ablations_empty_state(force_simt):
    """Before any row is retained the window and the summary have no valid row: zeros."""
    wl = _mid(rounds=1, flags=F.LS_FLAG_FORCE_SIMT if force_simt else 0)
    run = WL.DeviceRun(wl)  # initialised, never prefilled: len = 0
    inp = run.make_round_inputs()
    out = run.new_out()
    for view_set in (F.LS_VIEW_WINDOW, F.LS_VIEW_SUMMARY, F.LS_VIEW_WINDOW | F.LS_VIEW_SUMMARY):
        out.fill_(float("nan"))
        run.attend(inp, 0, out, views=view_set)
        torch.cuda.synchronize()
        assert not out.float().abs().sum().item() and not torch.isnan(out.float()).any().item(), view_set
    with pytest.raises(F.LsError):
        run.attend(inp, 0, out, views=0)
    with pytest.raises(F.LsError):
        run.attend(inp, 0, out, views=8)
    assert run.error() == (F.LS_OK, 0)


def test_paths_agree():
    """Tensor-core and CUDA-core attention on the same state agree within tolerance."""
    wl = _mid(rounds=5, flags=F.LS_FLAG_OUT_F32)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(wl.rounds):
        run.commit(inp, r)
    out_a = run.new_out()
    run.attend(inp, wl.rounds - 1, out_a)
    wl2 = _mid(rounds=5, flags=F.LS_FLAG_FORCE_SIMT | F.LS_FLAG_OUT_F32)
    run2 = WL.DeviceRun(wl2)
    run2.prefill()
    inp2 = run2.make_round_inputs()
    for r in range(wl.rounds):
        run2.commit(inp2, r)
    out_b = run2.new_out()
    run2.attend(inp2, wl.rounds - 1, out_b)
    torch.cuda.synchronize()
    assert (out_a.float() - out_b.float()).abs().max().item() <= OS.ATTEND_ATOL


def test_per_layer_calls_match_one_call():
    wl = _mid(rounds=3)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(3):
        run.commit(inp, r)
    full = run.new_out()
    run.attend(inp, 2, full)
    for l in range(wl.n_layers):
        one = run.new_out(1)
        run.attend(inp, 2, one, layer_begin=l, layer_count=1)
        torch.cuda.synchronize()
        assert torch.equal(one[:, 0], full[:, l])


def test_per_layer_calls_back_to_back_match_one_call():
    """Per-layer calls issued back to back, with no synchronisation: nothing writes the
    views between them, so each launch loads its first K/V chunks before the launch ahead
    of it has completed. They give the bits of one call over all layers."""
    wl = _mid(rounds=3)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(3):
        run.commit(inp, r)
    full = run.new_out()
    run.attend(inp, 2, full)
    torch.cuda.synchronize()
    ones = [run.new_out(1) for _ in range(wl.n_layers)]
    for rep in range(2):
        for l in range(wl.n_layers):
            ones[l].fill_(float("nan"))
        for l in range(wl.n_layers):
            run.attend(inp, 2, ones[l], layer_begin=l, layer_count=1)
        torch.cuda.synchronize()
        for l in range(wl.n_layers):
            assert torch.equal(ones[l][:, 0], full[:, l]), (rep, l)
    assert run.error() == (F.LS_OK, 0)


def test_per_layer_calls_with_inputs_ready_hint():
    """LS_ATTEND_INPUTS_READY (every layer's queries computed before the calls): the first
    per-layer call right after a commit reads its queries before the commit has completed
    (the views only after), the next ones do not wait for the call before them at all.
    Same bits as one call over all layers on a twin state; repeated back to back."""
    wl = _mid(rounds=3)
    runs = [WL.DeviceRun(wl), WL.DeviceRun(wl)]
    for run in runs:
        run.prefill()
    inp = runs[0].make_round_inputs()
    for run in runs:
        for r in range(3):
            run.commit(inp, r)
    full = runs[1].new_out()
    runs[1].attend(inp, 2, full)
    a = runs[0]
    a.commit(inp, 2)  # (both states get a third commit of the same round: still equal)
    runs[1].commit(inp, 2)
    runs[1].attend(inp, 2, full)
    torch.cuda.synchronize()
    qs = [inp["q"][2][:, l:l + 1].contiguous() for l in range(wl.n_layers)]
    ones = [a.new_out(1) for _ in range(wl.n_layers)]
    hint = F.LS_VIEW_ALL | F.LS_ATTEND_INPUTS_READY
    for rep in range(3):
        for o in ones:
            o.fill_(float("nan"))
        if rep == 2:
            a.commit(inp, 2)
            runs[1].commit(inp, 2)
            runs[1].attend(inp, 2, full)
        for l in range(wl.n_layers):
            F.ls_draft_attend_views(a.state, l, 1, qs[l], a.boundary_k, a.boundary_v, wl.hidden, a.softmax_scale,
                                    hint, ones[l], a.stream)
        torch.cuda.synchronize()
        for l in range(wl.n_layers):
            assert torch.equal(ones[l][:, 0], full[:, l]), (rep, l)
    assert a.error() == (F.LS_OK, 0) and runs[1].error() == (F.LS_OK, 0)
    with pytest.raises(F.LsError):  # the hint alone names no view
        F.ls_draft_attend_views(a.state, 0, 1, qs[0], a.boundary_k, a.boundary_v, wl.hidden, a.softmax_scale,
                                F.LS_ATTEND_INPUTS_READY, ones[0], a.stream)


def test_inputs_ready_hint_on_the_cuda_core_path():
    """The tiny fp32 config (CUDA-core attention, which launches no programmatic
    dependents): per-layer calls with LS_ATTEND_INPUTS_READY equal one call bit for bit."""
    wl = WL.CONFIGS["tiny"]
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(3):
        run.commit(inp, r)
    assert not F.ls_attend_uses_tensor_cores(run.state)
    full = run.new_out()
    run.attend(inp, 2, full)
    ones = [run.new_out(1) for _ in range(wl.n_layers)]
    for l in range(wl.n_layers):
        F.ls_draft_attend_views(run.state, l, 1, inp["q"][2][:, l:l + 1].contiguous(), run.boundary_k,
                                run.boundary_v, wl.hidden, run.softmax_scale,
                                F.LS_VIEW_ALL | F.LS_ATTEND_INPUTS_READY, ones[l], run.stream)
    torch.cuda.synchronize()
    for l in range(wl.n_layers):
        assert torch.equal(ones[l][:, 0], full[:, l])
    assert run.error() == (F.LS_OK, 0)


def test_attention_reads_the_previous_attentions_output():
    """Two attentions back to back, the second taking the first's output as its queries:
    the second launch may start before the first completes (its early loads are of the
    unchanged views only), but its queries are read after the first has completed. Same
    bits as the two calls with a synchronisation between them. Against the oracle with
    those queries through a state with fp32 outputs: these queries concentrate the softmax
    enough for outputs above 4, where a bf16 output's own rounding (up to 2^-5 / 2) would
    exceed the 1e-2 bound by itself."""
    wl = _mid(rounds=2)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(2):
        run.commit(inp, r)
    q = inp["q"][1]
    L, H, D = wl.n_layers, wl.n_kv_heads, wl.head_dim
    args = (run.boundary_k, run.boundary_v, wl.hidden, run.softmax_scale)
    o1, o2 = run.new_out(), run.new_out()
    F.ls_draft_attend(run.state, 0, L, q, *args, o1, run.stream)
    F.ls_draft_attend(run.state, 0, L, o1, *args, o2, run.stream)
    torch.cuda.synchronize()
    r1, r2 = run.new_out(), run.new_out()
    F.ls_draft_attend(run.state, 0, L, q, *args, r1, run.stream)
    torch.cuda.synchronize()
    q2 = r1.clone()
    torch.cuda.synchronize()
    F.ls_draft_attend(run.state, 0, L, q2, *args, r2, run.stream)
    torch.cuda.synchronize()
    assert torch.equal(o1, r1) and torch.equal(o2, r2)
    wl32 = _mid(rounds=2, flags=F.LS_FLAG_OUT_F32)
    run32 = WL.DeviceRun(wl32)
    run32.prefill()
    for r in range(2):
        run32.commit(inp, r)
    o32 = run32.new_out()
    F.ls_draft_attend(run32.state, 0, L, q2, run32.boundary_k, run32.boundary_v, wl.hidden, run32.softmax_scale,
                      o32, run32.stream)
    torch.cuda.synchronize()
    st = run.read_state()
    assert all(np.array_equal(st[k], v) for k, v in run32.read_state().items())
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    acc = OS.accepts_from_ids(draft[:2], target[:2])
    q2h = O.to_f64(q2.view(torch.int16).cpu().numpy().view(np.uint16), "bf16")
    for b, l, g in [(b, l, g) for b in range(wl.batch) for l in range(L) for g in range(H)]:
        sh, views = OS.tile_views(wl, b, l, g, int(run.prefix_len[b]), acc[:, b], run.scale_host)
        hv = O.to_f64(st["boundary"][b, l], "bf16")
        bk = hv[g * D:(g + 1) * D].reshape(1, 1, D)
        bv = hv[H * D + g * D:H * D + (g + 1) * D].reshape(1, 1, D)
        qt = q2h[b, l].reshape(wl.block, wl.n_q_heads, D)[:, g * wl.group:(g + 1) * wl.group][None]
        ref = O.draft_attend(sh, views, qt, bk, bv, 1.0 / np.sqrt(D))[0]
        assert OS.attend_error_excess(_out_tile(o32, wl, b, l, g), ref) <= 0
    assert run.error() == (F.LS_OK, 0) and run32.error() == (F.LS_OK, 0)


def test_chunked_prefill_matches_oracle():
    wl = _mid(rounds=6, prefix=(700, 1337), flags=F.LS_FLAG_OUT_F32)
    run = WL.DeviceRun(wl, prefill_chunk=256)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    for r in range(wl.rounds):
        run.commit(inp, r)
        run.attend(inp, r, out)
    torch.cuda.synchronize()
    _check_run_against_oracle(run, wl, wl.rounds, out, wl.rounds - 1)
    assert run.error() == (F.LS_OK, 0)


@pytest.mark.parametrize("prefix,accepts", [
    (0, None),                 # empty prefix: every view starts empty
    (5, None),                 # prefix shorter than the window and every scale
    (512, None),               # prefix a multiple of every scale: all partials empty
    (256 - 3, 16),             # one round crosses the 32-, 64- and 256-row boundaries at once
    (1000, 0),                 # a = 0 every round: Delta = 1
    (1000, 16),                # a = B every round: Delta = B + 1
], ids=["empty", "short", "aligned", "multi_crossing", "a0", "aB"])
def test_edge_cases(prefix, accepts):
    wl = _mid(rounds=12, prefix=prefix, flags=F.LS_FLAG_OUT_F32)
    run = WL.DeviceRun(wl, accepts_override=None if accepts is None else [accepts] * 12)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    for r in range(wl.rounds):
        run.commit(inp, r)
        run.attend(inp, r, out)
        if r in (0, wl.rounds - 1):
            torch.cuda.synchronize()
            _check_run_against_oracle(run, wl, r + 1, out, r)
    assert run.error() == (F.LS_OK, 0)


def test_large_logit_spread_takes_rescale_path():
    """Queries x16: later chunks raise rows' max by more than 2^8, so the tensor-core
    kernel must rescale its running output and sum; the result still matches the oracle."""
    wl = WL.Workload("spread", 7, 2, 1, 2, 8, 128, 512, 16, 512, (64, 512, 4096), 32, "bf16", (5000, 9000), 3,
                     None, 1000, head_scale=True, flags=F.LS_FLAG_OUT_F32)
    run = WL.DeviceRun(wl)
    assert F.ls_attend_uses_tensor_cores(run.state)
    run.prefill()
    inp = run.make_round_inputs()
    inp["q"].mul_(16.0)  # exact in bf16 (power of two)
    out = run.new_out()
    for r in range(wl.rounds):
        run.commit(inp, r)
    run.attend(inp, wl.rounds - 1, out)
    torch.cuda.synchronize()
    st = run.read_state()
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    acc = OS.accepts_from_ids(draft, target)
    jumped = 0
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            sh, views = OS.tile_views(wl, b, 0, h, int(run.prefix_len[b]), acc[:, b], run.scale_host)
            OS.check_tile_state(wl, st, b, 0, h, views)
            hid = OS.boundary_hidden(wl, b, 0, wl.rounds - 1, int(acc[-1, b]))
            hv = O.to_f64(hid, wl.dtype)
            bk = hv[h * 128:(h + 1) * 128].reshape(1, 1, 128)
            bv = hv[wl.n_kv_heads * 128 + h * 128:wl.n_kv_heads * 128 + (h + 1) * 128].reshape(1, 1, 128)
            q = OS.queries(wl, wl.rounds - 1, b, 0, h) * 16.0
            ref = O.draft_attend(sh, views, q, bk, bv, 1.0 / np.sqrt(128))[0]
            got = _out_tile(out, wl, b, 0, h)
            assert OS.attend_error_excess(got, ref) <= 0, float(np.abs(got - ref).max())
            # the kernel's chunks are the tile's arena rows in blocks of 128: boundary and
            # chunk 0 set the first reference, later chunks exceed it by > 8 log2 units?
            K, _, ok = O.attention_slots(sh, views, 0, 0, bk, bv)
            lg = (q[0].reshape(-1, 128) @ K.T) / np.sqrt(128) / np.log(2.0)
            lg[:, ~ok] = -np.inf
            first = np.maximum(lg[:, 0], lg[:, 1:129].max(axis=1))
            later = lg[:, 129:].max(axis=1)
            jumped += int(np.sum(later > first + 8.0))
    assert jumped > 0, "inputs never exercise the rescale path"
