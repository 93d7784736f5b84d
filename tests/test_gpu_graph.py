"""Calls captured into CUDA graphs and replayed give the bits of the same calls launched
from the stream: ls_round (commit and attention, with the programmatic edge between them
captured), the drafter's per-layer attention with LS_ATTEND_INPUTS_READY, and the drafting
round's four calls (sampled acceptance, commit, projections, attention).

A launch captured into a graph settles nothing for the launches made directly on the
stream afterwards: an attention launched straight after a capture, on a stream whose last
direct launch was a commit, still waits for that commit (with the hint it would otherwise
read the views with no wait at all).
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


def _wl(**kw):
    base = dict(name="graph", seed=23, batch=4, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128, hidden=512,
                block=16, window=128, scales=(32, 64, 256), slots=4, dtype="bf16", prefix=(300, 1400), rounds=4,
                accept_mean=None, vocab=1000, head_scale=True)
    base.update(kw)
    return WL.Workload(**base)


def _state_equal(a, b):
    sa, sb = a.read_state(), b.read_state()
    for k, v in sa.items():
        assert np.array_equal(v, sb[k]), k


def _captured(fn):
    """A graph of fn(stream) captured on a side stream."""
    g = torch.cuda.CUDAGraph()
    gs = torch.cuda.Stream()
    gs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(gs):
        with torch.cuda.graph(g, stream=gs):
            fn(gs)
    torch.cuda.current_stream().wait_stream(gs)
    return g


def test_round_graph_matches_stream_launches():
    """Every round of a run as ls_round launched from the stream, and the same rounds
    captured into one graph and replayed: outputs, accepted counts and the whole state
    bit for bit."""
    wl = _wl()
    ref = WL.DeviceRun(wl)
    ref.prefill()
    inp = ref.make_round_inputs()
    ref_out = [ref.new_out() for _ in range(wl.rounds)]
    ref_acc = []
    for r in range(wl.rounds):
        ref.round(inp, r, ref_out[r])
        ref_acc.append(ref.accept_len.clone())
    torch.cuda.synchronize()

    run = WL.DeviceRun(wl)
    run.prefill()
    inp2 = run.make_round_inputs()
    outs = [run.new_out().fill_(float("nan")) for _ in range(wl.rounds)]
    accs = [torch.full_like(run.accept_len, -1) for _ in range(wl.rounds)]
    torch.cuda.synchronize()
    home = run.stream

    def rounds(s):
        run.stream = s
        for r in range(wl.rounds):
            run.round(inp2, r, outs[r])
            accs[r].copy_(run.accept_len)

    g = _captured(rounds)
    run.stream = home
    g.replay()
    torch.cuda.synchronize()
    for r in range(wl.rounds):
        assert torch.equal(outs[r], ref_out[r]), r
        assert torch.equal(accs[r], ref_acc[r]), r
    _state_equal(run, ref)
    assert run.error() == (F.LS_OK, 0) and ref.error() == (F.LS_OK, 0)
    del g


def test_hinted_per_layer_calls_in_a_graph():
    """A drafter's per-layer attention calls with LS_ATTEND_INPUTS_READY, captured into a
    graph behind the round's commit and replayed twice: the bits of one call over all
    layers launched from the stream."""
    wl = _wl()
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(wl.rounds - 1):
        run.commit(inp, r)
    r = wl.rounds - 1
    H, D = wl.n_kv_heads, wl.head_dim
    qs = [inp["q"][r][:, l:l + 1].contiguous() for l in range(wl.n_layers)]
    # the drafter's boundary keys/values: complete before the commit, as the hint requires
    bkv = (torch.randn((wl.batch, wl.n_layers, 2 * H * D), device=run.dev,
                       generator=torch.Generator(device=run.dev).manual_seed(3)) * 0.5).to(torch.bfloat16)
    ones = [run.new_out(1).fill_(float("nan")) for _ in range(wl.n_layers)]
    torch.cuda.synchronize()
    home = run.stream

    def calls(s):
        run.stream = s
        run.commit(inp, r)
        for l in range(wl.n_layers):
            F.ls_draft_attend_views(run.state, l, 1, qs[l], bkv, bkv[..., H * D:], 2 * H * D,
                                    run.softmax_scale, F.LS_VIEW_ALL | F.LS_ATTEND_INPUTS_READY, ones[l], s)

    def one_call():
        full = run.new_out()
        F.ls_draft_attend(run.state, 0, wl.n_layers, inp["q"][r], bkv, bkv[..., H * D:], 2 * H * D,
                          run.softmax_scale, full, run.stream)
        torch.cuda.synchronize()
        return full

    g = _captured(calls)
    run.stream = home
    g.replay()
    torch.cuda.synchronize()
    full = one_call()
    for l in range(wl.n_layers):
        assert torch.equal(ones[l][:, 0], full[:, l]), l
    # a second replay commits round r again (the views move on): the per-layer calls still
    # match one call over the layers of the state as the replay left it
    for o in ones:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    full = one_call()
    for l in range(wl.n_layers):
        assert torch.equal(ones[l][:, 0], full[:, l]), ("second replay", l)
    assert run.error() == (F.LS_OK, 0)
    del g


def _probs(rng, shape, z=None, noise=0.5):
    x = rng.standard_normal(shape) * 2.0 if z is None else z + noise * rng.standard_normal(shape)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32), x


def test_drafting_round_in_a_graph():
    """The drafting round's four calls (ls_accept_sampled, ls_commit_accepted,
    ls_draft_prologue, ls_draft_attend) for every round, captured into one graph and
    replayed, against the same calls launched from the stream: every output and the state
    bit for bit."""
    wl = _wl(rounds=3, flags=F.LS_FLAG_OUT_F32)
    b, B, V, L, H, Hq, D, hid = (wl.batch, wl.block, 1000, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim,
                                 wl.hidden)
    dev = torch.device("cuda")
    rng = np.random.default_rng(41)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)  # noqa: E731
    rounds = []
    for _ in range(wl.rounds):
        q, zq = _probs(rng, (b, B, V))
        p, _ = _probs(rng, (b, B + 1, V), z=np.concatenate([zq, zq[:, -1:]], axis=1), noise=0.6)
        draft = np.array([[np.searchsorted(np.cumsum(q[i, j], dtype=np.float64), rng.random())
                           for j in range(B)] for i in range(b)]).clip(0, V - 1).astype(np.int32)
        u = rng.random((b, B + 1)).astype(np.float32)
        x = t(rng.standard_normal((b, L, B, hid)).astype(np.float32)).to(torch.bfloat16)
        rounds.append(dict(q=t(q), p=t(p), draft=t(draft), u=t(u), x=x))
    g0 = torch.Generator(device=dev).manual_seed(7)
    w_kv = (torch.randn((L, 2 * H * D, hid), device=dev, generator=g0) * hid ** -0.5).to(torch.bfloat16)
    w_q = (torch.randn((L, Hq * D, hid), device=dev, generator=g0) * hid ** -0.5).to(torch.bfloat16)

    def setup():
        run = WL.DeviceRun(wl)
        run.prefill()
        inp = run.make_round_inputs()
        outs = [dict(acc=torch.full((b,), -1, dtype=torch.int32, device=dev),
                     nxt=torch.full((b,), -1, dtype=torch.int32, device=dev),
                     bkv=torch.full((b, L, 2 * H * D), float("nan"), dtype=torch.bfloat16, device=dev),
                     qd=torch.full((b, L, B, Hq * D), float("nan"), dtype=torch.bfloat16, device=dev),
                     out=run.new_out().fill_(float("nan"))) for _ in range(wl.rounds)]
        torch.cuda.synchronize()
        return run, inp, outs

    def chain(run, inp, outs, s):
        for i, r in enumerate(rounds):
            o = outs[i]
            F.ls_accept_sampled(run.state, r["draft"], r["q"], r["p"], V, r["u"], o["acc"], o["nxt"], s)
            F.ls_commit_accepted(run.state, o["acc"], inp["vk"][i], inp["vv"][i], inp["vh"][i], s)
            F.ls_draft_prologue(run.state, w_kv, w_q, r["x"], o["bkv"], o["qd"], s)
            F.ls_draft_attend(run.state, 0, L, o["qd"], o["bkv"], o["bkv"][..., H * D:], 2 * H * D,
                              run.softmax_scale, o["out"], s)

    ref, ref_inp, ref_outs = setup()
    chain(ref, ref_inp, ref_outs, ref.stream)
    torch.cuda.synchronize()
    run, inp, outs = setup()
    g = _captured(lambda s: chain(run, inp, outs, s))
    g.replay()
    torch.cuda.synchronize()
    for i in range(wl.rounds):
        for k in outs[i]:
            assert torch.equal(outs[i][k], ref_outs[i][k]), (i, k)
    _state_equal(run, ref)
    assert run.error() == (F.LS_OK, 0) and ref.error() == (F.LS_OK, 0)
    del g


def test_capture_settles_nothing_for_later_direct_launches():
    """On a side stream held busy by a 1 GB memset: a commit launched directly, then an
    attention captured into a graph (not replayed), then an attention with
    LS_ATTEND_INPUTS_READY launched directly. The direct attention follows the commit on
    the stream, so it must see the commit's rows: the bits of the same attention launched
    after a synchronisation."""
    wl = _wl()
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    r = 0
    q = inp["q"][r]
    H, D = wl.n_kv_heads, wl.head_dim
    # the drafter's boundary keys/values: complete long before, as the hint requires
    bkv = (torch.randn((wl.batch, wl.n_layers, 2 * H * D), device=run.dev,
                       generator=torch.Generator(device=run.dev).manual_seed(4)) * 0.5).to(torch.bfloat16)
    hint = F.LS_VIEW_ALL | F.LS_ATTEND_INPUTS_READY

    def attend(out, views, s):
        F.ls_draft_attend_views(run.state, 0, wl.n_layers, q, bkv, bkv[..., H * D:], 2 * H * D,
                                run.softmax_scale, views, out, s)

    side = torch.cuda.Stream()
    busy = torch.empty(1 << 30, dtype=torch.uint8, device=run.dev)
    scratch = run.new_out()
    got = run.new_out().fill_(float("nan"))
    # an attention launched directly on the side stream first: the views are then settled
    # there, which is what a capture must not leave behind
    side.wait_stream(torch.cuda.current_stream())
    attend(scratch, F.LS_VIEW_ALL, side)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        busy.fill_(1)  # keeps the GPU busy while the host launches and captures below
        run.stream = side
        run.commit(inp, r)
        g = torch.cuda.CUDAGraph()
        g.capture_begin()
        attend(scratch, hint, side)
        g.capture_end()
        attend(got, hint, side)
    torch.cuda.synchronize()
    want = run.new_out()
    attend(want, F.LS_VIEW_ALL, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert run.error() == (F.LS_OK, 0)
    del g, busy
