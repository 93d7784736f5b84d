"""The drafting round a drafter runs with sampled decoding (T > 0), as one chain of calls
on one stream with no synchronisation between them: ls_accept_sampled (the verified
block's acceptance), ls_commit_accepted (the accepted rows into the views),
ls_draft_prologue (boundary keys/values from the new boundary view, queries from the
block inputs) and ls_draft_attend over the views with those projections.

The projections stream their weights before the commit ahead of them has completed, and
the attention loads its first rows of the views before the projections have completed;
every round's outputs must equal those of the same calls with a synchronisation after each
one, bit for bit. Against the oracle: accepted counts bit for bit, drawn tokens where the
oracle's CDF crosses the draw, the views after the last round, the projections of the last
round within their accumulation bound, and its attention within 1e-2.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
from tests import oracle_side as OS  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL

EPS_REL = 64 * 2.0 ** -24


def _wl():
    # fp32 attention output: the 1e-2 bound then holds whatever the outputs' magnitude
    return WL.Workload(name="chain", seed=17, batch=4, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128,
                       hidden=512, block=16, window=128, scales=(32, 64, 256), slots=4, dtype="bf16",
                       prefix=(300, 1400), rounds=3, accept_mean=None, vocab=1000, head_scale=True,
                       flags=F.LS_FLAG_OUT_F32)


def _probs(rng, shape, z=None, noise=0.5):
    x = rng.standard_normal(shape) * 2.0 if z is None else z + noise * rng.standard_normal(shape)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32), x


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _inputs(wl, rng, dev):
    b, B, V, L, H, Hq, D, hid = (wl.batch, wl.block, 1000, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim,
                                 wl.hidden)
    rounds = []
    for _ in range(wl.rounds):
        q, zq = _probs(rng, (b, B, V))
        p, _ = _probs(rng, (b, B + 1, V), z=np.concatenate([zq, zq[:, -1:]], axis=1), noise=0.6)
        draft = np.array([[np.searchsorted(np.cumsum(q[i, j], dtype=np.float64), rng.random())
                           for j in range(B)] for i in range(b)]).clip(0, V - 1).astype(np.int32)
        u = rng.random((b, B + 1)).astype(np.float32)
        x = torch.from_numpy(rng.standard_normal((b, L, B, hid)).astype(np.float32)).to(dev).to(torch.bfloat16)
        rounds.append(dict(q=q, p=p, draft=draft, u=u, x=x))
    g = torch.Generator(device=dev).manual_seed(5)
    w_kv = (torch.randn((L, 2 * H * D, hid), device=dev, generator=g) * hid ** -0.5).to(torch.bfloat16)
    w_q = (torch.randn((L, Hq * D, hid), device=dev, generator=g) * hid ** -0.5).to(torch.bfloat16)
    return rounds, w_kv, w_q


def _chain(wl, rounds, w_kv, w_q, sync):
    """Every round's four calls; returns the run, the device inputs and per-round outputs."""
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    dev, st = run.dev, run.stream
    H, D = wl.n_kv_heads, wl.head_dim
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)  # noqa: E731
    dev_in = [dict(q=t(r["q"]), p=t(r["p"]), draft=t(r["draft"]), u=t(r["u"])) for r in rounds]
    torch.cuda.synchronize()
    outs = []
    for i, r in enumerate(rounds):
        o = dict(acc=torch.full((wl.batch,), -1, dtype=torch.int32, device=dev),
                 nxt=torch.full((wl.batch,), -1, dtype=torch.int32, device=dev),
                 bkv=torch.full((wl.batch, wl.n_layers, 2 * H * D), float("nan"), dtype=torch.bfloat16, device=dev),
                 qd=torch.full((wl.batch, wl.n_layers, wl.block, wl.n_q_heads * D), float("nan"),
                               dtype=torch.bfloat16, device=dev),
                 out=run.new_out())
        d = dev_in[i]
        F.ls_accept_sampled(run.state, d["draft"], d["q"], d["p"], 1000, d["u"], o["acc"], o["nxt"], st)
        if sync:
            torch.cuda.synchronize()
        F.ls_commit_accepted(run.state, o["acc"], inp["vk"][i], inp["vv"][i], inp["vh"][i], st)
        if sync:
            torch.cuda.synchronize()
        F.ls_draft_prologue(run.state, w_kv, w_q, r["x"], o["bkv"], o["qd"], st)
        if sync:
            torch.cuda.synchronize()
        F.ls_draft_attend(run.state, 0, wl.n_layers, o["qd"], o["bkv"], o["bkv"][..., H * D:], 2 * H * D,
                          run.softmax_scale, o["out"], st)
        if sync:
            torch.cuda.synchronize()
        outs.append(o)
    torch.cuda.synchronize()
    return run, inp, outs


def test_drafting_round_chain():
    wl = _wl()
    dev = torch.device("cuda")
    rounds, w_kv, w_q = _inputs(wl, np.random.default_rng(31), dev)
    run, inp, outs = _chain(wl, rounds, w_kv, w_q, sync=False)
    ref_run, _, ref_outs = _chain(wl, rounds, w_kv, w_q, sync=True)
    for i in range(wl.rounds):
        for k in outs[i]:
            assert torch.equal(outs[i][k], ref_outs[i][k]), (i, k)
    st = run.read_state()
    for k, v in ref_run.read_state().items():
        assert np.array_equal(st[k], v), k
    assert run.error() == (F.LS_OK, 0) and ref_run.error() == (F.LS_OK, 0)

    # the oracle: acceptance, draws, views, projections, attention
    B, L, H, Hq, D, hid = wl.block, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden
    acc = np.zeros((wl.rounds, wl.batch), dtype=np.int64)
    for i, r in enumerate(rounds):
        a_gpu, n_gpu = outs[i]["acc"].cpu().numpy(), outs[i]["nxt"].cpu().numpy()
        for b in range(wl.batch):
            a, _ = O.accept_decisions(r["draft"][b], r["q"][b], r["p"][b], r["u"][b, :B])
            assert a_gpu[b] == a, (i, b)
            w = O.draw_weights(r["q"][b], r["p"][b], a)
            cdf = np.cumsum(w)
            z, thr, tk = cdf[-1], float(r["u"][b, B]) * cdf[-1], int(n_gpu[b])
            lo = cdf[tk - 1] if tk > 0 else 0.0
            assert w[tk] > 0 and lo <= thr + EPS_REL * z and cdf[tk] >= thr - EPS_REL * z, (i, b)
            acc[i, b] = a
    last = wl.rounds - 1
    o = outs[last]
    BKV, Q = O.to_f64(_bits(o["bkv"]), "bf16"), O.to_f64(_bits(o["qd"]), "bf16")
    Wkv, Wq = O.to_f64(_bits(w_kv), "bf16"), O.to_f64(_bits(w_q), "bf16")
    X = O.to_f64(_bits(rounds[last]["x"]), "bf16")
    for b in range(wl.batch):
        for l in range(L):
            hid_bl = OS.boundary_hidden(wl, b, l, last, int(acc[last, b]))
            assert np.array_equal(st["boundary"][b, l], hid_bl)
            h = O.to_f64(hid_bl, "bf16")
            ref_bkv, ref_q = O.draft_prologue(Wkv[l:l + 1], Wq[l:l + 1], h[None, None], X[b:b + 1, l:l + 1])
            bound = 2.0 ** -8 * np.abs(ref_bkv[0, 0]) + hid * 2.0 ** -24 * (np.abs(Wkv[l]) @ np.abs(h))
            assert np.all(np.abs(BKV[b, l] - ref_bkv[0, 0]) <= bound), (b, l, "bkv")
            bq = 2.0 ** -8 * np.abs(ref_q[0, 0]) + hid * 2.0 ** -24 * (np.abs(X[b, l]) @ np.abs(Wq[l]).T)
            assert np.all(np.abs(Q[b, l] - ref_q[0, 0]) <= bq), (b, l, "q")
            for g in range(H):
                sh, views = OS.tile_views(wl, b, l, g, int(run.prefix_len[b]), acc[:, b], run.scale_host)
                OS.check_tile_state(wl, st, b, l, g, views)
                qt = Q[b, l].reshape(B, Hq, D)[:, g * wl.group:(g + 1) * wl.group][None]
                bk = BKV[b, l, g * D:(g + 1) * D].reshape(1, 1, D)
                bv = BKV[b, l, H * D + g * D:H * D + (g + 1) * D].reshape(1, 1, D)
                ref = O.draft_attend(sh, views, qt, bk, bv, 1.0 / np.sqrt(D))[0]
                got = o["out"][b, l].view(B, Hq, D)[:, g * wl.group:(g + 1) * wl.group].double().cpu().numpy()
                assert OS.attend_error_excess(got, ref) <= 0, (b, l, g)
