"""Stochastic acceptance (speculative sampling for T > 0) on the GPU against the oracle.

The accepted count is compared bit for bit: both sides make the test u * q(d) < p(d) in
fp32. The drawn token is an inverse-CDF sample over up to 524288 fp32 weights summed in the
kernel's order; it must lie where the oracle's fp64 CDF (of the same weights) crosses
u_B * total, up to the fp32 summation bound 64 * 2^-24 * total (the kernel's sums are at
most about 42 additions deep), and carry mass.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL

EPS_REL = 64 * 2.0 ** -24


def _probs(rng, shape, z=None, noise=0.5):
    """fp32 softmax rows of seeded normal logits (shared logits z plus noise, if given)."""
    x = rng.standard_normal(shape) * 2.0 if z is None else z + noise * rng.standard_normal(shape)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32), x


def _state(batch, block):
    wl = WL.Workload(name="sample", seed=3, batch=batch, n_layers=1, n_kv_heads=2, n_q_heads=8, head_dim=128,
                     hidden=512, block=block, window=128, scales=(32, 64, 256), slots=4, dtype="bf16",
                     prefix=(300, 300), rounds=1, accept_mean=None, vocab=1000, head_scale=True)
    return WL.DeviceRun(wl)


def _run(run, draft, q, p, u):
    dev = run.dev
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    acc = torch.full((draft.shape[0],), -1, dtype=torch.int32, device=dev)
    nxt = torch.full((draft.shape[0],), -1, dtype=torch.int32, device=dev)
    F.ls_accept_sampled(run.state, t(draft.astype(np.int32)), t(q), t(p), q.shape[-1], t(u.astype(np.float32)),
                        acc, nxt, run.stream)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), nxt.cpu().numpy()


def _check(draft, q, p, u, acc, nxt):
    B = draft.shape[1]
    for b in range(draft.shape[0]):
        a, _ = O.accept_decisions(draft[b], q[b], p[b], u[b, :B])
        assert acc[b] == a, (b, acc[b], a)
        w = O.draw_weights(q[b], p[b], a)
        t = int(nxt[b])
        cdf = np.cumsum(w)
        z = cdf[-1]
        thr = float(np.float32(u[b, B])) * z
        lo = cdf[t - 1] if t > 0 else 0.0
        assert 0 <= t < len(w) and w[t] > 0, (b, t)
        assert lo <= thr + EPS_REL * z and cdf[t] >= thr - EPS_REL * z, (b, t, lo, cdf[t], thr)


@pytest.mark.parametrize("vocab", [1000, 8192, 40000])
def test_sampled_random(vocab):
    """Draft tokens drawn from q; p close to q (most drafts kept, some rejected)."""
    rng = np.random.default_rng(vocab)
    b, B = 8, 16
    run = _state(b, B)
    q, zq = _probs(rng, (b, B, vocab))
    p, _ = _probs(rng, (b, B + 1, vocab), z=np.concatenate([zq, zq[:, -1:]], axis=1), noise=0.7)
    draft = np.array([[np.searchsorted(np.cumsum(q[i, j], dtype=np.float64), rng.random() * q[i, j].sum(dtype=np.float64))
                       for j in range(B)] for i in range(b)]).clip(0, vocab - 1)
    u = rng.random((b, B + 1))
    acc, nxt = _run(run, draft, q, p, u)
    _check(draft, q, p, u, acc, nxt)
    assert (acc < B).any()  # the residual draw is exercised
    assert run.error() == (F.LS_OK, 0)


def test_sampled_edge_cases():
    rng = np.random.default_rng(7)
    b, B, V = 6, 8, 4096
    run = _state(b, B)
    q, _ = _probs(rng, (b, B, V))
    p = np.concatenate([q, _probs(rng, (b, 1, V))[0]], axis=1)
    draft = rng.integers(0, V, (b, B))
    u = rng.random((b, B + 1))
    # sequence 0: q = p everywhere: every draft kept, the bonus drawn from p_B
    # sequence 1: the first draft has no target mass: rejected, residual = p_0 there
    p[1, 0, draft[1, 0]] = 0.0
    # sequence 2: u_B near 1 and near 0 (ends of the inverse CDF)
    u[2, B] = 0.999999
    u[3, B] = 0.0
    p[3, 2, draft[3, 2]] = 0.0  # sequence 3 rejects at position 2
    # sequence 4: p_0 = q_0 and a first draft both give no mass: rejected, the residual has
    # no mass, the token comes from p_0 (draws in three different chunks of the row)
    q[4, 0, draft[4, 0]] = 0.0
    p[4, 0] = q[4, 0]
    u[4, B] = 0.73
    # sequence 5: rows equal up to rounding: p_0 one fp32 step below q_0 at the draft, whose
    # test fails only because u_0 * q_0(d) rounds to p_0(d)
    d5 = int(draft[5, 0])
    q[5, 0, d5] = np.float32(0.75)
    p[5, 0] = q[5, 0]
    p[5, 0, d5] = np.nextafter(np.float32(0.75), np.float32(0))
    u[5, 0] = 1 - 2.0 ** -24
    acc, nxt = _run(run, draft, q, p, u)
    _check(draft, q, p, u, acc, nxt)
    assert acc[0] == B and acc[1] == 0 and acc[3] == 2 and acc[4] == 0 and acc[5] == 0
    for i in (4, 5):
        assert not (O.sampling_weights(q[i], p[i], 0) > 0).any()  # the branch is taken
        assert p[i, 0, nxt[i]] > 0
    assert run.error() == (F.LS_OK, 0)


def test_sampled_qwen_vocab():
    """The Qwen3 vocabulary (151936 entries, 19 chunks) at batch 16, block 16."""
    rng = np.random.default_rng(11)
    b, B, V = 16, 16, 151936
    run = _state(b, B)
    q, zq = _probs(rng, (b, B, V))
    p, _ = _probs(rng, (b, B + 1, V), z=np.concatenate([zq, zq[:, -1:]], axis=1), noise=0.4)
    draft = np.argmax(q + 0.0, axis=-1)  # the drafter's likeliest token
    u = rng.random((b, B + 1))
    acc, nxt = _run(run, draft, q, p, u)
    _check(draft, q, p, u, acc, nxt)
    assert run.error() == (F.LS_OK, 0)


def test_sampled_errors():
    rng = np.random.default_rng(5)
    b, B, V = 2, 4, 64
    run = _state(b, B)
    q, _ = _probs(rng, (b, B, V))
    p, _ = _probs(rng, (b, B + 1, V))
    u = rng.random((b, B + 1))
    dev = run.dev
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    out = torch.zeros(b, dtype=torch.int32, device=dev)
    with pytest.raises(F.LsError):  # vocabulary not a multiple of 4
        F.ls_accept_sampled(run.state, t(np.zeros((b, B), np.int32)), t(q[..., :63]), t(p[..., :63]), 63,
                            t(u.astype(np.float32)), out, out, run.stream)
    draft = rng.integers(0, V, (b, B)).astype(np.int32)
    draft[1, 0] = V + 5  # outside the vocabulary: error bit, treated as rejected
    acc, nxt = _run(run, draft, q, p, u)
    assert acc[1] == 0
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_SAMPLE
    # a target row without mass to draw from: error bit, token 0
    F.ls_clear_error(run.state, run.stream)
    draft = rng.integers(0, V, (b, B)).astype(np.int32)
    p[0, 0] = 0.0  # the first draft is rejected (no target mass) and p_0 has none either
    acc, nxt = _run(run, draft, q, p, u)
    assert acc[0] == 0 and nxt[0] == 0
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_SAMPLE


def test_commit_accepted_equals_greedy_commit():
    """ls_commit_accepted with the greedy scan's counts leaves the state bit-identical."""
    wl = WL.Workload(name="acc", seed=9, batch=3, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128, hidden=512,
                     block=16, window=128, scales=(32, 64, 256), slots=4, dtype="bf16", prefix=(300, 1400), rounds=6,
                     accept_mean=None, vocab=1000, head_scale=True)
    runs = [WL.DeviceRun(wl), WL.DeviceRun(wl)]
    for r in runs:
        r.prefill()
    inp = runs[0].make_round_inputs()
    for i in range(wl.rounds):
        runs[0].commit(inp, i)
        torch.cuda.synchronize()
        F.ls_commit_accepted(runs[1].state, runs[0].accept_len.clone(), inp["vk"][i], inp["vv"][i], inp["vh"][i],
                             runs[1].stream)
    torch.cuda.synchronize()
    s0, s1 = runs[0].read_state(), runs[1].read_state()
    for k in s0:
        assert np.array_equal(s0[k], s1[k]), k
    assert runs[0].error() == (F.LS_OK, 0) and runs[1].error() == (F.LS_OK, 0)
