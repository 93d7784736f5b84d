"""The drafter's projections (ls_draft_prologue) on the tensor cores against the oracle.

Bound per output element, from the arithmetic: fp32 accumulation of K = hidden bf16
products (at most K * 2^-24 * sum_k |w x| whatever the order) plus the bf16 rounding of
the result (an 8-bit significand: within 2^-8 |y| when rounded to nearest):
    |gpu - ref| <= 2^-8 |ref| + hidden * 2^-24 * sum_k |w_nk x_mk|
Selection weights (ones that pick hidden dimensions) make every sum exact, so the
boundary keys/values then equal the slice stand-in bit for bit.

Where the tiles do not fill whole waves of CTAs, the boundary tiles left over are split
along the hidden size and their fp32 partial sums added in a fixed order: the bound above
holds for any association, and repeated calls give the same bits.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


def _wl(**kw):
    base = dict(name="pro", seed=13, batch=3, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128, hidden=512,
                block=16, window=128, scales=(32, 64, 256), slots=4, dtype="bf16", prefix=(300, 900), rounds=1,
                accept_mean=None, vocab=1000, head_scale=True)
    base.update(kw)
    return WL.Workload(**base)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _f64(t):
    return O.to_f64(_bits(t), "bf16")


def _gen(shape, seed, dev, scale):
    g = torch.Generator(device=dev).manual_seed(seed)
    return (torch.randn(shape, device=dev, generator=g) * scale).to(torch.bfloat16)


def _run_prologue(run, wl, w_kv, w_q, x):
    dev = run.dev
    H, Hq, D = wl.n_kv_heads, wl.n_q_heads, wl.head_dim
    bkv = torch.full((wl.batch, wl.n_layers, 2 * H * D), float("nan"), dtype=torch.bfloat16, device=dev)
    q = torch.full((wl.batch, wl.n_layers, wl.block, Hq * D), float("nan"), dtype=torch.bfloat16, device=dev)
    F.ls_draft_prologue(run.state, w_kv, w_q, x, bkv, q, run.stream)
    torch.cuda.synchronize()
    return bkv, q


def _check(got, ref, absprod):
    bound = 2.0 ** -8 * np.abs(ref) + absprod
    exc = np.abs(got - ref) - bound
    assert np.all(np.isfinite(got)) and exc.max() <= 0, float(exc.max())


def _bound_terms(w, x_rows, hidden):
    """hidden * 2^-24 * sum_k |w_nk x_mk| for rows x_rows [m][k] and weights w [n][k]."""
    return hidden * 2.0 ** -24 * (np.abs(x_rows) @ np.abs(w).T)


@pytest.mark.parametrize("batch,block", [(3, 16), (5, 8), (16, 16)])
def test_prologue_mid(batch, block):
    wl = _wl(batch=batch, block=block)
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 1, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 2, dev, hid ** -0.5)
    x = _gen((batch, L, B, hid), 3, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    h = O.to_f64(run.read_state()["boundary"], "bf16")
    Wkv, Wq, X = _f64(w_kv), _f64(w_q), _f64(x)
    ref_bkv, ref_q = O.draft_prologue(Wkv, Wq, h, X)
    for l in range(L):
        _check(_f64(bkv)[:, l], ref_bkv[:, l], _bound_terms(Wkv[l], h[:, l], hid))
        _check(_f64(q)[:, l].reshape(-1, Hq * D), ref_q[:, l].reshape(-1, Hq * D),
               _bound_terms(Wq[l], X[:, l].reshape(-1, hid), hid))
    assert run.error() == (F.LS_OK, 0)


def test_prologue_selection_weights_reproduce_the_slices():
    """W_kv picking hidden dims 0 .. 2 Hkv D - 1: the boundary keys/values are the slices
    of the boundary view the tests and the bench otherwise pass, bit for bit."""
    wl = _wl()
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = torch.zeros((L, 2 * H * D, hid), dtype=torch.bfloat16, device=dev)
    w_kv[:, torch.arange(2 * H * D), torch.arange(2 * H * D)] = 1.0
    w_q = torch.zeros((L, Hq * D, hid), dtype=torch.bfloat16, device=dev)
    sel = torch.randint(0, hid, (Hq * D,), generator=torch.Generator().manual_seed(4)).to(dev)  # one dim per row
    w_q[:, torch.arange(Hq * D, device=dev), sel] = 1.0
    x = _gen((wl.batch, L, B, hid), 5, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    h_bits = run.read_state()["boundary"]
    assert np.array_equal(_bits(bkv), h_bits[:, :, :2 * H * D])
    assert np.array_equal(_bits(q), _bits(x)[..., sel.cpu().numpy()])


def test_prologue_feeds_the_attention():
    """Prologue outputs as ls_draft_attend's queries and boundary rows (stride 2 Hkv D)
    against the oracle's attention over the same bf16 values."""
    from tests import oracle_side as OS
    wl = _wl(rounds=2)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    for r in range(wl.rounds):
        run.commit(inp, r)
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 6, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 7, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 8, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    out = run.new_out()
    F.ls_draft_attend(run.state, 0, L, q, bkv, bkv[..., H * D:], 2 * H * D, 1.0 / np.sqrt(D), out, run.stream)
    torch.cuda.synchronize()
    st = run.read_state()
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    acc = OS.accepts_from_ids(draft[:wl.rounds], target[:wl.rounds])
    BKV, Q = _f64(bkv), _f64(q)
    for b, l, g in [(0, 0, 0), (wl.batch - 1, L - 1, H - 1), (1, 1, 0)]:
        sh, views = OS.tile_views(wl, b, l, g, int(run.prefix_len[b]), acc[:, b], run.scale_host)
        OS.check_tile_state(wl, st, b, l, g, views)
        qt = Q[b, l].reshape(B, Hq, D)[:, g * wl.group:(g + 1) * wl.group][None]
        bk = BKV[b, l, g * D:(g + 1) * D].reshape(1, 1, D)
        bv = BKV[b, l, H * D + g * D:H * D + (g + 1) * D].reshape(1, 1, D)
        ref = O.draft_attend(sh, views, qt, bk, bv, 1.0 / np.sqrt(D))[0]
        got = out[b, l].view(B, Hq, D)[:, g * wl.group:(g + 1) * wl.group].double().cpu().numpy()
        assert OS.attend_error_excess(got, ref) <= 0
    assert run.error() == (F.LS_OK, 0)


def test_prologue_qwen_shapes():
    """Qwen3-8B shapes (hidden 4096, 32 query / 8 KV heads, 4 layers, batch 16, block 16:
    192 units of 128 weight rows), checked on sampled rows."""
    wl = _wl(batch=16, n_layers=4, n_kv_heads=8, n_q_heads=32, hidden=4096, prefix=(300, 300))
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 9, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 10, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 11, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    h = O.to_f64(run.read_state()["boundary"], "bf16")
    BKV, Q = _f64(bkv), _f64(q)
    for l in range(L):
        Wkv = _f64(w_kv[l])
        ref = h[:, l] @ Wkv.T
        _check(BKV[:, l], ref, _bound_terms(Wkv, h[:, l], hid))
        Wq = _f64(w_q[l])
        rows = [(0, 0), (7, 5), (15, 15)]
        Xs = np.stack([_f64(x[b, l, i]) for b, i in rows])
        _check(np.stack([Q[b, l, i] for b, i in rows]), Xs @ Wq.T, _bound_terms(Wq, Xs, hid))
    assert run.error() == (F.LS_OK, 0)


def test_prologue_split_tiles_match_the_oracle():
    """384 tiles on the GPU's CTAs (256 query tiles, 128 boundary tiles over 8 layers): the
    boundary tiles past the last whole wave run split along the hidden size. Every output
    against the oracle; a second call gives the same bits (pieces summed in a fixed order)."""
    wl = _wl(batch=16, n_layers=8, n_kv_heads=8, n_q_heads=32, hidden=512, prefix=(300, 300))
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 21, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 22, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 23, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    bkv2, q2 = _run_prologue(run, wl, w_kv, w_q, x)
    assert torch.equal(bkv, bkv2) and torch.equal(q, q2)
    h = O.to_f64(run.read_state()["boundary"], "bf16")
    Wkv, Wq, X = _f64(w_kv), _f64(w_q), _f64(x)
    ref_bkv, ref_q = O.draft_prologue(Wkv, Wq, h, X)
    for l in range(L):
        _check(_f64(bkv)[:, l], ref_bkv[:, l], _bound_terms(Wkv[l], h[:, l], hid))
        _check(_f64(q)[:, l].reshape(-1, Hq * D), ref_q[:, l].reshape(-1, Hq * D),
               _bound_terms(Wq[l], X[:, l].reshape(-1, hid), hid))
    assert run.error() == (F.LS_OK, 0)


def test_prologue_leftover_tiles_with_few_k_steps():
    """Hidden 128 (2 k-steps per tile) at Qwen3-8B head counts: 192 tiles on 148 CTAs leave
    44 boundary tiles, only 88 k-steps, fewer than the CTAs. Split over every CTA, some CTAs'
    ranges would be empty and a tile's pieces fewer than the CTAs its first and last k-steps
    span, so its sum would never be stored; such leftovers run whole instead. Every output
    against the oracle."""
    wl = _wl(batch=16, n_layers=4, n_kv_heads=8, n_q_heads=32, hidden=128, prefix=(300, 300))
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 51, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 52, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 53, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    h = O.to_f64(run.read_state()["boundary"], "bf16")
    Wkv, Wq, X = _f64(w_kv), _f64(w_q), _f64(x)
    ref_bkv, ref_q = O.draft_prologue(Wkv, Wq, h, X)
    for l in range(L):
        _check(_f64(bkv)[:, l], ref_bkv[:, l], _bound_terms(Wkv[l], h[:, l], hid))
        _check(_f64(q)[:, l].reshape(-1, Hq * D), ref_q[:, l].reshape(-1, Hq * D),
               _bound_terms(Wq[l], X[:, l].reshape(-1, hid), hid))
    assert run.error() == (F.LS_OK, 0)


def test_prologue_split_tiles_selection_exact():
    """The split boundary tiles with selection weights: every partial sum is exact, so the
    keys/values equal the boundary slices bit for bit however the pieces are cut."""
    wl = _wl(batch=16, n_layers=8, n_kv_heads=8, n_q_heads=32, hidden=2048, prefix=(300, 300))
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = torch.zeros((L, 2 * H * D, hid), dtype=torch.bfloat16, device=dev)
    w_kv[:, torch.arange(2 * H * D), torch.arange(2 * H * D)] = 1.0
    w_q = _gen((L, Hq * D, hid), 24, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 25, dev, 1.0)
    bkv, _ = _run_prologue(run, wl, w_kv, w_q, x)
    assert np.array_equal(_bits(bkv), run.read_state()["boundary"][:, :, :2 * H * D])
    assert run.error() == (F.LS_OK, 0)


def test_prologue_batch_past_one_activation_tile():
    """Batch 300: both problems run two activation tiles (the second ragged: 44 rows, the
    rest of its box zero-filled), and the 88 boundary tiles left after whole waves (all of
    the ragged tile) are split with 256-row partial sums. Every boundary key/value and the
    queries of sequences on both sides of the tile edge against the oracle."""
    wl = _wl(batch=300, n_layers=8, n_kv_heads=8, n_q_heads=32, hidden=512, prefix=(300, 300))
    run = WL.DeviceRun(wl)
    run.prefill()
    dev = run.dev
    L, H, Hq, D, hid, B = wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    w_kv = _gen((L, 2 * H * D, hid), 31, dev, hid ** -0.5)
    w_q = _gen((L, Hq * D, hid), 32, dev, hid ** -0.5)
    x = _gen((wl.batch, L, B, hid), 33, dev, 1.0)
    bkv, q = _run_prologue(run, wl, w_kv, w_q, x)
    h = O.to_f64(run.read_state()["boundary"], "bf16")
    BKV, Q = _f64(bkv), _f64(q)
    for l in range(L):
        Wkv = _f64(w_kv[l])
        _check(BKV[:, l], h[:, l] @ Wkv.T, _bound_terms(Wkv, h[:, l], hid))
    seqs = [0, 15, 16, 255, 256, 299]
    for l in (0, L - 1):
        Wq = _f64(w_q[l])
        Xs = _f64(x[seqs, l]).reshape(-1, hid)
        _check(Q[seqs, l].reshape(-1, Hq * D), Xs @ Wq.T, _bound_terms(Wq, Xs, hid))
    assert run.error() == (F.LS_OK, 0)
