"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one piece of the oracle against a closed form, a brute-force
enumeration, a hand-worked example (tests/golden/), an invariant the method states, or
a library routine. The sources: LongSpark paper page (thelatestinai.com), Figure 2
caption (round structure), Figure 3 caption (incremental summary, Delta <= B + 1),
Figure 1 caption (fixed-size state), Table 3 caption (greedy T = 0 acceptance).
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _shapes(**kw):
    base = dict(n_layers=2, n_kv_heads=2, n_q_heads=4, head_dim=8, hidden=32, block=4,
                window=8, scales=(5, 10, 40), slots=3)
    base.update(kw)
    return O.Shapes(**base)


def _rows(rng, L, H, n, D):
    return rng.standard_normal((L, H, n, D))


# ---------------------------------------------------------------------------------
# accept scan
# ---------------------------------------------------------------------------------
def test_scan_exhaustive_b16():
    """All 2^16 agreement patterns: a = count of leading agreements (cumulative product)."""
    B = 16
    masks = np.arange(1 << B, dtype=np.int64)
    agree = ((masks[:, None] >> np.arange(B)[None, :]) & 1) == 0  # bit set = disagreement
    brute = np.cumprod(agree, axis=1).sum(axis=1)
    draft = np.arange(B) + 100
    for m in range(1 << B):
        target = np.concatenate([draft + ((m >> np.arange(B)) & 1) * 7, [9999]])
        a, nxt = O.accept_scan(draft, target)
        assert a == brute[m]
        assert nxt == (target[a])
        assert a + 1 <= B + 1


def test_scan_golden_examples():
    with open(os.path.join(GOLDEN, "accept_scan_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        a, nxt = O.accept_scan(c["draft"], c["target"])
        assert (a, nxt, a + 1) == (c["a"], c["next"], c["delta"])


# ---------------------------------------------------------------------------------
# summary and window
# ---------------------------------------------------------------------------------
def _full_cache_run(sh, rng, P, accepts):
    """Prefill P random rows, commit rounds with the given accepts; return (views, cache)."""
    L, H, D, B = sh.n_layers, sh.n_kv_heads, sh.head_dim, sh.block
    pk = rng.standard_normal((L, P, H, D))
    pv = rng.standard_normal((L, P, H, D))
    hid = rng.standard_normal((L, sh.hidden))
    v = O.prefill(sh, pk, pv, P, hid)
    cache_k = [np.transpose(pk, (0, 2, 1, 3))]
    cache_v = [np.transpose(pv, (0, 2, 1, 3))]
    for a in accepts:
        draft = rng.integers(0, 50, B)
        target = np.concatenate([draft, [0]]).copy()
        if a < B:
            target[a] = draft[a] + 1
        vk = rng.standard_normal((L, B + 1, H, D))
        vv = rng.standard_normal((L, B + 1, H, D))
        vh = rng.standard_normal((L, B + 1, sh.hidden))
        got_a, _ = O.commit_round(sh, v, draft, target, vk, vv, vh)
        assert got_a == a
        cache_k.append(np.transpose(vk[:, :a + 1], (0, 2, 1, 3)))
        cache_v.append(np.transpose(vv[:, :a + 1], (0, 2, 1, 3)))
    return v, np.concatenate(cache_k, axis=2), np.concatenate(cache_v, axis=2)


def _assert_views_close(sh, a, b, rtol=1e-12):
    assert a.length == b.length
    assert a.n_seg == b.n_seg and a.part_count == b.part_count
    np.testing.assert_array_equal(a.ring_k, b.ring_k)
    np.testing.assert_array_equal(a.ring_v, b.ring_v)
    for k in range(len(sh.scales)):
        filled = min(a.n_seg[k], sh.slots)
        np.testing.assert_allclose(a.seg_k[k][:, :, :filled], b.seg_k[k][:, :, :filled], rtol=rtol, atol=1e-12)
        np.testing.assert_allclose(a.seg_v[k][:, :, :filled], b.seg_v[k][:, :, :filled], rtol=rtol, atol=1e-12)
        np.testing.assert_allclose(a.part_k[k], b.part_k[k], rtol=rtol, atol=1e-11)
        np.testing.assert_allclose(a.part_v[k], b.part_v[k], rtol=rtol, atol=1e-11)
    np.testing.assert_allclose(a.glob_k, b.glob_k, rtol=rtol, atol=1e-10)
    np.testing.assert_allclose(a.glob_v, b.glob_v, rtol=rtol, atol=1e-10)


@pytest.mark.parametrize("P", [0, 1, 7, 40, 123])
def test_incremental_equals_recompute(P):
    """Figure 3: updating with only the new rows N equals the summary of the whole cache."""
    sh = _shapes()
    rng = np.random.default_rng(P)
    accepts = rng.integers(0, sh.block + 1, 30)
    v, ck, cv = _full_cache_run(sh, rng, P, accepts)
    ref = O.views_from_scratch(sh, ck, cv, ck.shape[2])
    _assert_views_close(sh, v, ref)


def test_fold_from_empty_equals_recompute():
    """Folding every row one by one from an empty state equals the definition."""
    sh = _shapes(scales=(4, 8, 32), slots=2, window=5)
    rng = np.random.default_rng(5)
    n = 97
    fk, fv = _rows(rng, 2, 2, n, 8), _rows(rng, 2, 2, n, 8)
    v = O.empty_views(sh)
    for p in range(n):
        O.retain_row(sh, v, fk[:, :, p], fv[:, :, p])
    _assert_views_close(sh, v, O.views_from_scratch(sh, fk, fv, n))


def _ramp_cache(L, H, n, D):
    p = np.arange(n).reshape(1, 1, n, 1).astype(np.float64)
    h = np.arange(H).reshape(1, H, 1, 1)
    l = np.arange(L).reshape(L, 1, 1, 1)
    d = np.arange(D).reshape(1, 1, 1, D)
    k = p + 1000.0 * h + 10000.0 * l + 0.25 * d + np.zeros((L, H, n, D))
    return k, -3.0 * k


@pytest.mark.parametrize("n", [0, 3, 64, 200, 511, 512, 513])
def test_ramp_closed_forms(n):
    """K = p + const: segment j of scale s has mean j*s + (s-1)/2 + const, exactly."""
    sh = _shapes(scales=(8, 32, 128), slots=4, window=32, head_dim=4)
    L, H, D = sh.n_layers, sh.n_kv_heads, sh.head_dim
    fk, fv = _ramp_cache(L, H, n, D)
    # incremental fold, the form the round uses
    v = O.empty_views(sh)
    for p in range(n):
        O.retain_row(sh, v, fk[:, :, p], fv[:, :, p])
    const = (1000.0 * np.arange(H)[None, :, None] + 10000.0 * np.arange(L)[:, None, None]
             + 0.25 * np.arange(D)[None, None, :])
    for k, s in enumerate(sh.scales):
        n_c = n // s
        assert v.n_seg[k] == n_c and v.part_count[k] == n - n_c * s
        for j in range(max(0, n_c - sh.slots), n_c):
            want = j * s + (s - 1) / 2.0 + const
            assert np.array_equal(v.seg_k[k][:, :, j % sh.slots], want)
            assert np.array_equal(v.seg_v[k][:, :, j % sh.slots], -3.0 * want)
        c = n - n_c * s
        # partial = sum of rows n_c*s .. n-1 = c*n_c*s + c(c-1)/2 + c*const
        want_part = c * n_c * s + c * (c - 1) / 2.0 + c * const
        assert np.array_equal(v.part_k[k], want_part)
    assert np.array_equal(v.glob_k, n * (n - 1) / 2.0 + n * const)
    # window: ring slot r holds row p with p = r mod W and len - W <= p < len
    for r in range(sh.window):
        ps = [p for p in range(max(0, n - sh.window), n) if p % sh.window == r]
        if ps:
            assert np.array_equal(v.ring_k[:, :, r], ps[0] + const)


def test_constant_rows_give_exact_means():
    sh = _shapes(scales=(3, 9, 27), slots=2)
    c = 0.375
    n = 100
    fk = np.full((2, 2, n, 8), c)
    v = O.views_from_scratch(sh, fk, -fk, n)
    for k in range(3):
        assert np.all(v.seg_k[k][:, :, :min(v.n_seg[k], 2)] == c)
        if v.part_count[k]:
            assert np.all(v.part_k[k] / v.part_count[k] == c)
    assert np.all(v.glob_k / n == c)


def test_window_is_last_w_rows():
    sh = _shapes(window=7)
    rng = np.random.default_rng(1)
    v, ck, cv = _full_cache_run(sh, rng, 30, rng.integers(0, 5, 12))
    n = v.length
    for p in range(n - sh.window, n):
        assert np.array_equal(v.ring_k[:, :, p % sh.window], ck[:, :, p])
        assert np.array_equal(v.ring_v[:, :, p % sh.window], cv[:, :, p])


def test_boundary_is_last_retained_position():
    """The boundary view is the hidden state at position len - 1 after every round."""
    sh = _shapes()
    rng = np.random.default_rng(2)
    L, H, D, B = sh.n_layers, sh.n_kv_heads, sh.head_dim, sh.block
    P = 20
    hid = np.full((L, sh.hidden), P - 1.0)
    v = O.prefill(sh, np.zeros((L, P, H, D)), np.zeros((L, P, H, D)), P, hid)
    assert np.all(v.boundary == v.length - 1)
    for a in [0, 4, 2, 1, 3]:
        draft = np.arange(B)
        target = np.concatenate([draft, [0]])
        if a < B:
            target[a] += 1
        # verify row i sits at absolute position len + i
        vh = (v.length + np.arange(B + 1, dtype=np.float64)).reshape(1, B + 1, 1) * np.ones((L, 1, sh.hidden))
        O.commit_round(sh, v, draft, target, np.zeros((L, B + 1, H, D)), np.zeros((L, B + 1, H, D)), vh)
        assert np.all(v.boundary == v.length - 1)


def test_golden_worked_example():
    with open(os.path.join(GOLDEN, "ramp_worked_example.json")) as f:
        g = json.load(f)
    s = g["shapes"]
    sh = O.Shapes(n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=1, hidden=1, block=1,
                  window=s["window"], scales=tuple(s["scales"]), slots=s["slots"])
    n = g["length"]
    p = np.arange(n, dtype=np.float64).reshape(1, 1, n, 1)
    v = O.views_from_scratch(sh, p, 10 * p, n)
    assert v.ring_k[0, 0, :, 0].tolist() == g["ring_k"]
    assert [v.seg_k[k][0, 0, :, 0].tolist() for k in range(2)] == g["seg_k"]
    assert v.n_seg == g["n_seg"] and v.part_count == g["part_count"]
    assert [float(v.part_k[k][0, 0, 0]) for k in range(2)] == g["part_k"]
    assert float(v.glob_k[0, 0, 0]) == g["glob_k"]
    # the same by folding row by row
    w = O.empty_views(sh)
    for i in range(n):
        O.retain_row(sh, w, p[:, :, i], 10 * p[:, :, i])
    _assert_views_close(sh, v, w)
    out = O.draft_attend(sh, v, np.zeros((1, 1, 1, 1)), np.zeros((1, 1, 1)), np.full((1, 1, 1), 100.0), 1.0)
    assert abs(out[0, 0, 0, 0] - g["attend_q0_out"]) < 1e-12


def test_state_bytes_do_not_depend_on_prefix():
    """Figure 1 caption: the drafter state does not grow with the prefix (4K vs 128K)."""
    sh = _shapes(n_layers=1, n_kv_heads=1, n_q_heads=2, head_dim=4, hidden=16,
                 window=512, scales=(64, 512, 4096), slots=32, block=16)
    sizes = []
    for n in (4096, 131072):
        fk = np.ones((1, 1, n, 4))
        v = O.views_from_scratch(sh, fk, fk, n)
        sizes.append(O.state_bytes(sh, v))
    assert sizes[0] == sizes[1]


# ---------------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------------
def _random_views(sh, rng, P, rounds):
    v, _, _ = _full_cache_run(sh, rng, P, rng.integers(0, sh.block + 1, rounds))
    return v


def test_attend_matches_scalar_loops():
    """Brute force with Python scalars and math.exp on a tiny case."""
    sh = _shapes(n_layers=1, n_kv_heads=2, n_q_heads=4, head_dim=3, window=4,
                 scales=(5, 10), slots=2, block=2)
    rng = np.random.default_rng(3)
    v = _random_views(sh, rng, 13, 4)
    q = rng.standard_normal((1, 2, 4, 3))
    bk, bv = rng.standard_normal((1, 2, 3)), rng.standard_normal((1, 2, 3))
    scale = 0.7
    out = O.draft_attend(sh, v, q, bk, bv, scale)
    for qh in range(4):
        g = qh // 2
        K, V, ok = O.attention_slots(sh, v, 0, g, bk, bv)
        for i in range(2):
            logits = [sum(float(q[0, i, qh, d]) * float(K[s, d]) for d in range(3)) * scale
                      for s in range(len(K))]
            mx = max(lg for lg, o in zip(logits, ok) if o)
            ws = [math.exp(lg - mx) if o else 0.0 for lg, o in zip(logits, ok)]
            tot = sum(ws)
            for d in range(3):
                want = sum(w * float(V[s, d]) for s, w in enumerate(ws)) / tot
                assert abs(out[0, i, qh, d] - want) < 1e-12


def test_attend_matches_torch_sdpa():
    """Library cross-check: torch scaled_dot_product_attention in fp64 with a mask."""
    sh = _shapes(head_dim=16, window=16, scales=(5, 10, 20), slots=3, block=4)
    rng = np.random.default_rng(4)
    v = _random_views(sh, rng, 57, 9)
    q = rng.standard_normal((2, 4, 4, 16))
    bk, bv = rng.standard_normal((2, 2, 16)), rng.standard_normal((2, 2, 16))
    out = O.draft_attend(sh, v, q, bk, bv, 0.25)
    for l in range(2):
        for qh in range(4):
            K, V, ok = O.attention_slots(sh, v, l, qh // 2, bk, bv)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[l, :, qh][None]), torch.from_numpy(K[None]),
                torch.from_numpy(V[None]), attn_mask=torch.from_numpy(ok)[None, None, :].expand(1, 4, -1),
                scale=0.25)
            np.testing.assert_allclose(out[l, :, qh], ref[0].numpy(), rtol=1e-12, atol=1e-12)


def test_attend_special_cases():
    sh = _shapes(n_layers=1, n_kv_heads=1, n_q_heads=2, head_dim=4, window=4,
                 scales=(5, 10), slots=2, block=2)
    rng = np.random.default_rng(6)
    bk, bv = rng.standard_normal((1, 1, 4)), rng.standard_normal((1, 1, 4))
    # empty state: only the boundary slot is valid -> output is exactly its value
    v0 = O.empty_views(sh)
    out = O.draft_attend(sh, v0, rng.standard_normal((1, 2, 2, 4)), bk, bv, 1.0)
    assert np.array_equal(out[0, 0, 0], bv[0, 0]) and np.array_equal(out[0, 1, 1], bv[0, 0])
    # q = 0: uniform weights -> mean of the valid values
    v = _random_views(sh, rng, 23, 5)
    K, V, ok = O.attention_slots(sh, v, 0, 0, bk, bv)
    out = O.draft_attend(sh, v, np.zeros((1, 2, 2, 4)), bk, bv, 1.0)
    np.testing.assert_allclose(out[0, 0, 0], V[ok].mean(axis=0), rtol=1e-12, atol=1e-14)
    # identical keys everywhere -> again the mean of the valid values
    n = 23
    fk = np.ones((1, 1, n, 4))
    fv = rng.standard_normal((1, 1, n, 4))
    w = O.views_from_scratch(sh, fk, fv, n)
    K, V, ok = O.attention_slots(sh, w, 0, 0, np.ones((1, 1, 4)), bv)
    out = O.draft_attend(sh, w, rng.standard_normal((1, 2, 2, 4)), np.ones((1, 1, 4)), bv, 1.0)
    np.testing.assert_allclose(out[0, 1, 0], V[ok].mean(axis=0), rtol=1e-12, atol=1e-14)
    assert ok.sum() == 1 + 4 + (2 + 1) + (2 + 1) + 1


# ---------------------------------------------------------------------------------
# view subsets (Table 5: the component ablations drop one view each)
# ---------------------------------------------------------------------------------
def test_view_of_slots_counts():
    """Slot order [boundary, W window slots, the summary slots]: 1 / W / nsc*(slots+1)+1."""
    sh = _shapes()
    vs = O.view_of_slots(sh)
    assert len(vs) == sh.n_attn_slots
    assert (vs == O.VIEW_BOUNDARY).sum() == 1 and vs[0] == O.VIEW_BOUNDARY
    assert (vs == O.VIEW_WINDOW).sum() == sh.window and (vs[1:1 + sh.window] == O.VIEW_WINDOW).all()
    assert (vs == O.VIEW_SUMMARY).sum() == len(sh.scales) * (sh.slots + 1) + 1


def test_views_boundary_alone_is_its_value():
    """A softmax over the single boundary slot has weight 1: the output is that value row."""
    sh = _shapes()
    rng = np.random.default_rng(11)
    v = _random_views(sh, rng, 37, 6)
    q = rng.standard_normal((2, 4, 4, 8))
    bk, bv = rng.standard_normal((2, 2, 8)), rng.standard_normal((2, 2, 8))
    out, lse = O.draft_attend(sh, v, q, bk, bv, 0.3, views=O.VIEW_BOUNDARY, return_lse=True)
    for l in range(2):
        for qh in range(4):
            g = qh // 2
            assert np.array_equal(out[l, :, qh], np.broadcast_to(bv[l, g], (4, 8)))
            np.testing.assert_allclose(lse[l, :, qh], 0.3 * (q[l, :, qh] @ bk[l, g]), rtol=0, atol=1e-14)


def test_views_constant_values_per_view():
    """Window values all 1, summary values all 0, boundary value 2: attending over one view
    returns that view's constant whatever the keys, and the full attention lies strictly
    between (every view has a valid slot)."""
    sh = _shapes()
    rng = np.random.default_rng(12)
    v = _random_views(sh, rng, 61, 7)
    v.ring_v[:] = 1.0
    for k in range(len(sh.scales)):
        v.seg_v[k][:] = 0.0
        v.part_v[k][:] = 0.0
    v.glob_v[:] = 0.0
    q = rng.standard_normal((2, 4, 4, 8))
    bk, bv = rng.standard_normal((2, 2, 8)), np.full((2, 2, 8), 2.0)
    for views, want in [(O.VIEW_WINDOW, 1.0), (O.VIEW_SUMMARY, 0.0), (O.VIEW_BOUNDARY, 2.0)]:
        out = O.draft_attend(sh, v, q, bk, bv, 0.5, views=views)
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-13)
    out = O.draft_attend(sh, v, q, bk, bv, 0.5)
    assert (out > 0).all() and (out < 2).all()


@pytest.mark.parametrize("split", [(O.VIEW_BOUNDARY, O.VIEW_WINDOW | O.VIEW_SUMMARY),
                                   (O.VIEW_WINDOW, O.VIEW_BOUNDARY | O.VIEW_SUMMARY),
                                   (O.VIEW_SUMMARY, O.VIEW_BOUNDARY | O.VIEW_WINDOW)])
def test_views_partition_identity(split):
    """Softmax over a disjoint union: Z = Z_A + Z_B and O = (Z_A O_A + Z_B O_B) / Z."""
    sh = _shapes()
    rng = np.random.default_rng(13)
    v = _random_views(sh, rng, 53, 8)
    q = rng.standard_normal((2, 4, 4, 8))
    bk, bv = rng.standard_normal((2, 2, 8)), rng.standard_normal((2, 2, 8))
    oa, la = O.draft_attend(sh, v, q, bk, bv, 0.4, views=split[0], return_lse=True)
    ob, lb = O.draft_attend(sh, v, q, bk, bv, 0.4, views=split[1], return_lse=True)
    o, lz = O.draft_attend(sh, v, q, bk, bv, 0.4, return_lse=True)
    np.testing.assert_allclose(lz, np.logaddexp(la, lb), rtol=1e-13, atol=1e-13)
    wa, wb = np.exp(la - lz)[..., None], np.exp(lb - lz)[..., None]
    np.testing.assert_allclose(o, wa * oa + wb * ob, rtol=1e-12, atol=1e-13)


def test_views_with_no_valid_slot_give_zeros():
    """Before any row is retained the window and the summary hold no valid slot."""
    sh = _shapes()
    rng = np.random.default_rng(14)
    v0 = O.empty_views(sh)
    q = rng.standard_normal((2, 4, 4, 8))
    bk, bv = rng.standard_normal((2, 2, 8)), rng.standard_normal((2, 2, 8))
    for views in (O.VIEW_WINDOW, O.VIEW_SUMMARY, O.VIEW_WINDOW | O.VIEW_SUMMARY):
        out, lse = O.draft_attend(sh, v0, q, bk, bv, 1.0, views=views, return_lse=True)
        assert not out.any() and np.isneginf(lse).all()


# ---------------------------------------------------------------------------------
# stochastic acceptance (speculative sampling, T > 0)
# ---------------------------------------------------------------------------------
def test_sampled_emits_target_distribution():
    """The theorem of speculative sampling: with the draft token drawn from q, the token
    emitted at a position is distributed exactly as the target's p. The oracle's decisions
    are integrated over the draft token and a midpoint grid of both uniform draws."""
    rng = np.random.default_rng(21)
    V, N = 6, 4000
    grid = (np.arange(N) + 0.5) / N
    for _ in range(3):
        q = rng.dirichlet(np.ones(V)).astype(np.float32)
        p = rng.dirichlet(np.ones(V)).astype(np.float32)
        p_rows = np.stack([p, rng.dirichlet(np.ones(V)).astype(np.float32)])
        emitted = np.zeros(V)
        for d in range(V):
            rej_next = np.zeros(V)
            for v in grid:
                rej_next[O.accept_sampled([d], q[None], p_rows, [0.999999], v)[1]] += 1.0 / N
            for u in grid:
                a, _ = O.accept_decisions([d], q[None], p_rows, [u])
                if a == 1:
                    emitted[d] += q[d] / N
                else:
                    emitted += q[d] / N * rej_next
        np.testing.assert_allclose(emitted, p.astype(np.float64), rtol=0, atol=2.5 / N)


def test_sampled_equal_distributions_accept_everything():
    rng = np.random.default_rng(22)
    B, V = 5, 11
    q = rng.dirichlet(np.ones(V), size=B).astype(np.float32)
    p_rows = np.concatenate([q, rng.dirichlet(np.ones(V), size=1).astype(np.float32)])
    for _ in range(50):
        d = rng.integers(0, V, B)
        a, nxt = O.accept_sampled(d, q, p_rows, rng.random(B), rng.random())
        assert a == B and p_rows[B, nxt] > 0


def test_sampled_disjoint_support_rejects_first():
    """A draft token the target gives no mass is always rejected; the residual is p."""
    q = np.array([[0.5, 0.5, 0.0, 0.0]], dtype=np.float32)
    p_rows = np.array([[0.0, 0.0, 0.25, 0.75], [0.25, 0.25, 0.25, 0.25]], dtype=np.float32)
    for d in (0, 1):
        for v, want in [(0.1, 2), (0.2499, 2), (0.26, 3), (0.99, 3)]:
            assert O.accept_sampled([d], q, p_rows, [0.0], v) == (0, want)


def test_inverse_cdf_boundaries():
    w = np.array([1.0, 2.0, 3.0, 4.0])
    assert [O.inverse_cdf(w, v) for v in (0.0, 0.05, 0.1, 0.29, 0.3, 0.95, 0.999)] == [0, 0, 1, 1, 2, 3, 3]
    assert {O.inverse_cdf(np.array([0.0, 1.0, 0.0, 1.0]), v) for v in np.linspace(0, 0.999, 101)} == {1, 3}


def test_sampled_residual_without_mass_draws_from_target_row():
    """A rejection whose residual max(0, p_a - q_a) has no mass (p_a <= q_a everywhere).
    Speculative sampling emits samples of the target's distribution, so the token must
    lie in p_a's support, and with p_a = q_a its distribution over the draw v must be p_a
    itself. Hand-worked: p_0 = q_0 = (1/4, 3/4, 0, 0) and a draft (token 2) that both rows
    give no mass: 0 * 0 < 0 fails, a = 0, the residual is all zero, and the inverse CDF of
    p_0 gives token 0 for v < 1/4 and token 1 for 1/4 <= v < 1 (never the draft)."""
    q = np.array([[0.25, 0.75, 0.0, 0.0]], dtype=np.float32)
    p_rows = np.array([[0.25, 0.75, 0.0, 0.0], [0.0, 0.0, 0.0, 1.0]], dtype=np.float32)
    for v, want in [(0.0, 0), (0.1, 0), (0.2499, 0), (0.25, 1), (0.6, 1), (1 - 2.0 ** -24, 1)]:
        assert O.accept_sampled([2], q, p_rows, [0.5], v) == (0, want)
    # the emitted distribution over a midpoint grid of v is p_0 exactly (grid of 4: 1 and 3)
    grid = (np.arange(4) + 0.5) / 4
    assert [O.accept_sampled([2], q, p_rows, [0.5], v)[1] for v in grid] == [0, 1, 1, 1]
    # rows equal up to rounding: p_0(1) is one fp32 step below q_0(1); u = 1 - 2^-24 makes
    # u * q_0(1) round to p_0(1), so the test fails; the residual is zero everywhere and
    # the token comes from p_0 (token 0 for v < 1/4 of its total)
    q2 = np.array([[0.25, 0.75]], dtype=np.float32)
    p2 = np.array([[0.25, np.nextafter(np.float32(0.75), np.float32(0))], [0.5, 0.5]], dtype=np.float32)
    u = np.float32(1 - 2.0 ** -24)
    assert np.float32(u * q2[0, 1]) == p2[0, 1]
    assert not (O.sampling_weights(q2, p2, 0) > 0).any()
    assert O.accept_sampled([1], q2, p2, [u], 0.1) == (0, 0)
    assert O.accept_sampled([1], q2, p2, [u], 0.9) == (0, 1)
    # a target row without any mass is not a distribution: refused
    with pytest.raises(ValueError):
        O.accept_sampled([0], q2, np.zeros((2, 2), np.float32), [0.5], 0.5)


def test_inverse_cdf_exact_brute_force():
    """The draw against its definition in exact rational arithmetic: small integer weights
    (zeros included, leading and trailing) and draws on a dyadic grid of [0, 1) with its
    ends 0 and 1 - 2^-24. The index is the smallest t whose running sum exceeds v times
    the total, and it always carries mass."""
    from fractions import Fraction
    rng = np.random.default_rng(23)
    vs = [0.0, 1 - 2.0 ** -24] + [k / 64 for k in range(64)]
    for _ in range(200):
        n = int(rng.integers(1, 7))
        w = rng.integers(0, 4, n)
        if w.sum() == 0:
            w[int(rng.integers(0, n))] = 1
        tot = int(w.sum())
        for v in vs:
            thr = Fraction(v) * tot
            run, want = 0, None
            for t in range(n):
                run += int(w[t])
                if run > thr:
                    want = t
                    break
            got = O.inverse_cdf(w.astype(np.float64), v)
            assert got == want and w[got] > 0, (w, v, got, want)
    for bad in (1.0, -0.1):
        with pytest.raises(ValueError):
            O.inverse_cdf(np.ones(3), bad)


def test_sampled_decision_is_fp32():
    """u * q rounded to fp32 before the comparison: with p set to that rounded product the
    draft is rejected, although the exact product is below p."""
    u, q = np.float32(0.1), np.float32(0.7)
    prod32 = np.float32(u * q)
    exact = float(u) * float(q)
    assert exact < float(prod32)  # this pair rounds up
    p_rows = np.zeros((2, 2), dtype=np.float32)
    p_rows[0, 0], p_rows[0, 1] = prod32, 1 - prod32
    q_rows = np.array([[q, 1 - q]], dtype=np.float32)
    a, keep = O.accept_decisions([0], q_rows, p_rows, [u])
    assert a == 0 and not keep[0]


# ---------------------------------------------------------------------------------
# drafter prologue (projections of the boundary and the block inputs)
# ---------------------------------------------------------------------------------
def test_prologue_selection_weights_give_the_slices():
    """Weights that select hidden dimensions reproduce the slice stand-in: boundary keys
    h[g D:(g+1) D], values h[Hkv D + g D:...], queries the selected input dimensions."""
    rng = np.random.default_rng(31)
    b, L, B, H, Hq, D, hid = 2, 3, 4, 2, 4, 5, 40
    w_kv = np.zeros((L, 2 * H * D, hid))
    w_kv[:, np.arange(2 * H * D), np.arange(2 * H * D)] = 1.0
    w_q = np.zeros((L, Hq * D, hid))
    sel = rng.permutation(hid)[:Hq * D]
    w_q[:, np.arange(Hq * D), sel] = 1.0
    h = rng.standard_normal((b, L, hid))
    x = rng.standard_normal((b, L, B, hid))
    bkv, q = O.draft_prologue(w_kv, w_q, h, x)
    assert np.array_equal(bkv, h[:, :, :2 * H * D]) and np.array_equal(q, x[..., sel])


def test_prologue_orientation_and_layers():
    """y[n] = sum_k W[n][k] h[k] per layer, by scalar loops; W is not symmetric and every
    layer has its own weights."""
    rng = np.random.default_rng(32)
    b, L, B, hid, nkv, nq = 2, 2, 3, 7, 4, 6
    w_kv, w_q = rng.standard_normal((L, nkv, hid)), rng.standard_normal((L, nq, hid))
    h, x = rng.standard_normal((b, L, hid)), rng.standard_normal((b, L, B, hid))
    bkv, q = O.draft_prologue(w_kv, w_q, h, x)
    for bb in range(b):
        for l in range(L):
            for n in range(nkv):
                assert abs(bkv[bb, l, n] - sum(w_kv[l, n, k] * h[bb, l, k] for k in range(hid))) < 1e-12
            for i in range(B):
                for n in range(nq):
                    assert abs(q[bb, l, i, n] - sum(w_q[l, n, k] * x[bb, l, i, k] for k in range(hid))) < 1e-12


def test_prologue_is_linear():
    rng = np.random.default_rng(33)
    w_kv, w_q = rng.standard_normal((2, 6, 9)), rng.standard_normal((2, 8, 9))
    h1, h2 = rng.standard_normal((3, 2, 9)), rng.standard_normal((3, 2, 9))
    x1, x2 = rng.standard_normal((3, 2, 4, 9)), rng.standard_normal((3, 2, 4, 9))
    a1, q1 = O.draft_prologue(w_kv, w_q, h1, x1)
    a2, q2 = O.draft_prologue(w_kv, w_q, h2, x2)
    a3, q3 = O.draft_prologue(w_kv, w_q, 2 * h1 - h2, 2 * x1 - x2)
    np.testing.assert_allclose(a3, 2 * a1 - a2, atol=1e-12)
    np.testing.assert_allclose(q3, 2 * q1 - q2, atol=1e-12)


# ---------------------------------------------------------------------------------
# paged KV cache (position p in page block_table[b][p // page_size], offset p % page_size)
# ---------------------------------------------------------------------------------
def test_paged_rows_hand_worked():
    """Page size 2, sequence 1's pages 3, 0, 2: positions 0..5 sit in pages 3 3 0 0 2 2
    at offsets 0 1 0 1 0 1 (worked out by hand, stored values name their page/offset)."""
    L, NP, PS, H, D = 2, 4, 2, 1, 1
    pages = np.zeros((L, NP, PS, H, D))
    for l in range(L):
        for pg in range(NP):
            for off in range(PS):
                pages[l, pg, off] = 100 * l + 10 * pg + off
    table = [[1, 2, 3], [3, 0, 2]]
    got = O.paged_rows(pages, table, PS, 1, range(6))
    assert got.shape == (L, 6, H, D)
    assert got[0, :, 0, 0].tolist() == [30, 31, 0, 1, 20, 21]
    assert got[1, :, 0, 0].tolist() == [130, 131, 100, 101, 120, 121]
    assert O.paged_rows(pages, table, PS, 0, [5, 0]).ravel().tolist() == [31, 10, 131, 110]
    assert O.paged_rows(pages, table, PS, 0, []).shape == (L, 0, H, D)


def _scatter_pages(rng, dense, page_size, n_pages_total):
    """Cut [L][P][H][D] rows into pages placed at random page ids; return (pages, table row).
    Positions past P in the last page hold noise, pages nobody owns hold noise too."""
    L, P, H, D = dense.shape
    n_pages = -(-P // page_size)
    ids = rng.permutation(n_pages_total)[:n_pages]
    pages = rng.standard_normal((L, n_pages_total, page_size, H, D))
    for j in range(n_pages):
        chunk = dense[:, j * page_size:(j + 1) * page_size]
        pages[:, ids[j], :chunk.shape[1]] = chunk
    return pages, ids


@pytest.mark.parametrize("P,page_size", [(0, 4), (37, 1), (37, 4), (100, 16), (40, 64)])
def test_paged_prefill_equals_dense(P, page_size):
    sh = _shapes()
    rng = np.random.default_rng(P * 7 + page_size)
    L, H, D = sh.n_layers, sh.n_kv_heads, sh.head_dim
    pk, pv = rng.standard_normal((L, P, H, D)), rng.standard_normal((L, P, H, D))
    hid = rng.standard_normal((L, sh.hidden))
    kp, ids = _scatter_pages(rng, pk, page_size, -(-P // page_size) + 3)
    vp = rng.standard_normal(kp.shape)
    for j, pg in enumerate(ids):
        chunk = pv[:, j * page_size:(j + 1) * page_size]
        vp[:, pg, :chunk.shape[1]] = chunk
    table = [list(ids) + [0] * 2, [0]]  # sequence 0 owns the pages; row 1 is another sequence's
    got = O.prefill_paged(sh, kp, vp, table, page_size, 0, P, hid)
    _assert_views_close(sh, got, O.prefill(sh, pk, pv, P, hid), rtol=0)


@pytest.mark.parametrize("page_size", [1, 3, 16])
def test_paged_commit_equals_dense(page_size):
    """Rounds whose verify rows the target wrote into its pages at positions len .. len + B
    (crossing page boundaries) give the views of the dense rounds."""
    sh = _shapes()
    rng = np.random.default_rng(page_size)
    L, H, D, B = sh.n_layers, sh.n_kv_heads, sh.head_dim, sh.block
    P, accepts = 23, [4, 0, 2, 4, 1, 3]
    total = P + sum(a + 1 for a in accepts[:-1]) + B + 1
    n_pages = -(-total // page_size)
    ids = rng.permutation(n_pages + 5)[:n_pages]
    kp = rng.standard_normal((L, n_pages + 5, page_size, H, D))
    vp = rng.standard_normal(kp.shape)
    pk, pv = rng.standard_normal((L, P, H, D)), rng.standard_normal((L, P, H, D))
    for p in range(P):
        kp[:, ids[p // page_size], p % page_size] = pk[:, p]
        vp[:, ids[p // page_size], p % page_size] = pv[:, p]
    hid = rng.standard_normal((L, sh.hidden))
    dense = O.prefill(sh, pk, pv, P, hid)
    paged = O.prefill_paged(sh, kp, vp, [ids], page_size, 0, P, hid)
    for a in accepts:
        draft = rng.integers(0, 50, B)
        target = np.concatenate([draft, [0]])
        if a < B:
            target[a] = draft[a] + 1
        vk, vv = rng.standard_normal((L, B + 1, H, D)), rng.standard_normal((L, B + 1, H, D))
        vh = rng.standard_normal((L, B + 1, sh.hidden))
        for i in range(B + 1):  # the verify pass writes all B + 1 rows at len + i
            p = dense.length + i
            kp[:, ids[p // page_size], p % page_size] = vk[:, i]
            vp[:, ids[p // page_size], p % page_size] = vv[:, i]
        ra = O.commit_round(sh, dense, draft, target, vk, vv, vh)
        rb = O.commit_round_paged(sh, paged, draft, target, kp, vp, [ids], page_size, 0, vh)
        assert ra == rb and ra[0] == a
        _assert_views_close(sh, paged, dense, rtol=0)
        np.testing.assert_array_equal(paged.boundary, dense.boundary)


def test_mask_counts():
    """Valid slot count = boundary + min(len, W) + per scale min(n_c, slots) + [partial] + [len>0]."""
    sh = _shapes(n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=2, window=16,
                 scales=(4, 16, 64), slots=3)
    for n in [0, 1, 3, 4, 15, 16, 17, 63, 64, 65, 200]:
        fk = np.ones((1, 1, n, 2))
        v = O.views_from_scratch(sh, fk, fk, n)
        _, _, ok = O.attention_slots(sh, v, 0, 0, np.ones((1, 1, 2)), np.ones((1, 1, 2)))
        want = 1 + min(n, 16) + sum(min(n // s, 3) + (1 if n % s else 0) for s in (4, 16, 64)) + (1 if n else 0)
        assert ok.sum() == want and len(ok) == sh.n_attn_slots


def test_to_f64_exact():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], dtype=np.uint16)
    got = O.to_f64(bits, O.BF16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
