"""Test-side glue: rebuild a sampled tile's inputs from the generator and ask the oracle.

Nothing here computes the method: the views and the attention come from ``oracle``; the
inputs come from ``synth`` (the same draws the device runner writes on the GPU).
"""

from __future__ import annotations

import os

import numpy as np

import oracle as O
import synth as S


def shapes_for_tile(wl, n_layers=1, n_kv_heads=1):
    return O.Shapes(n_layers=n_layers, n_kv_heads=n_kv_heads, n_q_heads=wl.group * n_kv_heads,
                    head_dim=wl.head_dim, hidden=wl.hidden, block=wl.block, window=wl.window,
                    scales=tuple(wl.scales), slots=wl.slots)


def accepts_from_ids(draft, target):
    """Oracle scan over every (round, sequence): int [rounds][batch]."""
    R, b = draft.shape[:2]
    return np.array([[O.accept_scan(draft[r, i], target[r, i])[0] for i in range(b)] for r in range(R)],
                    dtype=np.int64)


def tile_cache(wl, b, l, h, P, accepts_b, scale=None):
    """Full K/V cache of tile (b, l, h) after prefill of P rows and len(accepts_b) rounds.

    Returns fp64 arrays [1][1][n][D] for K and V.
    """
    D, B1 = wl.head_dim, wl.block + 1
    R = len(accepts_b)
    ks, vs = [], []
    for tid_p, tid_v, dst in ((S.PREFIX_K, S.VERIFY_K, ks), (S.PREFIX_V, S.VERIFY_V, vs)):
        if P:
            pre = S.fill_normal(wl.seed, tid_p, (1, 1, 1, P, D), b0=b, l0=l, x0=h * D, head_dim=D,
                                scale=scale, dtype=wl.dtype)[0, 0, 0]
            dst.append(O.to_f64(pre, wl.dtype))
        if R:
            ver = S.fill_normal(wl.seed, tid_v, (R, 1, 1, B1, D), b0=b, l0=l, x0=h * D, head_dim=D,
                                scale=scale, dtype=wl.dtype)[:, 0, 0]
            for r in range(R):
                dst.append(O.to_f64(ver[r, :accepts_b[r] + 1], wl.dtype))
    k = np.concatenate(ks, axis=0) if ks else np.zeros((0, D))
    v = np.concatenate(vs, axis=0) if vs else np.zeros((0, D))
    return k[None, None], v[None, None]


def boundary_hidden(wl, b, l, last_round, a_last):
    """Hidden vector [hidden] of the boundary: verify row a of the last round, or the
    prefill's last hidden when no round ran."""
    if last_round < 0:
        h = S.fill_normal(wl.seed, S.LAST_HIDDEN, (1, 1, 1, 1, wl.hidden), b0=b, l0=l, dtype=wl.dtype)
    else:
        h = S.fill_normal(wl.seed, S.VERIFY_HIDDEN, (1, 1, 1, 1, wl.hidden), r0=last_round, b0=b, l0=l,
                          p0=a_last, dtype=wl.dtype)
    return h.reshape(-1)


def queries(wl, r, b, l, g):
    """Drafter queries of round r for the query heads of KV head g: fp64 [1][B][grp][D]."""
    D, grp = wl.head_dim, wl.group
    q = S.fill_normal(wl.seed, S.QUERY, (1, 1, 1, wl.block, grp * D), r0=r, b0=b, l0=l, x0=g * grp * D,
                      head_dim=D, dtype=wl.dtype)[0, 0, 0]
    return O.to_f64(q, wl.dtype).reshape(1, wl.block, grp, D)


def tile_views(wl, b, l, h, P, accepts_b, scale=None):
    sh = shapes_for_tile(wl)
    k, v = tile_cache(wl, b, l, h, P, accepts_b, scale)
    return sh, O.views_from_scratch(sh, k, v, k.shape[2])


def tile_attend(wl, sh, views, b, l, g, r, hidden_vec, view_set=O.VIEW_ALL):
    """Oracle attention output fp64 [B][grp][D] of tile (b, l, g) with round r's queries,
    over the views in view_set (VIEW_*)."""
    D, H = wl.head_dim, wl.n_kv_heads
    hv = O.to_f64(hidden_vec, wl.dtype)
    bk = hv[g * D:(g + 1) * D].reshape(1, 1, D)
    bv = hv[H * D + g * D:H * D + (g + 1) * D].reshape(1, 1, D)
    q = queries(wl, r, b, l, g)
    return O.draft_attend(sh, views, q, bk, bv, 1.0 / np.sqrt(D), views=view_set)[0]


# ---- comparisons (tolerances as stated for the path) ---------------------------------
SUMMARY_RTOL = 1e-3  # normwise per slot vector
ATTEND_ATOL = 1e-2   # max absolute, for every output dtype (a bf16 output's rounding included)

# largest max |gpu - oracle| of the attention seen per test (printed at the end of a run)
ATTEND_MAX_ERR: dict = {}


def attend_error_excess(got, ref):
    """max |got - ref| - 1e-2: <= 0 when the attention output is within tolerance. The
    bound is flat: a bf16 output's own rounding (at most 2^-8 |out|) has to fit in it."""
    err = float(np.max(np.abs(np.asarray(got, np.float64) - ref))) if np.size(ref) else 0.0
    key = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0] or "?"
    ATTEND_MAX_ERR[key] = max(ATTEND_MAX_ERR.get(key, 0.0), err)
    return err - ATTEND_ATOL


def gpu_f64(x, dtype):
    return O.to_f64(x, dtype)


def normwise(gpu, ref):
    num = np.linalg.norm(np.asarray(gpu, np.float64) - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def f32_to_bf16_bits(x):
    return S.f32_to_bf16_bits(np.asarray(x, np.float32))


def assert_mean_row(mirror, mean, dtype, where):
    """A partial / global mean row (the attention's copy) against the mean of the device's
    own fp32 sum: within one rounding of the row's type plus fp32 reciprocal rounding."""
    got = gpu_f64(mirror, dtype)
    rel = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -21
    assert np.all(np.abs(got - mean) <= rel * np.abs(mean) + 1e-30), where


def check_tile_state(wl, st, b, l, h, views):
    """Asserts the device state of tile (b, l, h) against the oracle views."""
    sh = shapes_for_tile(wl)
    nsc = len(wl.scales)
    n = views.length
    cnt = st["counters"][b, l]
    assert int(cnt[0]) == n, (b, l, int(cnt[0]), n)
    for k in range(nsc):
        assert int(cnt[1 + k]) == views.n_seg[k], (b, l, k, int(cnt[1 + k]), views.n_seg[k])
    kv = st["kv"][b, l, h]
    W, D = wl.window, wl.head_dim
    # ring window: bit-exact
    for t, ring in ((0, views.ring_k), (1, views.ring_v)):
        got = gpu_f64(kv[t, :W], wl.dtype)
        assert np.array_equal(got, ring[0, 0]), (b, l, h, t, "ring")
    for k in range(nsc):
        filled = min(views.n_seg[k], wl.slots)
        for t, seg in ((0, views.seg_k[k]), (1, views.seg_v[k])):
            g = st["seg"][b, l, h, k, :filled, t]
            err = normwise(g, seg[0, 0, :filled])
            assert np.all(err <= SUMMARY_RTOL), (b, l, h, k, t, "seg", float(err.max()))
            # the attention's copy is the rounding of the fp32 mean
            mirror = kv[t, W + k * (wl.slots + 1):W + k * (wl.slots + 1) + filled]
            want = g if wl.dtype == "f32" else f32_to_bf16_bits(g)
            assert np.array_equal(mirror, want), (b, l, h, k, t, "seg mirror")
        c = views.part_count[k]
        for t, part in ((0, views.part_k[k]), (1, views.part_v[k])):
            g = st["part"][b, l, h, k, t]
            if c == 0:
                assert np.all(g == 0), (b, l, h, k, t, "empty partial")
            else:
                err = normwise(g, part[0, 0])
                assert err <= SUMMARY_RTOL, (b, l, h, k, t, "part", float(err))
            mean = np.zeros_like(g, dtype=np.float64) if c == 0 else g.astype(np.float64) / c
            mirror = kv[t, W + k * (wl.slots + 1) + wl.slots]
            assert_mean_row(mirror, mean, wl.dtype, (b, l, h, k, t, "partial mirror"))
    for t, glob in ((0, views.glob_k), (1, views.glob_v)):
        g = st["glob"][b, l, h, t]
        if n:
            err = normwise(g, glob[0, 0])
            assert err <= SUMMARY_RTOL, (b, l, h, t, "glob", float(err))
            mirror = kv[t, -1]
            assert_mean_row(mirror, g.astype(np.float64) / n, wl.dtype, (b, l, h, t, "global mirror"))
        else:
            assert np.all(g == 0)


def slice_views(views, l, h):
    """The views of one (layer, KV head) tile out of a multi-tile oracle state."""
    sl = lambda a: a[l:l + 1, h:h + 1].copy()  # noqa: E731
    return O.Views(
        length=views.length, ring_k=sl(views.ring_k), ring_v=sl(views.ring_v),
        seg_k=[sl(a) for a in views.seg_k], seg_v=[sl(a) for a in views.seg_v],
        n_seg=list(views.n_seg), part_k=[sl(a) for a in views.part_k],
        part_v=[sl(a) for a in views.part_v], part_count=list(views.part_count),
        glob_k=sl(views.glob_k), glob_v=sl(views.glob_v), boundary=views.boundary[l:l + 1].copy())
