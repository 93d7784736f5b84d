"""Prefill and commit reading the target's paged KV cache in place (block table, pages
scattered over the pool) against the dense path and the oracle's paged reading.

The paged calls do the same arithmetic in the same order as the dense ones (only where
the rows are loaded from changes), so their state, accepted counts, next tokens and
attention outputs must be bit-identical; the oracle check takes the pages themselves to
the host and runs the oracle's paged prefill / commit over them.
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


def _wl(**kw):
    base = dict(name="paged", seed=21, batch=3, n_layers=2, n_kv_heads=2, n_q_heads=8, head_dim=128, hidden=512,
                block=16, window=128, scales=(32, 64, 256), slots=4, dtype="bf16", prefix=(300, 1400), rounds=9,
                accept_mean=None, vocab=1000, head_scale=True)
    base.update(kw)
    return WL.Workload(**base)


def _capacity(run):
    wl = run.wl
    return run.prefix_len + (run.rounds + 1) * (wl.block + 1)


def _same_state(a, b):
    sa, sb = a.read_state(), b.read_state()
    for key in sa:
        assert np.array_equal(sa[key], sb[key]), key


def _pair(wl, page_size, layout, chunk=None, seed=0):
    dense = WL.DeviceRun(wl, prefill_chunk=chunk)
    paged = WL.DeviceRun(wl, prefill_chunk=chunk)
    cache = WL.PagedCache(paged, page_size, _capacity(paged), layout=layout, seed=seed)
    paged.fill_pages(cache)
    dense.prefill()
    paged.prefill_paged(cache)
    torch.cuda.synchronize()
    return dense, paged, cache


@pytest.mark.parametrize("page_size,layout,chunk", [(16, "packed", None), (1, "packed", None),
                                                    (48, "interleaved", None), (256, "padded", None),
                                                    (64, "packed", 512)])
def test_paged_prefill_and_commits_match_dense(page_size, layout, chunk):
    wl = _wl()
    dense, paged, cache = _pair(wl, page_size, layout, chunk, seed=page_size)
    _same_state(dense, paged)
    inp = dense.make_round_inputs()
    for r in range(dense.rounds):
        paged.write_verify_pages(cache, inp, r)
        dense.commit(inp, r)
        paged.commit_paged(cache, inp, r)
        torch.cuda.synchronize()
        assert torch.equal(dense.accept_len, paged.accept_len) and torch.equal(dense.next_token, paged.next_token)
    _same_state(dense, paged)
    # and against the oracle's views of the same synthetic rows
    st = paged.read_state()
    acc = OS.accepts_from_ids(dense.draft.cpu().numpy(), dense.target.cpu().numpy())
    for b, l, g in [(0, 0, 0), (wl.batch - 1, wl.n_layers - 1, wl.n_kv_heads - 1), (1, 1, 0)]:
        _, views = OS.tile_views(wl, b, l, g, int(paged.prefix_len[b]), acc[:, b], paged.scale_host)
        OS.check_tile_state(wl, st, b, l, g, views)
    assert paged.error() == (F.LS_OK, 0) and dense.error() == (F.LS_OK, 0)


@pytest.mark.parametrize("page_size,layout", [(16, "packed"), (48, "interleaved")])
def test_paged_commit_with_slot_mapping(page_size, layout):
    """The commit reading the verify rows at the slots the verify pass wrote (an engine's
    slot mapping) instead of through the block table: same state as the dense path."""
    wl = _wl()
    dense, paged, cache = _pair(wl, page_size, layout, seed=page_size + 1)
    inp = dense.make_round_inputs()
    for r in range(dense.rounds):
        paged.write_verify_pages(cache, inp, r)
        dense.commit(inp, r)
        paged.commit_paged(cache, inp, r, with_slots=True)
        torch.cuda.synchronize()
        assert torch.equal(dense.accept_len, paged.accept_len) and torch.equal(dense.next_token, paged.next_token)
    _same_state(dense, paged)
    assert paged.error() == (F.LS_OK, 0)


def test_paged_bad_slot_is_flagged():
    wl = _wl(rounds=1)
    run = WL.DeviceRun(wl)
    cache = WL.PagedCache(run, 16, _capacity(run), seed=12)
    run.fill_pages(cache)
    run.prefill_paged(cache)
    inp = run.make_round_inputs()
    run.write_verify_pages(cache, inp, 0)
    run.verify_slots[0][1, 0] = cache.num_pages * cache.page_size  # one slot past the pool
    run.commit_paged(cache, inp, 0, with_slots=True)
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_PAGE


def _pages_f64(t, H, D):
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return O.to_f64(bits, "bf16").reshape(t.shape[0], t.shape[1], H, D)


def test_paged_against_the_oracle_reading():
    """The oracle's prefill_paged / commit_round_paged over the device's own pages and
    block table (copied to the host), every tile."""
    wl = _wl(batch=2, prefix=(200, 700), rounds=5, scales=(32, 64, 128), slots=3)
    run = WL.DeviceRun(wl)
    ps = 16
    cache = WL.PagedCache(run, ps, _capacity(run), layout="interleaved", seed=3)
    run.fill_pages(cache)
    run.prefill_paged(cache)
    inp = run.make_round_inputs()
    for r in range(run.rounds):
        run.write_verify_pages(cache, inp, r)
    for r in range(run.rounds):
        run.commit_paged(cache, inp, r)
    torch.cuda.synchronize()
    L, H, D = wl.n_layers, wl.n_kv_heads, wl.head_dim
    sh = O.Shapes(n_layers=L, n_kv_heads=H, n_q_heads=wl.n_q_heads, head_dim=D, hidden=wl.hidden, block=wl.block,
                  window=wl.window, scales=wl.scales, slots=wl.slots)
    kp = np.stack([_pages_f64(cache.k[l], H, D) for l in range(L)])
    vp = np.stack([_pages_f64(cache.v[l], H, D) for l in range(L)])
    hid = O.to_f64(run.last_hidden.view(torch.int16).cpu().numpy().view(np.uint16), "bf16")
    vh = O.to_f64(inp["vh"].view(torch.int16).cpu().numpy().view(np.uint16), "bf16")
    draft, target = run.draft.cpu().numpy(), run.target.cpu().numpy()
    st = run.read_state()
    for b in range(wl.batch):
        v = O.prefill_paged(sh, kp, vp, cache.table_host, ps, b, int(run.prefix_len[b]), hid[b])
        for r in range(run.rounds):
            O.commit_round_paged(sh, v, draft[r, b], target[r, b], kp, vp, cache.table_host, ps, b, vh[r, b])
        for l in range(L):
            for g in range(H):
                OS.check_tile_state(wl, st, b, l, g, OS.slice_views(v, l, g))
        np.testing.assert_array_equal(O.to_f64(st["boundary"][b], "bf16"), v.boundary)
    assert run.error() == (F.LS_OK, 0)


def test_paged_round_and_given_counts():
    """ls_round_paged equals ls_round; ls_commit_accepted_paged equals ls_commit_accepted."""
    wl = _wl(rounds=6)
    dense, paged, cache = _pair(wl, 32, "packed", seed=5)
    given = WL.DeviceRun(wl)
    gcache = WL.PagedCache(given, 32, _capacity(given), layout="padded", seed=6)
    given.fill_pages(gcache)
    given.prefill_paged(gcache, workspace=False)  # the library's fixed scratch
    inp = dense.make_round_inputs()
    out_d, out_p = dense.new_out(), paged.new_out()
    for r in range(dense.rounds):
        paged.write_verify_pages(cache, inp, r)
        given.write_verify_pages(gcache, inp, r)
        dense.round(inp, r, out_d)
        F.ls_round_paged(paged.state, paged.draft[r], paged.target[r], cache.descriptor(), inp["vh"][r],
                         paged.accept_len, paged.next_token, inp["q"][r], 0, wl.n_kv_heads * wl.head_dim,
                         paged.softmax_scale, out_p, paged.stream)
        torch.cuda.synchronize()
        F.ls_commit_accepted_paged(given.state, dense.accept_len.clone(), gcache.descriptor(), inp["vh"][r],
                                   given.stream)
        torch.cuda.synchronize()
        assert torch.equal(out_d, out_p), r
        assert torch.equal(dense.accept_len, paged.accept_len) and torch.equal(dense.next_token, paged.next_token)
    _same_state(dense, paged)
    _same_state(dense, given)
    for run in (dense, paged, given):
        assert run.error() == (F.LS_OK, 0)


def test_paged_empty_and_short_prefixes():
    """Prefix lengths 0, 1 and one page exactly: nothing read for the empty sequence."""
    wl = _wl(rounds=3)
    dense = WL.DeviceRun(wl, prefix_override=[0, 1, 16])
    paged = WL.DeviceRun(wl, prefix_override=[0, 1, 16])
    cache = WL.PagedCache(paged, 16, _capacity(paged), seed=8)
    paged.fill_pages(cache)
    dense.prefill()
    paged.prefill_paged(cache)
    inp = dense.make_round_inputs()
    for r in range(dense.rounds):
        paged.write_verify_pages(cache, inp, r)
        dense.commit(inp, r)
        paged.commit_paged(cache, inp, r)
    torch.cuda.synchronize()
    _same_state(dense, paged)
    assert paged.error() == (F.LS_OK, 0)


def test_paged_bad_pages_are_flagged():
    """A page id outside the pool and a prefix longer than the block table: the kernels
    read page 0 in their place and set LS_DEVERR_PAGE (no access leaves the pool)."""
    wl = _wl(rounds=1)
    run = WL.DeviceRun(wl)
    cache = WL.PagedCache(run, 16, _capacity(run), seed=9)
    run.fill_pages(cache)
    table = cache.table_host.copy()
    table[1, 3] = cache.num_pages  # one prefix page of sequence 1 out of range
    cache.block_table.copy_(torch.from_numpy(table))
    run.prefill_paged(cache)
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_PAGE

    run2 = WL.DeviceRun(wl)
    short = WL.PagedCache(run2, 16, run2.prefix_len - 40, seed=10)  # the table ends before the prefix does
    run2.prefill_paged(short)
    status, word = run2.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_PAGE


def test_paged_host_checks():
    wl = _wl(rounds=1)
    run = WL.DeviceRun(wl)
    cache = WL.PagedCache(run, 16, _capacity(run), seed=11)
    plen = torch.from_numpy(run.prefix_len).to(run.dev)
    good = cache.descriptor()

    def variant(**kw):
        kv = F.ls_paged_kv.from_buffer_copy(good)
        for k, v in kw.items():
            setattr(kv, k, v)
        return kv

    bad = [variant(slot_stride=wl.n_kv_heads * wl.head_dim - 8), variant(slot_stride=good.slot_stride + 4),
           variant(verify_slots=cache.block_table.data_ptr() + 4),
           variant(page_size=0), variant(num_pages=0), variant(max_blocks=0), variant(block_table=None)]
    k1 = variant()
    k1.k_layers[1] = None
    bad.append(k1)
    k2 = variant()
    k2.v_layers[0] = good.v_layers[0] + 8
    bad.append(k2)
    vh = torch.zeros((wl.batch, wl.n_layers, wl.block + 1, wl.hidden), dtype=torch.bfloat16, device=run.dev)
    for kv in bad:
        with pytest.raises(F.LsError):
            F.ls_prefill_paged(run.state, kv, plen, 0, 256, None, None, 0, run.stream)
        with pytest.raises(F.LsError):
            F.ls_commit_round_paged(run.state, run.draft[0], run.target[0], kv, vh, run.accept_len, run.next_token,
                                    run.stream)
    assert run.error() == (F.LS_OK, 0)


def test_paged_fp32_tiny_round_matches_dense():
    """The fp32 instantiations (4-byte rows) and ls_round_paged on the CUDA-core attention:
    the tiny fp32 config with a page size of 5 (not a power of two) and keys and values
    interleaved per page, against ls_round on the dense rows, bit for bit."""
    wl = WL.CONFIGS["tiny"]
    dense = WL.DeviceRun(wl)
    paged = WL.DeviceRun(wl)
    cache = WL.PagedCache(paged, 5, _capacity(paged), layout="interleaved", seed=13)
    paged.fill_pages(cache)
    dense.prefill()
    paged.prefill_paged(cache)
    torch.cuda.synchronize()
    _same_state(dense, paged)
    inp = dense.make_round_inputs()
    out_d, out_p = dense.new_out(), paged.new_out()
    for r in range(dense.rounds):
        paged.write_verify_pages(cache, inp, r)
        dense.round(inp, r, out_d)
        F.ls_round_paged(paged.state, paged.draft[r], paged.target[r],
                         paged.paged_descriptor(cache, r, with_slots=bool(r & 1)), inp["vh"][r],
                         paged.accept_len, paged.next_token, inp["q"][r], paged.bk_off, paged.bv_off,
                         paged.softmax_scale, out_p, paged.stream)
        torch.cuda.synchronize()
        assert torch.equal(out_d, out_p), r
        assert torch.equal(dense.accept_len, paged.accept_len) and torch.equal(dense.next_token, paged.next_token)
    _same_state(dense, paged)
    assert not F.ls_attend_uses_tensor_cores(paged.state)
    assert paged.error() == (F.LS_OK, 0) and dense.error() == (F.LS_OK, 0)
