"""GPU checks of the generator twin and of the device error word (no fault is caused)."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import synth as S  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_device_generator_matches_host(dtype):
    shape = (3, 2, 2, 33, 256)  # r, b, l, p, x (x = 2 heads x 128)
    scale = S.head_scales(9, 4, 8)
    sdev = torch.from_numpy(scale).cuda()
    for tid, hd, use_scale, off in [(S.PREFIX_K, 128, True, dict(r0=0, b0=3, l0=1, p0=1000)),
                                    (S.VERIFY_V, 128, False, dict(r0=17, b0=0, l0=2, p0=0)),
                                    (S.VERIFY_HIDDEN, 0, False, dict(r0=5, b0=1, l0=0, p0=3)),
                                    # a column block starting at KV head 6 (a KV-head shard)
                                    (S.PREFIX_V, 128, True, dict(r0=0, b0=2, l0=2, p0=77, x0=768))]:
        t = torch.empty(int(np.prod(shape)), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                        device="cuda")
        S.device_fill_normal(t.data_ptr(), 9, tid, shape, head_dim=hd,
                             scale_ptr=sdev.data_ptr() if use_scale else None, scale_heads=8, dtype=dtype,
                             stream=torch.cuda.current_stream().cuda_stream, scale_layers=4, **off)
        torch.cuda.synchronize()
        host = S.fill_normal(9, tid, shape, head_dim=hd, scale=scale if use_scale else None, dtype=dtype,
                             **off).reshape(-1)
        got = t.view(torch.int16).cpu().numpy().view(np.uint16) if dtype == "bf16" else t.cpu().numpy()
        assert np.array_equal(got, host)


def test_negative_prefix_length_sets_error_word():
    wl = WL.Workload("neg", 0, 2, 1, 2, 4, 64, 256, 4, 32, (8, 32, 128), 4, "f32", 64, 1, None, 1000)
    run = WL.DeviceRun(wl, prefix_override=[64, -5])
    run.prefill()
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_PREFIX_LEN


def test_out_of_order_chunk_sets_error_word():
    wl = WL.Workload("order", 0, 1, 1, 2, 4, 64, 256, 4, 32, (8, 32, 128), 4, "f32", 512, 1, None, 1000)
    run = WL.DeviceRun(wl)
    plen = torch.tensor([512], dtype=torch.int64, device="cuda")
    k = torch.zeros((1, 1, 128, 128), dtype=torch.float32, device="cuda")
    wsb = F.ls_prefill_workspace_bytes(run.cfg, 128, 256)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    # the state holds 0 rows, so a chunk starting at row 128 does not continue it
    F.ls_prefill_summary(run.state, k, k, 128 * 128, 128, plen, 128, 256, None, ws, wsb)
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE and word & F.LS_DEVERR_ORDER


def test_host_validation_rejects_bad_calls():
    wl = WL.CONFIGS["tiny"]
    run = WL.DeviceRun(wl)
    with pytest.raises(F.LsError) as e:
        F.ls_draft_attend(run.state, 0, 2, run.arena, run.boundary_k, run.boundary_v, wl.hidden, 0.1,
                          run.arena)
    assert e.value.status == F.LS_ERR_INVALID_ARG
    with pytest.raises(F.LsError) as e:
        F.ls_prefill_summary(run.state, run.arena, run.arena, 0, 128, run.accept_len, 5, 10, None,
                             run.arena, 1 << 20)
    assert e.value.status == F.LS_ERR_SHAPE  # row_begin not a multiple of the largest scale


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """Failure detection on the device, without a fault: a wait that nothing signals gives
    up after its poll limit, the host reads LS_ERR_DEVICE_TIMEOUT, and after clearing the
    error word the same state runs prefill and rounds normally."""
    wl = WL.Workload("waitcheck", 41, 2, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16", (300, 700), 3, None,
                     1000, head_scale=True)
    run = WL.DeviceRun(wl)
    F.ls_check_wait_timeout(run.state, 1000, run.stream)
    status, word = run.error()
    assert status == F.LS_ERR_DEVICE_TIMEOUT and word == F.LS_DEVERR_WAIT_TIMEOUT
    F.ls_clear_error(run.state, run.stream)
    assert run.error() == (F.LS_OK, 0)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    for r in range(wl.rounds):
        run.round(inp, r, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert run.error() == (F.LS_OK, 0)
    with pytest.raises(F.LsError):
        F.ls_check_wait_timeout(run.state, 0, run.stream)


def test_clear_error_resets_left_over_arrival_counts():
    """Arrival counts a call that gave up part-way could leave (planted here by hand in the
    arena) are zeroed by ls_clear_error: rounds and the projections then give exactly what
    a clean state gives."""
    wl = WL.Workload("clear", 43, 3, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16", (300, 900), 4, None,
                     1000, head_scale=True)
    clean, dirty = WL.DeviceRun(wl), WL.DeviceRun(wl)
    for run in (clean, dirty):
        run.prefill()
    y = dirty.layout
    b, L = wl.batch, wl.n_layers
    dirty.arena[y.off_sync:y.off_sync + b * L * 4] = 1                      # commit arrivals
    dirty.arena[y.off_sample:y.off_sample + b * 4] = 2                      # sampler arrivals
    cnt = y.off_prologue + 320 * 128 * 16 * 4                               # after the partial-sum slots
    dirty.arena[cnt:cnt + 160 * 4] = 3                                      # projections' tile arrivals
    F.ls_clear_error(dirty.state, dirty.stream)
    inp = clean.make_round_inputs()
    outs = [clean.new_out(), dirty.new_out()]
    for r in range(wl.rounds):
        for run, out in zip((clean, dirty), outs):
            run.round(inp, r, out)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]) and torch.equal(clean.accept_len, dirty.accept_len)
    g = torch.Generator(device="cuda").manual_seed(5)
    w_kv = (torch.randn((L, 2 * 2 * 128, 512), device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    w_q = (torch.randn((L, 8 * 128, 512), device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    x = torch.randn((b, L, 16, 512), device="cuda", generator=g).to(torch.bfloat16)
    res = []
    for run in (clean, dirty):
        bkv = torch.empty((b, L, 512), dtype=torch.bfloat16, device="cuda")
        q = torch.empty((b, L, 16, 1024), dtype=torch.bfloat16, device="cuda")
        F.ls_draft_prologue(run.state, w_kv, w_q, x, bkv, q, run.stream)
        res.append((bkv, q))
    torch.cuda.synchronize()
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    sc, sd = clean.read_state(), dirty.read_state()
    for k in sc:
        assert np.array_equal(sc[k], sd[k]), k
    assert clean.error() == (F.LS_OK, 0) and dirty.error() == (F.LS_OK, 0)
