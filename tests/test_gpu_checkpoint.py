"""Checkpoint and resume: the whole drafting state is the fixed-size arena, so a snapshot
is a device-to-device copy of it and a restore is the copy back (into the same state or
into a fresh one). The rounds that follow a restore must give bit-identical state,
accepted counts, next tokens and attention outputs.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


def _wl():
    return WL.Workload("ckpt", 31, 3, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16", (300, 1400), 12, None,
                       1000, head_scale=True)


def _rounds(run, inp, r0, r1):
    outs, accs, nxts = [], [], []
    out = run.new_out()
    for r in range(r0, r1):
        run.round(inp, r, out)
        torch.cuda.synchronize()
        outs.append(out.clone())
        accs.append(run.accept_len.clone())
        nxts.append(run.next_token.clone())
    return outs, accs, nxts


def _same(a, b):
    for x, y in zip(a, b):
        for u, v in zip(x, y):
            assert torch.equal(u, v)


def test_snapshot_restore_same_state():
    wl = _wl()
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    _rounds(run, inp, 0, 5)
    snap = run.arena.clone()  # checkpoint: one device-to-device copy of the arena
    first = _rounds(run, inp, 5, wl.rounds)
    after_first = run.read_state()
    run.arena.copy_(snap)  # restore
    again = _rounds(run, inp, 5, wl.rounds)
    _same(first, again)
    for k, v in run.read_state().items():
        assert np.array_equal(v, after_first[k]), k
    assert run.error() == (F.LS_OK, 0)


def test_resume_into_a_fresh_state():
    """A state created anew (ls_init_state zeroes its arena) that receives the snapshot
    continues exactly like the state the snapshot was taken from."""
    wl = _wl()
    a = WL.DeviceRun(wl)
    a.prefill()
    inp = a.make_round_inputs()
    _rounds(a, inp, 0, 7)
    snap = a.arena.clone()
    host = snap.cpu()  # e.g. written to disk between processes
    first = _rounds(a, inp, 7, wl.rounds)
    b = WL.DeviceRun(wl)
    b.arena.copy_(host.to(b.arena.device))
    torch.cuda.synchronize()
    again = _rounds(b, inp, 7, wl.rounds)
    _same(first, again)
    sa, sb = a.read_state(), b.read_state()
    for k in sa:
        assert np.array_equal(sa[k], sb[k]), k
    assert a.error() == (F.LS_OK, 0) and b.error() == (F.LS_OK, 0)
