"""ls_round (commit + attention in one call) against the two-call path and the oracle.

Where the tcgen05 kernel applies, ls_round launches the attention kernel as a programmatic
dependent of the commit kernel (scheduled while the commit runs, waiting on the device for
its writes); the state it leaves and its outputs must be bit-identical to
ls_commit_round followed by ls_draft_attend.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from tests import oracle_side as OS  # noqa: E402

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


@pytest.mark.parametrize("case", ["mid_ragged", "qwen3_8b_shapes", "multi_crossing"])
def test_round_equals_two_calls(case):
    from dataclasses import replace
    if case == "qwen3_8b_shapes":
        wl = replace(WL.CONFIGS["qwen3_8b_64k"], prefix=8192, rounds=6)
        acc = None
    else:
        wl = WL.Workload("round_mid", 11, 3, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16",
                         (300, 1400) if case == "mid_ragged" else 253, 9, None, 1000, head_scale=True)
        acc = None if case == "mid_ragged" else [16] * 9
    one_call = WL.DeviceRun(wl, accepts_override=acc)
    split = WL.DeviceRun(wl, accepts_override=acc)
    assert F.ls_round_overlaps(one_call.state)
    one_call.prefill()
    split.prefill()
    inp = one_call.make_round_inputs()
    out_1, out_s = one_call.new_out(), split.new_out()
    for r in range(one_call.rounds):
        one_call.round(inp, r, out_1)
        split.commit(inp, r)
        split.attend(inp, r, out_s)
        torch.cuda.synchronize()
        assert torch.equal(one_call.accept_len, split.accept_len)
        assert torch.equal(one_call.next_token, split.next_token)
        assert torch.equal(out_1, out_s), r
    sf, ss = one_call.read_state(), split.read_state()
    for key in sf:
        assert np.array_equal(sf[key], ss[key]), key
    assert one_call.error() == (F.LS_OK, 0)


def test_round_matches_oracle():
    wl = WL.Workload("round_oracle", 12, 3, 2, 2, 8, 128, 512, 16, 128, (32, 64, 256), 4, "bf16", (200, 900),
                     7, None, 1000, head_scale=True, flags=F.LS_FLAG_OUT_F32)
    run = WL.DeviceRun(wl)
    run.prefill()
    inp = run.make_round_inputs()
    out = run.new_out()
    for r in range(wl.rounds):
        run.round(inp, r, out)
    torch.cuda.synchronize()
    st = run.read_state()
    acc = OS.accepts_from_ids(run.draft.cpu().numpy(), run.target.cpu().numpy())
    for b in range(wl.batch):
        for l in range(wl.n_layers):
            for h in range(wl.n_kv_heads):
                sh, views = OS.tile_views(wl, b, l, h, int(run.prefix_len[b]), acc[:, b], run.scale_host)
                OS.check_tile_state(wl, st, b, l, h, views)
                hid = OS.boundary_hidden(wl, b, l, wl.rounds - 1, int(acc[-1, b]))
                ref = OS.tile_attend(wl, sh, views, b, l, h, wl.rounds - 1, hid)
                o = out[b, l].view(wl.block, wl.n_q_heads, wl.head_dim)[:, h * wl.group:(h + 1) * wl.group]
                got = o.float().cpu().numpy().astype(np.float64)
                assert OS.attend_error_excess(got, ref) <= 0


def test_round_fallback_equals_two_calls():
    """Shapes the tcgen05 kernel does not take (fp32, GQA x B != 64): ls_round makes the two calls."""
    wl = WL.CONFIGS["tiny"]
    one_call = WL.DeviceRun(wl)
    split = WL.DeviceRun(wl)
    assert not F.ls_round_overlaps(one_call.state)
    one_call.prefill()
    split.prefill()
    inp = one_call.make_round_inputs()
    out_1, out_s = one_call.new_out(), split.new_out()
    for r in range(wl.rounds):
        one_call.round(inp, r, out_1)
        split.commit(inp, r)
        split.attend(inp, r, out_s)
    torch.cuda.synchronize()
    assert torch.equal(out_1, out_s)
    sf, ss = one_call.read_state(), split.read_state()
    for key in sf:
        assert np.array_equal(sf[key], ss[key]), key


def test_round_rejects_bad_offsets():
    wl = WL.CONFIGS["tiny"]
    run = WL.DeviceRun(wl)
    inp = run.make_round_inputs(0, 1)
    out = run.new_out()
    with pytest.raises(F.LsError) as e:
        F.ls_round(run.state, run.draft[0], run.target[0], inp["vk"][0], inp["vv"][0], inp["vh"][0],
                   run.accept_len, run.next_token, inp["q"][0], 4, 128, 0.125, out)
    assert e.value.status == F.LS_ERR_SHAPE
