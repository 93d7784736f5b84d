"""KV-head sharding (the natural split for a tensor-parallel target): KV heads are
independent in the commit and in the attention, so a run holding KV heads h0 .. h1 - 1 of
every sequence (with their query heads, and the replicated boundary hidden vectors) must
give exactly those heads' state and outputs of the whole run. The shards run one after the
other on one GPU here; nothing in them waits on another shard.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WL


@pytest.mark.parametrize("ranges", [[(0, 2), (2, 4)], [(0, 1), (1, 3), (3, 4)]])
def test_kv_head_shards_equal_the_whole(ranges):
    wl = WL.Workload("shard", 51, 3, 2, 4, 16, 128, 1024, 16, 128, (32, 64, 256), 4, "bf16", (300, 1400), 6,
                     None, 1000, head_scale=True)
    whole = WL.DeviceRun(wl)
    whole.prefill()
    inp = whole.make_round_inputs()
    out = whole.new_out()
    shards = [WL.DeviceRun(wl, kv_heads=r) for r in ranges]
    s_inp, s_out = [], []
    for sh in shards:
        sh.prefill()
        s_inp.append(sh.make_round_inputs())
        s_out.append(sh.new_out())
    D, g = wl.head_dim, wl.group
    for r in range(wl.rounds):
        whole.round(inp, r, out)
        for sh, si, so in zip(shards, s_inp, s_out):
            sh.round(si, r, so)
        torch.cuda.synchronize()
        for (h0, h1), sh, so in zip(ranges, shards, s_out):
            assert torch.equal(sh.accept_len, whole.accept_len) and torch.equal(sh.next_token, whole.next_token)
            assert torch.equal(so, out[..., h0 * g * D:h1 * g * D]), (r, h0)
    st = whole.read_state()
    for (h0, h1), sh in zip(ranges, shards):
        ss = sh.read_state()
        assert np.array_equal(ss["counters"], st["counters"])
        assert np.array_equal(ss["boundary"], st["boundary"])
        for key in ("kv", "seg", "part", "glob"):
            assert np.array_equal(ss[key], st[key][:, :, h0:h1]), key
        assert sh.error() == (F.LS_OK, 0)
    assert whole.error() == (F.LS_OK, 0)
