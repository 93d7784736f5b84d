"""World-size-2 gloo run of the bench's multi-rank host logic on CPU.

The path shards with no data-path collective: every rank owns a disjoint batch (weak
scaling) or a disjoint share of every sequence's KV heads (strong scaling); the only
collective is the max over ranks of the timed region.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, _ = bench.dist_env()
    off = bench.sequence_offset(r, 16)
    heads = bench.kv_head_range(r, w, 8)
    t = bench.max_over_ranks(1.0 + r, w, torch.device("cpu"))
    bench.barrier(w)
    # the job's rate: 20 rounds per rank, rank r's timed region 0.5 (r + 1) s
    tr = bench.max_over_ranks(0.5 * (r + 1), w, torch.device("cpu"))
    rates = (bench.job_rate(20, tr, w, False), bench.job_rate(20, tr, w, True))
    q.put((r, off, heads, t, rates))
    dist.destroy_process_group()


def test_two_ranks_shard_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o for _, o, _, _, _ in res] == [0, 16]            # disjoint sequence ranges
    assert [h for _, _, h, _, _ in res] == [(0, 4), (4, 8)]   # or disjoint KV-head ranges covering all
    assert all(t == 2.0 for _, _, _, t, _ in res)              # every rank sees the slowest rank's time
    # weak scaling: both ranks' 20 rounds over the slowest rank's 1.0 s; strong: the batch's 20
    assert all(rt == (40.0, 20.0) for _, _, _, _, rt in res)


def test_kv_head_ranges():
    for world in (1, 2, 4, 8):
        got = [bench.kv_head_range(r, world, 8) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == 8
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
    with pytest.raises(ValueError):
        bench.kv_head_range(0, 3, 8)


def test_reference_arm_other_ranks_exit(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0


def test_reference_arm_line(monkeypatch, capsys):
    """Rank 0 of the reference arm times the oracle on the host and prints one JSON line
    with the contract's fields (the oracle's bounded sample, its core count, e2e)."""
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    lines = [x for x in capsys.readouterr().out.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "rounds/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["metric"] == bench.METRIC
    # whole rounds on every host core, and the same config dict the GPU arm prints
    assert d["cpu_baseline"]["cores"] == min(bench.host_cores(), 64)
    assert d["cpu_baseline"]["one_core"]["cores"] == 1 and d["cpu_baseline"]["one_core"]["value"] > 0
    from synth.workloads import CONFIGS
    assert d["config"] == bench.workload_config(CONFIGS[bench.WORKLOAD])


def test_reference_arm_does_not_load_the_library():
    """The oracle's timing runs in processes that never map the CUDA library."""
    import subprocess
    import sys
    code = ("import sys; sys.argv = ['bench.py']; import bench; "
            "assert bench.main(['--impl', 'reference', '--steps', '1', '--warmup', '3']) == 0; "
            "maps = open('/proc/self/maps').read(); "
            "assert 'liblongspark' not in maps and 'fixed_cost_drafter_b200' not in sys.modules, 'library loaded'")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
