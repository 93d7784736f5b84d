"""Benchmark of the LongSpark drafting round on B200.

One step = one decoding round of the hot path over a batch of 16 sequences at Qwen3-8B
shapes with a 64K-token prefix: ``ls_round``, i.e. the commit (accept scan, ring-window
commit, summary update, boundary gather) and the drafter's block attention over all 4
tapped layers, the attention kernel launched as a programmatic dependent of the commit
kernel. The same round as two plain calls (``ls_commit_round`` then ``ls_draft_attend``,
CUDA events around each) gives the per-kernel times; ``roofline`` is the attention kernel's
(the dominant one) and ``round_roofline`` the whole round's.
The prefill summary over the prefix runs once per request before the rounds; it is timed
separately in the same run and reported under ``prefill``.

Timing: W untimed warm-up rounds, then K timed rounds. Before every round (untimed) a
256 MB buffer is written and a second 256 MB buffer is read, so the round starts with a
cold L2 that holds no dirty lines of the flush (as after the target's verification pass,
whose big reads leave clean lines); each round is bracketed by CUDA events on the
launching stream (a third event splits commit from attention). ``value`` is rounds per second over
all ranks (weak scaling: every rank owns its own batch of 16 sequences).

``--impl reference`` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import glob
import hashlib
import json
import re
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft rounds/s at batch 16 (Qwen3-8B shapes), 32K-128K prefix; % HBM roofline"
WORKLOAD = "qwen3_8b_64k"
FALLBACK_HBM_GBS = 6650.0
LOADED_W = 300.0  # power draw above which a clock sample counts as under load (idle: about 200 W)


# ---------------------------------------------------------------------------------------
# multi-rank plumbing (host logic; covered by CPU gloo tests)
# ---------------------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def sequence_offset(rank: int, batch_per_rank: int) -> int:
    """First global sequence index owned by `rank` (weak scaling: disjoint batches)."""
    return rank * batch_per_rank


def kv_head_range(rank: int, world: int, n_kv_heads: int):
    """KV heads (h0, h1) owned by `rank` when the ranks split every sequence's KV heads
    (the natural split for a tensor-parallel target: heads are independent in the commit
    and the attention, so there is no exchange)."""
    if n_kv_heads % world:
        raise ValueError(f"{n_kv_heads} KV heads do not split evenly over {world} ranks")
    per = n_kv_heads // world
    return rank * per, (rank + 1) * per


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, seconds_max: float, world: int, strong: bool) -> float:
    """Units per second of the whole job over the slowest rank's time: weak scaling (every
    rank its own batch) counts every rank's units, strong scaling (ranks share one batch's
    KV heads) counts the batch's once."""
    return (1 if strong else world) * units_per_rank / seconds_max


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------------------
# algorithmic bytes (the layout built: bf16 window and mean rows, fp32 summary sums)
# ---------------------------------------------------------------------------------------
VIEW_BOUNDARY, VIEW_WINDOW, VIEW_SUMMARY, VIEW_ALL = 0x1, 0x2, 0x4, 0x7  # LS_VIEW_*
LS_FLAG_OUT_F32 = 0x2

# Table 5's component ablations: the views each variant keeps
ABLATIONS = {"full": VIEW_ALL, "without_global_summary": VIEW_BOUNDARY | VIEW_WINDOW,
             "without_boundary_state": VIEW_WINDOW | VIEW_SUMMARY,
             "without_recent_kv_window": VIEW_BOUNDARY | VIEW_SUMMARY}


def attend_bytes(wl, views: int = VIEW_ALL) -> int:
    """Algorithmic bytes of one attention launch over the given views."""
    e = wl.elem()
    e_out = 4 if wl.flags & LS_FLAG_OUT_F32 else e
    b, L, H, Hq, D, B = wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.block
    summary_rows = len(wl.scales) * (wl.slots + 1) + 1
    return (b * L * B * Hq * D * (e + e_out)                                  # Q in, O out
            + (b * L * H * wl.window * 2 * D * e if views & VIEW_WINDOW else 0)  # ring window K/V
            + (b * L * H * summary_rows * 2 * D * e if views & VIEW_SUMMARY else 0)  # summary mean rows
            + (b * L * H * 2 * D * e if views & VIEW_BOUNDARY else 0)          # boundary K/V
            + b * L * (1 + len(wl.scales)) * 8)                                # counters


def commit_bytes(wl, mean_delta: float) -> int:
    e = wl.elem()
    b, L, H, D, nsc = wl.batch, wl.n_layers, wl.n_kv_heads, wl.head_dim, len(wl.scales)
    rows = b * mean_delta * L * H * 2 * D * e
    return int(2 * rows                                          # read retained rows, write ring
               + 2 * b * L * H * (nsc + 1) * 2 * D * 4           # fp32 partial + global RMW
               + b * L * H * 2 * D * (4 + e) * sum(mean_delta / s for s in wl.scales)  # finalised means
               + b * L * H * (nsc + 1) * 2 * D * e               # partial/global mean rows
               + 2 * b * L * wl.hidden * e                       # boundary gather
               + b * (2 * wl.block + 1) * 4 + 8 * b              # token ids, outputs
               + 2 * b * L * (1 + nsc) * 8)                      # counters


def prefill_bytes(wl, prefix_len) -> int:
    return int(np.sum(prefix_len)) * wl.n_layers * wl.n_kv_heads * wl.head_dim * 2 * wl.elem()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed: edits to comments and
    documentation do not change a kernel, so they must not void its recorded counters."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha(name: str) -> str:
    """Hash of the code of a kernel's source file and of the package headers it includes
    (recursively), comments and whitespace left out."""
    csrc = os.path.join(ROOT, "fixed_cost_drafter_b200", "csrc")
    inc = os.path.join(ROOT, "include")
    seen, order, todo = set(), [], [os.path.join(csrc, name)]
    while todo:
        q = todo.pop(0)
        if q in seen:
            continue
        seen.add(q)
        order.append(q)
        with open(q, encoding="utf-8") as f:
            for m in re.finditer(r'^\s*#\s*include\s+"([^"]+)"', f.read(), re.M):
                for d in (os.path.dirname(q), csrc, inc):
                    cand = os.path.join(d, m.group(1))
                    if os.path.exists(cand):
                        todo.append(os.path.normpath(cand))
                        break
    h = hashlib.sha256()
    for q in order:
        with open(q, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str, key: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it matches the source."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)
        ent = rec.get(key)
        if ent and ent.get("source_sha") == kernel_source_sha(kernel_file):
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str, period_ms: int = 100):
        self.path, self.proc, self.gpu, self.period = path, None, gpu_index, period_ms

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self, min_power_w: float = 0.0):
        """Median SM clock, max clock and the throttle reasons seen, over the samples drawn
        at min_power_w or more (the GPU under load)."""
        if self.proc is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    if float(parts[3]) >= min_power_w:
                        rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        if not min_power_w:
            rows = rows[1:] if len(rows) > 1 else rows  # the first sample may precede the load
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, v in enumerate(flags) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------------------
class OracleSlices:
    """The CPU oracle's drafting state for some (sequence, layer) slices of a workload.

    The oracle's views are fixed-size, so its per-round work does not depend on the
    prefix: each slice's views are initialised (untimed) from its first ``prefix_rows``
    prefix rows. ``step(r)`` runs one round on every slice it holds: the commit of the
    retained rows and the attention of all query heads, with the round's own synthetic
    inputs (``n_inputs`` distinct rounds, cycled). A whole round of the workload is every
    (sequence, layer) slice once.
    """

    def __init__(self, wl_name, slices, prefix_rows=4096, n_inputs=4):
        import oracle as O
        import synth as S
        from synth.workloads import CONFIGS
        wl = CONFIGS[wl_name]
        self.O, self.wl, self.slices = O, wl, list(slices)
        H, Hq, D, B = wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.block
        self.sh = O.Shapes(n_layers=1, n_kv_heads=H, n_q_heads=Hq, head_dim=D, hidden=wl.hidden, block=B,
                           window=wl.window, scales=tuple(wl.scales), slots=wl.slots)
        scale = S.head_scales(wl.seed, wl.n_layers, H) if wl.head_scale else None
        P = prefix_rows
        f = lambda tid, shape, **kw: O.to_f64(S.fill_normal(wl.seed, tid, shape, **kw), wl.dtype)  # noqa: E731
        acc = S.accept_lengths(wl.seed, n_inputs, wl.batch, B, wl.accept_mean)
        self.draft, self.target = S.token_ids(wl.seed, n_inputs, wl.batch, B, acc, wl.vocab)
        self.views, self.inputs = [], []
        for b, l in self.slices:
            pk = f(S.PREFIX_K, (1, 1, 1, P, H * D), b0=b, l0=l, head_dim=D, scale=scale)[0, 0]
            pv = f(S.PREFIX_V, (1, 1, 1, P, H * D), b0=b, l0=l, head_dim=D, scale=scale)[0, 0]
            hid = f(S.LAST_HIDDEN, (1, 1, 1, 1, wl.hidden), b0=b, l0=l)[0, 0, :, 0]
            self.views.append(O.prefill(self.sh, pk.reshape(1, P, H, D), pv.reshape(1, P, H, D), P, hid))
            ins = []
            for r in range(n_inputs):
                kw = dict(r0=r, b0=b, l0=l)
                vk = f(S.VERIFY_K, (1, 1, 1, B + 1, H * D), head_dim=D, scale=scale, **kw)[0, 0]
                vv = f(S.VERIFY_V, (1, 1, 1, B + 1, H * D), head_dim=D, scale=scale, **kw)[0, 0]
                vh = f(S.VERIFY_HIDDEN, (1, 1, 1, B + 1, wl.hidden), **kw)[0, 0]
                q = f(S.QUERY, (1, 1, 1, B, Hq * D), head_dim=D, **kw)[0, 0]
                ins.append((vk.reshape(1, B + 1, H, D), vv.reshape(1, B + 1, H, D), vh, q.reshape(1, B, Hq, D)))
            self.inputs.append(ins)
        self.sm = 1.0 / math.sqrt(D)

    def step(self, r: int) -> float:
        """Seconds for round r on every slice held."""
        O, H, D = self.O, self.wl.n_kv_heads, self.wl.head_dim
        t0 = time.perf_counter()
        for (b, _), views, ins in zip(self.slices, self.views, self.inputs):
            k = r % len(ins)
            vk, vv, vh, q = ins[k]
            O.commit_round(self.sh, views, self.draft[k, b], self.target[k, b], vk, vv, vh)
            bk = views.boundary[:, :H * D].reshape(1, H, D)
            bv = views.boundary[:, H * D:2 * H * D].reshape(1, H, D)
            O.draft_attend(self.sh, views, q, bk, bv, self.sm)
        return time.perf_counter() - t0


def _oracle_worker(conn, wl_name, slices, prefix_rows):
    """A worker process: one BLAS thread, its slices' state; steps on request."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        st = OracleSlices(wl_name, slices, prefix_rows)
        conn.send("ready")
        while True:
            r = conn.recv()
            if r is None:
                break
            conn.send(st.step(r))
    conn.close()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleRounds:
    """Whole rounds of the CPU oracle on ``workers`` processes (spawned, one thread each),
    the workload's (sequence, layer) slices dealt round-robin over them. ``round(r)``
    returns the wall time of one whole round, from the request to the last worker's
    answer."""

    def __init__(self, wl_name, workers, prefix_rows=4096):
        import multiprocessing as mp
        from synth.workloads import CONFIGS
        wl = CONFIGS[wl_name]
        all_slices = [(b, l) for b in range(wl.batch) for l in range(wl.n_layers)]
        self.workers = max(1, min(int(workers), len(all_slices)))
        self.n_slices = len(all_slices)
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for w in range(self.workers):
            a, b = ctx.Pipe()
            proc = ctx.Process(target=_oracle_worker, args=(b, wl_name, all_slices[w::self.workers], prefix_rows),
                               daemon=True)
            proc.start()
            self.conns.append(a)
            self.procs.append(proc)
        for c in self.conns:
            if c.recv() != "ready":
                raise RuntimeError("oracle worker failed to start")

    def round(self, r: int):
        """(wall seconds of the whole round, its compute seconds summed over the workers)."""
        t0 = time.perf_counter()
        for c in self.conns:
            c.send(r)
        busy = sum(c.recv() for c in self.conns)
        return time.perf_counter() - t0, busy

    def close(self):
        for c in self.conns:
            c.send(None)
        for p in self.procs:
            p.join(timeout=30)


def oracle_sample_text(wl, workers, rounds, prefix_rows=4096):
    return (f"{rounds} whole rounds of the oracle (commit + attention of all {wl.n_q_heads} query heads for "
            f"every one of the {wl.batch} sequences x {wl.n_layers} tapped layers) on {workers} worker "
            f"processes of one thread each; views initialised from a {prefix_rows}-row prefix (the oracle's "
            f"per-round work does not depend on the prefix)")


def oracle_timing(wl_name, warmup, steps=None, budget_s=None):
    """Whole oracle rounds on every host core: ``warmup`` untimed rounds, then ``steps``
    rounds (or rounds until ``budget_s`` has passed). Returns (wall seconds per round,
    summed worker seconds per round, rounds timed, workers)."""
    pool = OracleRounds(wl_name, host_cores())
    try:
        for i in range(warmup):
            pool.round(i)
        walls, busy = [], []
        t_end = time.perf_counter() + (budget_s or 0.0)
        while (steps is not None and len(walls) < steps) or (steps is None and (time.perf_counter() < t_end
                                                                                  or len(walls) < 2)):
            w, b = pool.round(warmup + len(walls))
            walls.append(w)
            busy.append(b)
    finally:
        pool.close()
    return float(np.mean(walls)), float(np.mean(busy)), len(walls), pool.workers


def cpu_record(wl, per_round, busy, rounds, workers):
    return {"value": 1.0 / per_round, "unit": "rounds/s", "cores": workers, "kind": "oracle",
            "sample": oracle_sample_text(wl, workers, rounds),
            "one_core": {"value": 1.0 / busy, "unit": "rounds/s", "cores": 1,
                         "sample": "the same rounds' compute time summed over the worker processes (each "
                                   "worker times its own slices on its own core, all running at once): "
                                   "a whole round's work at one core's speed"}}


def cpu_baseline(wl, budget_s: float = 15.0):
    """The oracle on the host cores: one untimed round, then whole rounds for about budget_s."""
    per_round, busy, n, workers = oracle_timing(wl.name, 1, budget_s=budget_s)
    return cpu_record(wl, per_round, busy, n, workers)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from dataclasses import replace
    from synth.workloads import CONFIGS
    wl = CONFIGS[args.config]
    if args.out == "f32":  # (the oracle computes in fp64 either way; the config names the GPU's output)
        wl = replace(wl, flags=wl.flags | LS_FLAG_OUT_F32)
    per_round, busy, n, workers = oracle_timing(wl.name, args.warmup, steps=args.steps)
    v = 1.0 / per_round
    line = {"metric": METRIC, "value": v, "unit": "rounds/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_round * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(wl), "parallelism": f"{workers} host processes",
            "cpu_baseline": cpu_record(wl, per_round, busy, n, workers),
            "e2e": {"value": v, "unit": "rounds/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def workload_config(wl):
    return {"workload": f"{wl.name}: batch {wl.batch}, {wl.n_layers} tapped layers, {wl.n_kv_heads} KV / "
                        f"{wl.n_q_heads} query heads, head_dim {wl.head_dim}, hidden {wl.hidden}, B {wl.block}, "
                        f"W {wl.window}, summary scales {'/'.join(map(str, wl.scales))} x {wl.slots} slots + "
                        f"partials + global mean, prefix {wl.prefix}",
            "batch": wl.batch, "prefix": wl.prefix if not isinstance(wl.prefix, tuple) else list(wl.prefix),
            "accept_mean": wl.accept_mean,
            "attention_output": "f32" if wl.flags & LS_FLAG_OUT_F32 else wl.dtype,
            "l2": "flushed before every timed round: 256 MB written then 256 MB read (untimed), "
                  "so the round starts cold with no dirty flush lines to write back"}


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------
def run_gpu(args):
    import torch
    import fixed_cost_drafter_b200 as F
    from fixed_cost_drafter_b200 import workloads as WLM

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from dataclasses import replace
    wl = WLM.CONFIGS[args.config]
    if args.out == "f32":
        wl = replace(wl, flags=wl.flags | F.LS_FLAG_OUT_F32)
    if args.prefix:  # profiling runs: same per-round work, smaller prefix to generate
        wl = replace(wl, prefix=args.prefix)
    K, W = args.steps, args.warmup
    # distinct rounds of generated inputs; the timed loop cycles through them (the state
    # keeps growing, every round re-reads its inputs from HBM after the L2 flush)
    n_rounds = min(K + W, args.distinct_rounds)
    if args.shard == "kv-heads":  # every rank: all sequences, its share of the KV heads
        run = WLM.DeviceRun(wl, device=dev, rounds=n_rounds, kv_heads=kv_head_range(rank, world, wl.n_kv_heads))
    else:  # every rank: its own batch of sequences
        run = WLM.DeviceRun(wl, device=dev, rounds=n_rounds, seq_offset=sequence_offset(rank, wl.batch))
    # from here on `wl` is this rank's part (its KV heads under kv-heads sharding)
    full_wl, wl = wl, run.wl
    strong = args.shard == "kv-heads"

    # prefill (timed separately, after one untimed prefill into a state then reset)
    run.prefill()
    run.reset_state()
    pre = []
    run.prefill(timer=lambda e0, e1, nbytes: pre.append((e0, e1, nbytes)))
    torch.cuda.synchronize()
    prefill_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in pre)
    prefill_b = sum(n for _, _, n in pre)

    inp = run.make_round_inputs(0, n_rounds)
    out = run.new_out()
    flush = L2Flush(dev)
    stream = run.stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]

    clock_path = (args.clock_log or os.path.join(ROOT, "_build", "clocks_rank{rank}.csv")).format(rank=rank)
    os.makedirs(os.path.dirname(clock_path), exist_ok=True)
    overlapped = F.ls_round_overlaps(run.state)
    # clocks over the whole GPU part of the run (20 ms samples; the timed rounds last a few
    # ms only), and over the warm-up and timed rounds alone
    run_clk = ClockSampler(local, clock_path.replace(".csv", "_run.csv"), period_ms=20)
    run_clk.__enter__()
    import atexit
    atexit.register(run_clk.__exit__)  # (also on an error before the end)
    # the sampler starts with the warm-up rounds so that its samples cover a loaded GPU
    with ClockSampler(local, clock_path) as clk:
        for r in range(W):
            flush.zero_()
            run.round(inp, r % n_rounds, out)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        for i in range(K):
            r = (W + i) % n_rounds
            flush.zero_()
            evs[i][0].record(stream)
            run.round(inp, r, out)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    round_ms = [e[0].elapsed_time(e[1]) for e in evs]
    total_s = sum(round_ms) / 1e3
    # the same round as two calls, for the per-kernel split
    KS = min(K, 500)
    for i in range(KS):
        r = (W + K + i) % n_rounds
        flush.zero_()
        evs[i][0].record(stream)
        run.commit(inp, r)
        evs[i][1].record(stream)
        run.attend(inp, r, out)
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    commit_ms = [e[0].elapsed_time(e[1]) for e in evs[:KS]]
    attend_ms = [e[1].elapsed_time(e[2]) for e in evs[:KS]]

    # the attention launched back to back (no flush: the 213 MB state read is larger than
    # L2, so every launch still streams it from HBM; each launch's latency overlaps the one
    # before it)
    KB = min(K, 200)
    e_b0, e_b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run.attend(inp, W % n_rounds, out)
    e_b0.record(stream)
    for i in range(KB):
        run.attend(inp, (W + i) % n_rounds, out)
    e_b1.record(stream)
    torch.cuda.synchronize()
    attend_b2b_s = e_b0.elapsed_time(e_b1) / 1e3 / KB

    total_max = max_over_ranks(total_s, world, dev)
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} after the timed rounds")

    # the cost side of Table 5's component ablations: the attention over fewer views
    ablations = None
    if not args.no_ablations:
        KA = min(K, 200)
        ablations = {}
        for name, views in ABLATIONS.items():
            ms = []
            for i in range(KA):
                r = (W + i) % n_rounds
                flush.zero_()
                evs[i][0].record(stream)
                run.attend(inp, r, out, views=views)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            ms = [e[0].elapsed_time(e[1]) for e in evs[:KA]]
            us = float(np.mean(ms)) * 1e3
            nb = attend_bytes(wl, views)
            ablations[name] = {"views": views, "attend_us": us, "bytes": nb, "GBps": nb / us / 1e3,
                               "state_bytes_per_sequence": F.ls_view_state_bytes(run.cfg, views) / wl.batch}
        status, word = run.error()
        if status != F.LS_OK:
            raise RuntimeError(f"device error word {word:#x} after the ablation launches")

    # stochastic acceptance (T > 0) at the Qwen3 vocabulary: its own measurement
    sampled = None
    if not args.no_sampling:
        sampled = sampling_measure(F, run, wl, dev, flush, stream, evs, min(K, 200))

    # the drafter's projections (boundary keys/values, block queries) on the tensor cores
    prologue = None
    if not args.no_prologue:
        prologue = prologue_measure(F, run, wl, dev, flush, stream, evs, min(K, 200))

    # back-to-back rounds in one CUDA graph (no flush; L2 warm between rounds)
    # the attention as a drafter calls it layer by layer (one launch per tapped layer), with
    # every layer's queries computed before the calls (as ls_draft_prologue computes them):
    # LS_ATTEND_INPUTS_READY; and without the hint (inputs as if written just before each call)
    per_layer = None
    if not args.no_ablations:
        KP = min(K, 200)
        pl_outs = [run.new_out(layer_count=1) for _ in range(wl.n_layers)]
        rs = sorted({(W + i) % n_rounds for i in range(KP)})
        q_l = {r: [inp["q"][r - inp["r0"]][:, l:l + 1].contiguous() for l in range(wl.n_layers)] for r in rs}
        peak, _ = hbm_peak()
        per_layer = {"launches_per_round": wl.n_layers, "rounds": KP}
        for key, views in (("inputs_ready", VIEW_ALL | F.LS_ATTEND_INPUTS_READY), ("inputs_written_before", VIEW_ALL)):
            for i in range(KP):
                r = (W + i) % n_rounds
                flush.zero_()
                evs[i][0].record(stream)
                for l in range(wl.n_layers):
                    F.ls_draft_attend_views(run.state, l, 1, q_l[r][l], run.boundary_k, run.boundary_v, wl.hidden,
                                            run.softmax_scale, views, pl_outs[l], stream)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            us = float(np.mean([e[0].elapsed_time(e[1]) for e in evs[:KP]])) * 1e3
            per_layer[key] = {"us_per_round": us, "GBps": attend_bytes(wl) / us / 1e3,
                              "frac": attend_bytes(wl) / us / 1e3 / peak}
        per_layer["us_per_round"] = per_layer["inputs_ready"]["us_per_round"]
        per_layer["GBps"] = per_layer["inputs_ready"]["GBps"]
        status, word = run.error()
        if status != F.LS_OK:
            raise RuntimeError(f"device error word {word:#x} after the per-layer launches")
        del q_l, pl_outs

    graph_rps = None
    if not args.no_graph:
        g = torch.cuda.CUDAGraph()
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(gs):
            run.stream = gs
            with torch.cuda.graph(g, stream=gs):
                for j in range(8):
                    run.round(inp, j % n_rounds, out)
        run.stream = stream
        torch.cuda.current_stream(dev).wait_stream(gs)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        reps = 20
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        graph_rps = 8 * reps / (e0.elapsed_time(e1) / 1e3)
        del g

    # end to end through the public API with host buffers (pinned), copies inside the region
    e2e = e2e_measure(run, wl, dev, flush, K, world, inp, strong)

    # the drafting round with sampled acceptance and the projections (4 launches)
    drafting = None
    if not args.no_drafting_round:
        drafting = drafting_round_measure(WLM, wl, dev, flush, max(16, min(K, 200)),
                                          WLM.SWEEP_PREFIXES if rank == 0 and not args.no_sweep else None)

    # the same round with the attention output in the other dtype
    other_out = None
    if not args.no_configs and rank == 0 and not strong:
        other_out = out_dtype_measure(WLM, wl, dev, flush, max(16, min(K, 200)), wl.flags ^ F.LS_FLAG_OUT_F32)

    # the other workload configurations, end to end (prefill and every round)
    configs = None
    if not args.no_configs and rank == 0 and not strong:
        configs = {name: config_record(WLM, name, dev, flush, 0, wl.flags & F.LS_FLAG_OUT_F32)
                   for name in ("tiny", "qwen3_4b_32k", "qwen3_8b_128k_ragged")}

    # the prefix x concurrency x accept-mean sweep; flatness over the prefixes
    grid, flat = None, None
    if not args.no_sweep and rank == 0:
        grid = sweep_grid(WLM, dev, flush, args.sweep_rounds, wl.flags & F.LS_FLAG_OUT_F32)
        b16 = {str(p["prefix"]): p["us_per_round"] for p in grid["points"] if p["batch"] == 16
               and p["accept_mean"] == 4.0}
        flat = {"us_per_round": b16, "flatness": grid["flatness"]["batch16_mean4.0"], "batch": 16,
                "accept_mean": 4.0, "rounds": grid["rounds_per_point"]}

    # prefill and rounds reading the target's paged KV cache in place (page size 16); last:
    # it frees an 18 GB page pool, and the launch overlap of what runs right after a free
    # that large is the benchmark's artefact (see drafting_round_measure)
    paged = None
    if not args.no_paged:
        # its own round count (two halves of 3 warm-up rounds and at least 5 timed ones)
        paged = paged_measure(WLM, wl, dev, flush, max(16, min(K, 200)), rank)

    run_clk.__exit__()
    peak, peak_kind = hbm_peak()
    a_bytes = attend_bytes(wl)
    deltas = run.accept_host[[(W + i) % n_rounds for i in range(K)]] + 1
    c_bytes = commit_bytes(wl, float(deltas.mean()))
    att_s = float(np.mean(attend_ms)) / 1e3
    rnd_s = float(np.mean(round_ms)) / 1e3
    r_bytes = a_bytes + c_bytes
    achieved = a_bytes / att_s / 1e9
    tc = F.ls_attend_uses_tensor_cores(run.state)
    traffic = recorded_traffic("ls_attend_tc.cu" if tc else "ls_attend_simt.cu", f"attend_{wl.name}")

    if rank == 0:
        line = {
            "metric": METRIC, "value": job_rate(K, total_max, world, strong), "unit": "rounds/s",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": total_max * 1e3 / K, "higher_is_better": True,
            "scaling": "strong" if strong else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(full_wl),
            "parallelism": f"kv-heads x {world}" if strong else f"batch x {world}",
            "roofline": {"bound": "hbm",
                         "kernel": "ls_draft_attend (" + ("tcgen05" if tc else "CUDA cores") + ")",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "frac_of_nominal_8TBps": achieved / 8000.0,
                         "back_to_back": {"us": attend_b2b_s * 1e6, "achieved": a_bytes / attend_b2b_s / 1e9,
                                          "frac": a_bytes / attend_b2b_s / 1e9 / peak, "launches": KB},
                         "traffic": traffic, "algorithmic_bytes": a_bytes,
                         "us": att_s * 1e6, "timed_launches": KS},
            "round_roofline": {"kernels": "ls_round: commit + attention" + (
                                   " (programmatic dependent launch)" if overlapped else " (two launches)"),
                               "bytes": r_bytes, "achieved": r_bytes / rnd_s / 1e9,
                               "frac": r_bytes / rnd_s / 1e9 / peak, "unit": "GB/s"},
            "us_per_round": {"median": float(np.median(round_ms)) * 1e3, "mean": rnd_s * 1e6,
                             "p90": float(np.percentile(round_ms, 90)) * 1e3},
            "split": {"steps": KS, "commit_us": float(np.mean(commit_ms)) * 1e3,
                      "attend_us": att_s * 1e6, "commit_bytes": c_bytes,
                      "commit_GBps": c_bytes / (float(np.mean(commit_ms)) / 1e3) / 1e9},
            "graph_rounds_per_s": graph_rps,
            "attend_per_layer": per_layer,
            "view_ablations": ablations,
            "sampled_acceptance": sampled,
            "prologue": prologue,
            "paged": paged,
            "prefill": {"ms": prefill_ms, "bytes": prefill_b, "achieved_GBps": prefill_b / (prefill_ms / 1e3) / 1e9,
                        "frac": prefill_b / (prefill_ms / 1e3) / 1e9 / peak},
            "state_bytes_per_sequence": F.ls_state_bytes(run.cfg) / wl.batch,
            "flatness": flat,
            "other_output_dtype": other_out,
            "configs": configs,
            "sweep": grid,
            "drafting_round": drafting,
            "gpu_launches": 2 * K,
            "e2e": e2e,
            "clocks": dict(run_clk.summary(min_power_w=LOADED_W) or {},
                           window=f"the run's GPU work, {run_clk.period} ms samples at {LOADED_W:.0f} W or more "
                                  "(the timed rounds included)"),
            "clocks_timed_region": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget)
            if configs:  # the oracle on the other configurations' rounds, a shorter sample each
                for name in configs:
                    cwl = WLM.CONFIGS[name]
                    configs[name]["cpu_oracle"] = cpu_record(cwl, *oracle_timing(name, 1, budget_s=args.cpu_budget / 3))
        print(json.dumps(line))
    run.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


QWEN3_VOCAB = 151936
PAGE_SIZE = 16
LARGE_PAGE_SIZE = 256


def paged_measure(WLM, wl, dev, flush, n, rank):
    """ls_prefill_paged and ls_round_paged on the workload with its prefix and verify rows in
    a paged cache (page size 16, each sequence's pages scattered over the pool; the prefill
    also with 256-row pages). The
    verify pass's writes into the pages happen before the timed region (the target's work);
    every timed round is preceded by an L2 flush. Returns the timings and their HBM rates."""
    import torch
    import fixed_cost_drafter_b200 as F
    peak, _ = hbm_peak()
    # prefill with large pages first (locality of each copy), then the rounds' page size
    by_ps = {}
    for ps in (LARGE_PAGE_SIZE, PAGE_SIZE):
        run = WLM.DeviceRun(wl, device=dev, rounds=n, seq_offset=sequence_offset(rank, wl.batch))
        cache = WLM.PagedCache(run, ps, run.prefix_len + (n + 1) * (wl.block + 1), seed=1)
        run.fill_pages(cache)
        run.prefill_paged(cache)  # untimed, then a fresh state
        run.reset_state()
        torch.cuda.synchronize()
        pre = []
        run.prefill_paged(cache, timer=lambda e0, e1, nbytes: pre.append((e0, e1, nbytes)))
        torch.cuda.synchronize()
        pre_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in pre)
        pre_b = sum(nb for _, _, nb in pre)
        by_ps[ps] = {"ms": pre_ms, "bytes": pre_b, "achieved_GBps": pre_b / (pre_ms / 1e3) / 1e9,
                     "frac": pre_b / (pre_ms / 1e3) / 1e9 / peak}
        if ps != PAGE_SIZE:
            run.close()
            del cache
            torch.cuda.empty_cache()
    inp = run.make_round_inputs(0, n)
    for r in range(n):
        run.write_verify_pages(cache, inp, r)
    torch.cuda.synchronize()
    out = run.new_out()
    stream = run.stream
    kv = cache.descriptor()
    span = wl.n_kv_heads * wl.head_dim
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    warm = 3  # the first rounds load the kernels; rounds run in order (the pages hold them)
    half = n // 2  # rounds [0, half): block-table lookups; [half, n): the engine's slot mapping
    for i in range(n):
        d = kv if i < half else run.paged_descriptor(cache, i, with_slots=True)
        flush.zero_()
        evs[i][0].record(stream)
        F.ls_round_paged(run.state, run.draft[i], run.target[i], d, inp["vh"][i], run.accept_len, run.next_token,
                         inp["q"][i], 0, span, run.softmax_scale, out, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = [e[0].elapsed_time(e[1]) for e in evs[warm:half]]
    ms_slots = [e[0].elapsed_time(e[1]) for e in evs[half + warm:n]]
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} after the paged rounds")
    deltas = run.accept_host[warm:half] + 1
    r_bytes = attend_bytes(wl) + commit_bytes(wl, float(deltas.mean()))
    us = float(np.mean(ms)) * 1e3
    res = {"page_size": PAGE_SIZE, "num_pages": cache.num_pages, "prefill": by_ps[PAGE_SIZE],
           "prefill_page_size_%d" % LARGE_PAGE_SIZE: by_ps[LARGE_PAGE_SIZE],
           "round_us": {"mean": us, "median": float(np.median(ms)) * 1e3}, "round_bytes": r_bytes,
           "round_GBps": r_bytes / us / 1e3, "rounds": half - warm,
           "round_slots_us": {"mean": float(np.mean(ms_slots)) * 1e3, "median": float(np.median(ms_slots)) * 1e3,
                              "rounds": len(ms_slots)}}
    run.close()
    del cache
    torch.cuda.empty_cache()
    return res


def prologue_measure(F, run, wl, dev, flush, stream, evs, n):
    """ls_draft_prologue at the workload's shapes with seeded bf16 weights and block inputs:
    algorithmic bytes = weights + block inputs + boundary view + outputs, each once."""
    import torch
    b, L, H, Hq, D, hid, B = wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden, wl.block
    gen = torch.Generator(device=dev).manual_seed(20261)
    w_kv = (torch.randn((L, 2 * H * D, hid), device=dev, generator=gen) * hid ** -0.5).to(torch.bfloat16)
    w_q = (torch.randn((L, Hq * D, hid), device=dev, generator=gen) * hid ** -0.5).to(torch.bfloat16)
    x = torch.randn((b, L, B, hid), device=dev, generator=gen).to(torch.bfloat16)
    bkv = torch.empty((b, L, 2 * H * D), dtype=torch.bfloat16, device=dev)
    q = torch.empty((b, L, B, Hq * D), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        F.ls_draft_prologue(run.state, w_kv, w_q, x, bkv, q, stream)
    for i in range(n):
        flush.zero_()
        evs[i][0].record(stream)
        F.ls_draft_prologue(run.state, w_kv, w_q, x, bkv, q, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} after the prologue launches")
    us = float(np.mean([e[0].elapsed_time(e[1]) for e in evs[:n]])) * 1e3
    e = 2
    nbytes = (w_kv.numel() + w_q.numel() + x.numel() + b * L * hid + bkv.numel() + q.numel()) * e
    flops = 2.0 * (b * L * 2 * H * D * hid + b * L * B * Hq * D * hid)
    peak, kind = hbm_peak()
    del w_kv, w_q, x, bkv, q
    return {"us": us, "bytes": int(nbytes), "GBps": nbytes / us / 1e3, "TFLOPs": flops / us / 1e6,
            "hbm_frac": nbytes / us / 1e3 / peak, "peak_kind": kind, "launches": n}


def sampling_measure(F, run, wl, dev, flush, stream, evs, n):
    """ls_accept_sampled at batch wl.batch, block wl.block and the Qwen3 vocabulary: fp32
    probability rows (softmax of seeded normal logits, the target's close to the drafter's),
    drafts drawn from the drafter's rows, seeded draws. Algorithmic bytes: the gathered test
    values and the draw's rows (two after a rejection, one for the bonus draw)."""
    import torch
    b, B, V = wl.batch, wl.block, QWEN3_VOCAB
    gen = torch.Generator(device=dev).manual_seed(20260)
    zq = torch.randn((b, B, V), device=dev, generator=gen) * 2.0
    q = torch.softmax(zq, -1)
    zp = torch.cat([zq, zq[:, -1:]], 1) + 0.5 * torch.randn((b, B + 1, V), device=dev, generator=gen)
    pr = torch.softmax(zp, -1)
    del zq, zp
    draft = torch.multinomial(q.view(-1, V), 1, generator=gen).view(b, B).to(torch.int32)
    u = torch.rand((b, B + 1), device=dev, generator=gen)
    acc = torch.empty(b, dtype=torch.int32, device=dev)
    nxt = torch.empty(b, dtype=torch.int32, device=dev)
    for _ in range(3):
        F.ls_accept_sampled(run.state, draft, q, pr, V, u, acc, nxt, stream)
    for i in range(n):
        flush.zero_()
        evs[i][0].record(stream)
        F.ls_accept_sampled(run.state, draft, q, pr, V, u, acc, nxt, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} after the sampling launches")
    us = float(np.mean([e[0].elapsed_time(e[1]) for e in evs[:n]])) * 1e3
    a = acc.cpu().numpy()
    nbytes = int(b * 2 * B * 4 + b * (B + 1) * 4 + sum((2 if x < B else 1) * V * 4 for x in a))
    del q, pr
    return {"vocab": V, "batch": b, "block": B, "us": us, "bytes": nbytes, "GBps": nbytes / us / 1e3,
            "accept_mean": float(a.mean()), "launches": n}


class L2Flush:
    """Evicts L2 between rounds: writes a buffer larger than L2, then reads another one."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.float32, device=dev)

    def zero_(self):  # same call shape as the plain write-only buffer it replaces
        self.w.zero_()
        self.r.sum()


def pack_layout(ts):
    """Byte offsets of tensors ``ts`` packed back to back in one buffer, each starting on a
    256-byte boundary, and the buffer's size."""
    offs, off = [], 0
    for t in ts:
        offs.append(off)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    return offs, off


def pack_views(buf, ts, offs):
    """Views of the uint8 buffer ``buf`` with the dtypes and shapes of ``ts`` at ``offs``."""
    return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(ts, offs)]


def e2e_measure(run, wl, dev, flush, steps, world, inp, strong=False):
    """Rounds/s through the public entry point with every step's inputs in pinned host memory
    and its results read back to pinned host memory, inside one timed region.

    The steps are pipelined the way a caller streaming rounds would do it: two device
    buffer slots; step i's inputs go host -> device on one copy stream while step i-1's
    round runs on the compute stream (rounds stay in order: they update the state), and
    step i-1's outputs go device -> host on another copy stream. Events order the slot
    reuse. The per-step working set (213 MB of state + 30 MB of inputs and outputs) is
    larger than L2, so no flush is needed between steps.
    """
    import torch
    import fixed_cost_drafter_b200 as F
    n_distinct = min(8, run.rounds)
    # A step's inputs travel as one block of pinned memory and land in one device buffer
    # (256-byte aligned pieces, viewed as the call's tensors), and its results come back as
    # one block: one copy each way per step, as a streaming caller would pack them.
    keys = ("vk", "vv", "vh", "q", "draft", "target")
    layout, views = pack_layout, pack_views

    proto = [inp[k][0] for k in keys[:4]] + [run.draft[0], run.target[0]]
    in_offs, in_bytes = layout(proto)
    host = []
    for r in range(n_distinct):
        hb = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        for v, t in zip(views(hb, proto, in_offs), [inp[k][r] for k in keys[:4]] + [run.draft[r], run.target[r]]):
            v.copy_(t.cpu())
        host.append(hb)
    out0 = run.new_out()
    small = torch.empty(wl.batch, dtype=torch.int32, device=dev)
    out_offs, out_bytes = layout([out0, small, small])
    slots = []
    for _ in range(2):
        din = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        dout = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        o, acc, nxt = views(dout, [out0, small, small], out_offs)
        slots.append({"din": din, "in": dict(zip(keys, views(din, proto, in_offs))), "dout": dout,
                      "out": o, "acc": acc, "nxt": nxt,
                      "hout": torch.empty(out_bytes, dtype=torch.uint8).pin_memory()})
    del out0
    h2d, d2h = in_bytes, out_bytes
    comp = run.stream
    cin, cout = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    steps = max(3, min(steps, 200))
    warm = 3

    def run_steps(n, first):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            sl, hb = slots[i % 2], host[(first + i) % n_distinct]
            if i >= 2:
                cin.wait_event(ev_comp[i - 2])  # slot's inputs consumed by step i-2's round
            with torch.cuda.stream(cin):
                sl["din"].copy_(hb, non_blocking=True)
            ev_in[i].record(cin)
            comp.wait_event(ev_in[i])
            if i >= 2:
                comp.wait_event(ev_out[i - 2])  # slot's outputs read back
            F.ls_round(run.state, sl["in"]["draft"], sl["in"]["target"], sl["in"]["vk"], sl["in"]["vv"],
                       sl["in"]["vh"], sl["acc"], sl["nxt"], sl["in"]["q"], 0, wl.n_kv_heads * wl.head_dim,
                       run.softmax_scale, sl["out"], comp)
            ev_comp[i].record(comp)
            cout.wait_event(ev_comp[i])
            with torch.cuda.stream(cout):
                sl["hout"].copy_(sl["dout"], non_blocking=True)
            ev_out[i].record(cout)
        return ev_out[n - 1]

    run_steps(warm, 0).synchronize()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cin)
    last = run_steps(steps, warm)
    cout.wait_event(last)
    e1.record(cout)
    e1.synchronize()
    tot = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    return {"value": job_rate(steps, tot, world, strong), "unit": "rounds/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "pipelined": "2 buffer slots, copy streams in and out; one packed copy each way per step"}


def out_dtype_measure(WLM, wl, dev, flush, n, flags):
    """The workload's round (``ls_round``) and attention alone with the attention output in
    the other dtype (``flags`` the state's flags for it), L2 flushed before each."""
    import torch
    import fixed_cost_drafter_b200 as F
    from dataclasses import replace
    peak, _ = hbm_peak()
    w = replace(wl, flags=flags)
    run = WLM.DeviceRun(w, device=dev, rounds=n, prefill_chunk=8192)
    run.prefill()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    inp = run.make_round_inputs(0, n)
    out = run.new_out()
    ms = time_rounds(run, inp, out, flush, n)
    stream = run.stream
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for r in range(n):
        flush.zero_()
        evs[r][0].record(stream)
        run.attend(inp, r, out)
        evs[r][1].record(stream)
    torch.cuda.synchronize()
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} in the output-dtype measurement")
    att = [e0.elapsed_time(e1) for e0, e1 in evs[3:]]
    deltas = run.accept_host[3:] + 1
    a_b = attend_bytes(w)
    r_b = a_b + commit_bytes(w, float(deltas.mean()))
    st, at = us_stats(ms), us_stats(att)
    res = {"out_dtype": "f32" if flags & LS_FLAG_OUT_F32 else w.dtype, "us_per_round": st,
           "round_frac": r_b / st["mean"] / 1e3 / peak, "attend_us": at,
           "attend_frac": a_b / at["mean"] / 1e3 / peak, "attend_bytes": a_b, "rounds": len(ms)}
    run.close()
    del run, inp, out
    torch.cuda.empty_cache()
    return res


def time_rounds(run, inp, out, flush, n, warm=3):
    """CUDA-event times (ms) of rounds warm .. n - 1 of ``run`` (``ls_round``), each after an
    untimed L2 flush; rounds 0 .. warm - 1 run untimed first (they load the kernels)."""
    import torch
    stream = run.stream
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for r in range(n):
        flush.zero_()
        evs[r][0].record(stream)
        run.round(inp, r, out)
        evs[r][1].record(stream)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in evs[warm:]]


def us_stats(ms):
    return {"mean": float(np.mean(ms)) * 1e3, "median": float(np.median(ms)) * 1e3,
            "p90": float(np.percentile(ms, 90)) * 1e3}


def config_record(WLM, name, dev, flush, rank, flags=0):
    """One of the workload configurations end to end: its prefill (after one untimed
    prefill into a state then reset) and all of its rounds (3 untimed), an L2 flush before
    each round."""
    import torch
    import fixed_cost_drafter_b200 as F
    from dataclasses import replace
    peak, _ = hbm_peak()
    wl = WLM.CONFIGS[name]
    wl = replace(wl, flags=wl.flags | flags)
    run = WLM.DeviceRun(wl, device=dev, seq_offset=sequence_offset(rank, wl.batch))
    run.prefill()
    run.reset_state()
    pre = []
    run.prefill(timer=lambda e0, e1, nbytes: pre.append((e0, e1, nbytes)))
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    pre_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in pre)
    pre_b = sum(nb for _, _, nb in pre)
    inp = run.make_round_inputs()
    out = run.new_out()
    warm = 3
    ms = time_rounds(run, inp, out, flush, run.rounds, warm)
    status, word = run.error()
    if status != F.LS_OK:
        raise RuntimeError(f"device error word {word:#x} in {name}")
    deltas = run.accept_host[warm:] + 1
    r_bytes = attend_bytes(wl) + commit_bytes(wl, float(deltas.mean()))
    st = us_stats(ms)
    rec = {"workload": workload_config(wl)["workload"],
           "prefix_rows": int(np.sum(run.prefix_len)),
           "prefill": {"ms": pre_ms, "bytes": pre_b, "achieved_GBps": pre_b / (pre_ms / 1e3) / 1e9,
                       "frac": pre_b / (pre_ms / 1e3) / 1e9 / peak, "calls": len(pre)},
           "rounds": len(ms), "us_per_round": st, "rounds_per_s": 1e6 / st["mean"],
           "realised_accept_mean": float(deltas.mean() - 1), "round_bytes": r_bytes,
           "round_frac": r_bytes / st["mean"] / 1e3 / peak,
           "state_bytes_per_sequence": F.ls_state_bytes(run.cfg) / wl.batch}
    run.close()
    del run, inp, out
    torch.cuda.empty_cache()
    return rec


def sweep_grid(WLM, dev, flush, rounds, flags=0):
    """The prefix x concurrency x accept-mean sweep (Qwen3-8B shapes): per point the
    per-round time (median over the rounds after 3 untimed ones, an L2 flush before each)
    and the drafter state bytes; flatness of the per-round time over the prefixes for
    every (batch, accept mean). The prefill runs in chunks of 8192 rows."""
    import torch
    import fixed_cost_drafter_b200 as F
    from dataclasses import replace
    peak, _ = hbm_peak()
    points, flat = [], {}
    for b in WLM.SWEEP_BATCHES:
        for m in WLM.SWEEP_MEANS:
            row = {}
            for P in WLM.SWEEP_PREFIXES:
                wl = WLM.sweep_point(P, b, m)
                wl = replace(wl, flags=wl.flags | flags)
                # 8192-row prefill chunks: no large buffer is freed right before the timed
                # rounds (see drafting_round_measure)
                run = WLM.DeviceRun(wl, device=dev, rounds=rounds, prefill_chunk=8192)
                run.prefill()
                torch.cuda.synchronize()
                torch.cuda.empty_cache()
                inp = run.make_round_inputs(0, rounds)
                out = run.new_out()
                ms = time_rounds(run, inp, out, flush, rounds)
                status, word = run.error()
                if status != F.LS_OK:
                    raise RuntimeError(f"device error word {word:#x} at sweep point {wl.name}")
                deltas = run.accept_host[3:] + 1
                st = us_stats(ms)
                r_bytes = attend_bytes(wl) + commit_bytes(wl, float(deltas.mean()))
                sb = F.ls_state_bytes(run.cfg)
                points.append({"prefix": P, "batch": b, "accept_mean": m, "us_per_round": st["median"],
                               "us_mean": st["mean"], "rounds": len(ms),
                               "realised_accept_mean": float(deltas.mean() - 1),
                               "round_frac": r_bytes / st["median"] / 1e3 / peak,
                               "state_bytes": sb, "state_bytes_per_sequence": sb / b})
                row[P] = st["median"]
                run.close()
                del run, inp, out
                torch.cuda.empty_cache()
            v = list(row.values())
            flat[f"batch{b}_mean{m}"] = (max(v) - min(v)) / min(v)
    return {"points": points, "flatness": flat, "rounds_per_point": rounds - 3,
            "state_bytes_identical_across_prefixes": all(
                len({p["state_bytes"] for p in points if p["batch"] == b}) == 1 for b in WLM.SWEEP_BATCHES)}


def drafting_round_measure(WLM, wl, dev, flush, n, prefixes=None):
    """The round a drafter runs with sampled decoding (T > 0): the stochastic acceptance of
    the verified block (``ls_accept_sampled`` at the Qwen3 vocabulary), the commit of the
    accepted rows (``ls_commit_accepted``), the drafter's projections of the new boundary
    and of its block inputs (``ls_draft_prologue``, seeded weights) and the attention over
    the views with those projections (``ls_draft_attend``), an L2 flush before each round.
    Timed at the workload's prefix and, with ``prefixes``, at batch 16 over those prefixes
    (flatness)."""
    import torch
    import fixed_cost_drafter_b200 as F
    from dataclasses import replace
    peak, _ = hbm_peak()
    b, L, H, Hq, D, hid, B, V = (wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.hidden,
                                 wl.block, QWEN3_VOCAB)
    gen = torch.Generator(device=dev).manual_seed(20262)
    zq = torch.randn((b, B, V), device=dev, generator=gen) * 2.0
    qp = torch.softmax(zq, -1)
    zp = torch.cat([zq, zq[:, -1:]], 1) + 0.5 * torch.randn((b, B + 1, V), device=dev, generator=gen)
    pp = torch.softmax(zp, -1)
    del zq, zp
    draft = torch.multinomial(qp.view(-1, V), 1, generator=gen).view(b, B).to(torch.int32)
    n_u = 8
    us_draws = torch.rand((n_u, b, B + 1), device=dev, generator=gen)
    w_kv = (torch.randn((L, 2 * H * D, hid), device=dev, generator=gen) * hid ** -0.5).to(torch.bfloat16)
    w_q = (torch.randn((L, Hq * D, hid), device=dev, generator=gen) * hid ** -0.5).to(torch.bfloat16)
    x = torch.randn((b, L, B, hid), device=dev, generator=gen).to(torch.bfloat16)
    bkv = torch.empty((b, L, 2 * H * D), dtype=torch.bfloat16, device=dev)
    qd = torch.empty((b, L, B, Hq * D), dtype=torch.bfloat16, device=dev)
    acc = torch.empty(b, dtype=torch.int32, device=dev)
    nxt = torch.empty(b, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)

    def series(w, rounds):
        # prefill in 8192-row chunks: freeing one large prefix buffer (34 GB at 128K) right
        # before the timed rounds took the launch overlap away from most rounds (a driver
        # state after a large free, not the round's work: the same rounds with 40 GB freed
        # just before were as slow at a 4K prefix, and as fast with it held)
        run = WLM.DeviceRun(w, device=dev, rounds=rounds, prefill_chunk=8192)
        run.prefill()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        inp = run.make_round_inputs(0, rounds)
        out = run.new_out()
        st = run.stream
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(rounds)]
        a_seen = []

        def one_round(r, e=None):
            # events between the calls (the split) serialise them: the chained time is
            # taken without them
            F.ls_accept_sampled(run.state, draft, qp, pp, V, us_draws[r % n_u], acc, nxt, st)
            if e is not None:
                e[1].record(st)
            F.ls_commit_accepted(run.state, acc, inp["vk"][r], inp["vv"][r], inp["vh"][r], st)
            if e is not None:
                e[2].record(st)
            F.ls_draft_prologue(run.state, w_kv, w_q, x, bkv, qd, st)
            if e is not None:
                e[3].record(st)
            F.ls_draft_attend(run.state, 0, L, qd, bkv, bkv[..., H * D:], 2 * H * D, scale, out, st)

        half = rounds // 2
        for r in range(rounds):
            flush.zero_()
            e = evs[r]
            e[0].record(st)
            one_round(r, e if r >= half else None)
            e[4].record(st)
            if r < n_u:
                a_seen.append(acc.clone())
        torch.cuda.synchronize()
        status, word = run.error()
        if status != F.LS_OK:
            raise RuntimeError(f"device error word {word:#x} in the drafting round")
        warm = 3
        tot = [e[0].elapsed_time(e[4]) for e in evs[warm:half]]
        parts = {k: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs[half:]])) * 1e3
                 for i, k in enumerate(("accept_sampled_us", "commit_accepted_us", "prologue_us", "attend_us"))}
        parts["sum_us"] = sum(parts.values())
        a_all = torch.stack(a_seen).cpu().numpy()
        rows = float(np.mean(np.where(a_all < B, 2, 1).sum(axis=1)))  # probability rows the draw reads
        run.close()
        del run, inp, out
        torch.cuda.empty_cache()
        return tot, parts, float(a_all.mean()), rows

    tot, parts, a_mean, rows = series(wl, max(2 * n, 32))
    nbytes = (int(b * 2 * B * 4 + b * (B + 1) * 4 + rows * V * 4)  # sampling: tests, draws, the drawn rows
              + commit_bytes(wl, a_mean + 1)
              + (w_kv.numel() + w_q.numel() + x.numel() + b * L * hid + bkv.numel() + qd.numel()) * 2
              + attend_bytes(wl))
    st = us_stats(tot)
    res = {"kernels": "ls_accept_sampled -> ls_commit_accepted -> ls_draft_prologue -> ls_draft_attend",
           "vocab": V, "us_per_round": st, "rounds_per_s": 1e6 / st["mean"], "rounds": len(tot),
           "split": dict(parts, note="other rounds, with an event between the calls (which serialises them)"),
           "accept_mean": a_mean, "bytes": nbytes, "frac": nbytes / st["mean"] / 1e3 / peak, "launches_per_round": 4}
    if prefixes:
        by_p, split_p = {}, {}
        for P in prefixes:
            t, parts_p, _, _ = series(replace(wl, name=f"{wl.name}_p{P}", prefix=P), 32)
            by_p[str(P)] = float(np.median(t)) * 1e3
            split_p[str(P)] = parts_p
        v = list(by_p.values())
        res["over_prefix"] = {"us_per_round_median": by_p, "flatness": (max(v) - min(v)) / min(v),
                              "batch": wl.batch, "split": split_p}
    del qp, pp, w_kv, w_q, x
    torch.cuda.empty_cache()
    return res


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--distinct-rounds", type=int, default=128)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=WORKLOAD)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-ablations", action="store_true", help="skip the view-ablation attention timings")
    ap.add_argument("--no-sampling", action="store_true", help="skip the stochastic-acceptance timing")
    ap.add_argument("--no-prologue", action="store_true", help="skip the drafter-projection timing")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged-KV prefill and round timings")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="batch", choices=["batch", "kv-heads"],
                    help="N > 1: each rank owns a batch of sequences (weak scaling) or a share of every "
                         "sequence's KV heads (strong scaling)")
    ap.add_argument("--clock-log", default=None,
                    help="CSV of the nvidia-smi clock samples ('{rank}' is replaced; default _build/clocks_rank{rank}.csv)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--sweep-rounds", type=int, default=128, help="rounds per sweep point (3 of them untimed)")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workload configurations")
    ap.add_argument("--no-drafting-round", action="store_true",
                    help="skip the drafting round with sampled acceptance and projections")
    ap.add_argument("--prefix", type=int, default=0, help="override the workload's prefix length")
    ap.add_argument("--out", default="bf16", choices=["bf16", "f32"], help="dtype of the attention output")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
