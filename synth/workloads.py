"""Workload recipes of the drafting round: shapes, sizes, seeds and accept-length laws.

The workloads take the shapes of the paper page's experiments only (Qwen3-4B/8B tapped
state, prefix 32K/64K/128K, concurrency 16, accept means near the reported tau); the
values are seeded synthetic draws from ``synth`` (no dataset, no trained weights). This
module holds no arithmetic of the method and does not load the CUDA library: the CPU
oracle's timing runs use it too.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    hidden: int
    block: int
    window: int
    scales: tuple
    slots: int
    dtype: str  # "bf16" | "f32"
    prefix: object  # int, or (lo, hi) for per-sequence lengths uniform on {lo..hi}
    rounds: int
    accept_mean: float | None  # None: uniform on 0..B
    vocab: int
    head_scale: bool = False
    flags: int = 0

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads

    def config(self):
        """The library's ``ls_config`` for these shapes (loads the CUDA library)."""
        import fixed_cost_drafter_b200 as F
        return F.make_config(self.batch, self.n_layers, self.n_kv_heads, self.n_q_heads,
                             self.head_dim, self.hidden, self.block, self.window, list(self.scales),
                             self.slots, F.LS_BF16 if self.dtype == "bf16" else F.LS_F32, self.flags)

    def prefix_lengths(self):
        import synth
        if isinstance(self.prefix, tuple):
            return synth.prefix_lengths(self.seed, self.batch, *self.prefix)
        return np.full(self.batch, int(self.prefix), dtype=np.int64)

    def accepts(self):
        import synth
        return synth.accept_lengths(self.seed, self.rounds, self.batch, self.block, self.accept_mean)

    def token_ids(self):
        import synth
        return synth.token_ids(self.seed, self.rounds, self.batch, self.block, self.accepts(), self.vocab)

    def elem(self):
        return 2 if self.dtype == "bf16" else 4


QWEN3_8B = dict(n_layers=4, n_kv_heads=8, n_q_heads=32, head_dim=128, hidden=4096, block=16,
                window=512, scales=(64, 512, 4096), slots=32, dtype="bf16", vocab=151936)

CONFIGS = {
    "tiny": Workload("tiny", 0, 1, 1, 2, 4, 64, 256, 4, 32, (8, 32, 128), 4, "f32", 512, 20, None, 1000),
    "qwen3_4b_32k": Workload("qwen3_4b_32k", 1, 16, **{**QWEN3_8B, "hidden": 2560}, prefix=32768,
                             rounds=256, accept_mean=4.7),
    "qwen3_8b_64k": Workload("qwen3_8b_64k", 2, 16, **QWEN3_8B, prefix=65536, rounds=256,
                             accept_mean=5.0, head_scale=True),
    "qwen3_8b_128k_ragged": Workload("qwen3_8b_128k_ragged", 3, 16, **QWEN3_8B, prefix=(98304, 131072),
                                     rounds=512, accept_mean=3.5),
}


def sweep_point(prefix: int, batch: int, accept_mean: float) -> Workload:
    """One point of the prefix x concurrency x accept-mean sweep (Qwen3-8B shapes)."""
    return Workload(f"sweep_p{prefix}_b{batch}_m{accept_mean}", 4, batch, **QWEN3_8B, prefix=prefix,
                    rounds=128, accept_mean=accept_mean)


SWEEP_PREFIXES = (4096, 16384, 32768, 65536, 131072)
SWEEP_BATCHES = (1, 4, 16, 64)
SWEEP_MEANS = (2.5, 4.0, 6.0)
