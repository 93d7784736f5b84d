"""Plain fp64 CPU oracle of the LongSpark fixed-cost drafting round.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the CUDA
library; both sides only receive the same seeded inputs.

Source: "LongSpark: Efficient speculative decoding with a fixed-cost parallel drafter"
(arXiv 2609.37029), thelatestinai.com paper page:

* Figure 2 caption — one decoding round: (a) the target verifies the proposed tokens,
  (b) three fixed-size views are extracted from the target's state (boundary state,
  recent KV window, global context summary), (c) the drafter proposes the next block
  from the views at a cost independent of the prefix length.
* Figure 3 caption — the global summary is initialised over the full prefix at target
  prefill, then updated with only the newly retained KV rows N, Delta = |N| <= B + 1.
* Figure 1 caption and the abstract — fixed-size, multiscale views; O(1) drafting cost.
* Table 3 caption — greedy decoding (T = 0): acceptance is an exact token match.

The pages print no formula for the views. The readings taken here (each listed with its
reason in the design notes of the repository):

1. Verify row 0 is the previous round's bonus token, rows 1..B are the drafts;
   ``target[i]`` is the target's greedy choice after verify row i. The accepted count
   ``a`` is the number of leading ``i < B`` with ``draft[i] == target[i]``; verify rows
   0..a are retained (Delta = a + 1 <= B + 1, Figure 3 caption) and ``target[a]`` is the
   next (bonus) token, whose K/V only exist after the next verify pass.
2. Window: the last min(len, W) retained rows; row p sits in ring slot p mod W.
3. Summary, per tapped layer and KV head and for each scale s_k: segment j covers the
   absolute rows [j*s_k, (j+1)*s_k) (aligned to position 0, so that a complete segment
   never changes); the slots hold the means of the ``slots`` most recent complete
   segments (segment j in slot j mod slots); the open partial segment keeps its sum and
   row count; one running sum covers all retained rows (the global mean).
4. Boundary: the hidden vectors of the last retained position (verify row a; after
   prefill, the caller's hidden at position P - 1).
5. Attention, per layer and query head qh with KV head g = qh // (Hq / Hkv) (contiguous
   grouping): keys/values in the order [boundary, window slots, for each scale: the
   ``slots`` segment means then the partial mean, global mean]; empty slots masked;
   logits q.k * softmax_scale; no mask among the B block queries; no positional bias.

Everything is computed in fp64 from inputs that are read exactly (bf16 and fp32 both
convert to fp64 without rounding).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"

# the three views (Figure 2 caption (b)); Table 5 ablates each of them
VIEW_BOUNDARY = 0x1
VIEW_WINDOW = 0x2
VIEW_SUMMARY = 0x4
VIEW_ALL = 0x7


# ----------------------------------------------------------------------------------
# configuration and exact input conversion
# ----------------------------------------------------------------------------------
@dataclass(frozen=True)
class Shapes:
    """Shapes of one drafting state (one sequence is simulated at a time).

    ``n_layers`` / ``n_kv_heads`` / ``n_q_heads`` are the sizes of the arrays the
    oracle is given, so a caller may pass a subset of layers and KV heads (with the
    matching ``Hq / Hkv`` query heads per KV head) and get that subset's views.
    """

    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    hidden: int
    block: int  # B
    window: int  # W
    scales: tuple  # s_0 < s_1 < ...
    slots: int

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_attn_slots(self) -> int:
        """S = 1 boundary + W window + per scale (slots + 1 partial) + 1 global."""
        return 1 + self.window + len(self.scales) * (self.slots + 1) + 1


def to_f64(x, dtype: str) -> np.ndarray:
    """Exact fp64 value of fp32 data, or of bf16 data given as its uint16 bit patterns."""
    x = np.asarray(x)
    if dtype == F32:
        return x.astype(np.float32).astype(np.float64)
    if dtype == BF16:
        bits = x.astype(np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------------
# (a) verification: greedy accept-length scan (Table 3, T = 0; Figure 3: Delta <= B+1)
# ----------------------------------------------------------------------------------
def accept_scan(draft_ids, target_ids):
    """Greedy acceptance of one block.

    ``draft_ids`` has B entries, ``target_ids`` B + 1. Returns ``(a, next_token)``:
    ``a`` is the index of the first draft the target disagrees with (B if it accepts
    all), ``next_token`` is the target's own choice at that position.
    """
    B = len(draft_ids)
    assert len(target_ids) == B + 1
    for i in range(B):
        if int(draft_ids[i]) != int(target_ids[i]):
            return i, int(target_ids[i])
    return B, int(target_ids[B])


# ----------------------------------------------------------------------------------
# (b) the three views of one sequence
# ----------------------------------------------------------------------------------
@dataclass
class Views:
    """Fixed-size views of one sequence; every array has a size set by the shapes."""

    length: int
    ring_k: np.ndarray  # [L][Hkv][W][D]
    ring_v: np.ndarray
    seg_k: list  # per scale: [L][Hkv][slots][D] segment means
    seg_v: list
    n_seg: list  # per scale: number of complete segments so far
    part_k: list  # per scale: [L][Hkv][D] sum of the open partial segment
    part_v: list
    part_count: list  # per scale: rows in the open partial segment
    glob_k: np.ndarray  # [L][Hkv][D] sum of all retained rows
    glob_v: np.ndarray
    boundary: np.ndarray  # [L][hidden]

    def state_arrays(self):
        arrs = [self.ring_k, self.ring_v, self.glob_k, self.glob_v, self.boundary]
        arrs += self.seg_k + self.seg_v + self.part_k + self.part_v
        return arrs


def empty_views(sh: Shapes) -> Views:
    L, H, D = sh.n_layers, sh.n_kv_heads, sh.head_dim
    nsc = len(sh.scales)
    z = lambda *s: np.zeros(s, dtype=np.float64)  # noqa: E731
    return Views(
        length=0,
        ring_k=z(L, H, sh.window, D),
        ring_v=z(L, H, sh.window, D),
        seg_k=[z(L, H, sh.slots, D) for _ in range(nsc)],
        seg_v=[z(L, H, sh.slots, D) for _ in range(nsc)],
        n_seg=[0] * nsc,
        part_k=[z(L, H, D) for _ in range(nsc)],
        part_v=[z(L, H, D) for _ in range(nsc)],
        part_count=[0] * nsc,
        glob_k=z(L, H, D),
        glob_v=z(L, H, D),
        boundary=z(L, sh.hidden),
    )


def state_bytes(sh: Shapes, views: Views) -> int:
    """Bytes of drafter state the oracle holds for one sequence (no prefix term)."""
    return int(sum(a.nbytes for a in views.state_arrays())) + 8 * (1 + 2 * len(sh.scales))


def retain_row(sh: Shapes, v: Views, k_row: np.ndarray, v_row: np.ndarray) -> None:
    """Incremental update with one newly retained row (Figure 3 caption).

    ``k_row``/``v_row`` are [L][Hkv][D] fp64: the row at absolute position ``v.length``.
    The row enters the ring, every scale's open segment and the global sum; a segment
    whose last row this is becomes a slot mean and the partial restarts empty.
    """
    p = v.length
    v.ring_k[:, :, p % sh.window, :] = k_row
    v.ring_v[:, :, p % sh.window, :] = v_row
    for k, s in enumerate(sh.scales):
        v.part_k[k] += k_row
        v.part_v[k] += v_row
        v.part_count[k] += 1
        if v.part_count[k] == s:
            j = v.n_seg[k]
            v.seg_k[k][:, :, j % sh.slots, :] = v.part_k[k] / s
            v.seg_v[k][:, :, j % sh.slots, :] = v.part_v[k] / s
            v.n_seg[k] += 1
            v.part_k[k] = np.zeros_like(v.part_k[k])
            v.part_v[k] = np.zeros_like(v.part_v[k])
            v.part_count[k] = 0
    v.glob_k += k_row
    v.glob_v += v_row
    v.length = p + 1


def views_from_scratch(sh: Shapes, full_k: np.ndarray, full_v: np.ndarray, n: int,
                       boundary: np.ndarray | None = None) -> Views:
    """The views by their definition over the first ``n`` rows of a full KV cache.

    ``full_k``/``full_v`` are [L][Hkv][>=n][D] fp64 (the target's cache of the tapped
    layers, as stored). This is the from-scratch recompute the incremental form must
    equal, and it is how the summary is initialised over the full prefix at prefill.
    """
    v = empty_views(sh)
    v.length = n
    for p in range(max(0, n - sh.window), n):
        v.ring_k[:, :, p % sh.window, :] = full_k[:, :, p, :]
        v.ring_v[:, :, p % sh.window, :] = full_v[:, :, p, :]
    for k, s in enumerate(sh.scales):
        n_c = n // s
        for j in range(max(0, n_c - sh.slots), n_c):
            v.seg_k[k][:, :, j % sh.slots, :] = full_k[:, :, j * s:(j + 1) * s, :].mean(axis=2)
            v.seg_v[k][:, :, j % sh.slots, :] = full_v[:, :, j * s:(j + 1) * s, :].mean(axis=2)
        v.n_seg[k] = n_c
        v.part_k[k] = full_k[:, :, n_c * s:n, :].sum(axis=2)
        v.part_v[k] = full_v[:, :, n_c * s:n, :].sum(axis=2)
        v.part_count[k] = n - n_c * s
    v.glob_k = full_k[:, :, :n, :].sum(axis=2)
    v.glob_v = full_v[:, :, :n, :].sum(axis=2)
    if boundary is not None:
        v.boundary = np.array(boundary, dtype=np.float64)
    return v


def prefill(sh: Shapes, prefix_k: np.ndarray, prefix_v: np.ndarray, n: int,
            last_hidden: np.ndarray) -> Views:
    """Views after target prefill (Figure 3: summary initialised over the full prefix).

    ``prefix_k``/``prefix_v`` are [L][P][Hkv][D] fp64 (position-major, as a KV cache
    stores them) with P >= n; ``last_hidden`` is [L][hidden], the tapped-layer hidden
    vectors at position n - 1, which become the boundary state.
    """
    fk = np.transpose(prefix_k[:, :n], (0, 2, 1, 3))
    fv = np.transpose(prefix_v[:, :n], (0, 2, 1, 3))
    return views_from_scratch(sh, fk, fv, n, boundary=last_hidden)


def commit_round(sh: Shapes, v: Views, draft_ids, target_ids, verify_k: np.ndarray,
                 verify_v: np.ndarray, verify_hidden: np.ndarray):
    """Figure 2 (a)-(b): accept, then extract the views from the verification pass.

    ``verify_k``/``verify_v`` are [L][B+1][Hkv][D] fp64 (the K/V the target wrote for
    the B + 1 verified positions), ``verify_hidden`` is [L][B+1][hidden]. Rows 0..a are
    the newly retained rows N (|N| = a + 1 <= B + 1). Returns ``(a, next_token)``.
    """
    a, nxt = accept_scan(draft_ids, target_ids)
    assert a + 1 <= sh.block + 1
    for i in range(a + 1):
        retain_row(sh, v, verify_k[:, i], verify_v[:, i])
    v.boundary = np.array(verify_hidden[:, a], dtype=np.float64)
    return a, nxt


# ----------------------------------------------------------------------------------
# (b') the same extraction reading the target's paged KV cache
# ----------------------------------------------------------------------------------
# The views come from the target's state (Figure 2 caption (b)); an inference engine keeps
# that state's K/V rows in fixed-size pages. The reading taken: every tapped layer has
# pages of its own, [num_pages][page_size][Hkv][D]; position p of sequence b sits in page
# block_table[b][p // page_size] at offset p % page_size. Prefill reads positions
# 0 .. P - 1; a round's verify row i is the target's position len + i (the bonus token
# of verify row 0 follows the last retained row), so the retained rows N of Figure 3 are
# positions len .. len + a.
def paged_rows(pages, block_table, page_size: int, b: int, positions) -> np.ndarray:
    """Rows of sequence ``b`` at ``positions`` from ``pages`` [L][num_pages][page_size]
    [Hkv][D]: returns [L][len(positions)][Hkv][D] fp64 (position-major, as ``prefill``
    and ``commit_round`` take them)."""
    pages = np.asarray(pages)
    L, _, _, H, D = pages.shape
    out = np.zeros((L, len(positions), H, D), dtype=np.float64)
    for i, pos in enumerate(positions):
        page = int(block_table[b][pos // page_size])
        out[:, i] = pages[:, page, pos % page_size]
    return out


def prefill_paged(sh: Shapes, k_pages, v_pages, block_table, page_size: int, b: int, n: int,
                  last_hidden: np.ndarray) -> Views:
    """``prefill`` of sequence ``b`` over its first ``n`` positions read from the pages."""
    pos = range(n)
    return prefill(sh, paged_rows(k_pages, block_table, page_size, b, pos),
                   paged_rows(v_pages, block_table, page_size, b, pos), n, last_hidden)


def commit_round_paged(sh: Shapes, v: Views, draft_ids, target_ids, k_pages, v_pages, block_table,
                       page_size: int, b: int, verify_hidden: np.ndarray):
    """``commit_round`` of sequence ``b`` with verify row i read from the pages at
    position ``v.length + i``. Returns ``(a, next_token)``."""
    pos = range(v.length, v.length + sh.block + 1)
    return commit_round(sh, v, draft_ids, target_ids, paged_rows(k_pages, block_table, page_size, b, pos),
                        paged_rows(v_pages, block_table, page_size, b, pos), verify_hidden)


# ----------------------------------------------------------------------------------
# (c) the drafter's block attention over the views
# ----------------------------------------------------------------------------------
def attention_slots(sh: Shapes, v: Views, l: int, g: int, boundary_k: np.ndarray,
                    boundary_v: np.ndarray):
    """Keys, values and validity of the S attention slots of (layer l, KV head g).

    Order: [boundary, window ring slots 0..W-1, for each scale: segment slots
    0..slots-1 then the partial mean, global mean]. ``boundary_k``/``boundary_v`` are
    [L][Hkv][D]: the drafter's key/value for the boundary state.
    """
    keys, vals, valid = [], [], []
    keys.append(boundary_k[l, g]); vals.append(boundary_v[l, g]); valid.append(True)
    for r in range(sh.window):
        keys.append(v.ring_k[l, g, r]); vals.append(v.ring_v[l, g, r])
        valid.append(r < v.length)  # slot r holds a row once len > r
    for k, s in enumerate(sh.scales):
        for i in range(sh.slots):
            keys.append(v.seg_k[k][l, g, i]); vals.append(v.seg_v[k][l, g, i])
            valid.append(i < v.n_seg[k])  # slot i is filled once n_seg > i
        c = v.part_count[k]
        if c > 0:
            keys.append(v.part_k[k][l, g] / c); vals.append(v.part_v[k][l, g] / c)
        else:
            keys.append(np.zeros(sh.head_dim)); vals.append(np.zeros(sh.head_dim))
        valid.append(c > 0)
    if v.length > 0:
        keys.append(v.glob_k[l, g] / v.length); vals.append(v.glob_v[l, g] / v.length)
    else:
        keys.append(np.zeros(sh.head_dim)); vals.append(np.zeros(sh.head_dim))
    valid.append(v.length > 0)
    return np.stack(keys), np.stack(vals), np.array(valid, dtype=bool)


def view_of_slots(sh: Shapes) -> np.ndarray:
    """The view (VIEW_*) each of the S attention slots belongs to, in slot order."""
    n_summary = sh.n_attn_slots - 1 - sh.window
    return np.array([VIEW_BOUNDARY] + [VIEW_WINDOW] * sh.window + [VIEW_SUMMARY] * n_summary)


def draft_attend(sh: Shapes, v: Views, q: np.ndarray, boundary_k: np.ndarray,
                 boundary_v: np.ndarray, softmax_scale: float, views: int = VIEW_ALL,
                 return_lse: bool = False):
    """Figure 2 (c): block attention of the B drafter queries over the views.

    ``q`` is [L][B][Hq][D] fp64; returns [L][B][Hq][D] fp64. Softmax in fp64 with
    masked slots at -inf; the B queries see the same key set (no causal mask).

    ``views`` (OR of VIEW_*): only the slots of these views take part (Table 5's
    component ablations drop one view each). A row left with no valid slot gets zeros.
    With ``return_lse`` also returns the natural-log partition function of every row,
    [L][B][Hq] (-inf for a row with no valid slot).
    """
    out = np.zeros_like(q, dtype=np.float64)
    lse = np.full(q.shape[:3], -np.inf)
    grp = sh.group
    keep = (view_of_slots(sh) & views) != 0
    for l in range(sh.n_layers):
        for qh in range(sh.n_q_heads):
            g = qh // grp
            K, V, ok = attention_slots(sh, v, l, g, boundary_k, boundary_v)
            ok = ok & keep
            if not ok.any():
                continue  # nothing to attend to: zero output
            logits = (q[l, :, qh, :] @ K.T) * softmax_scale  # [B][S]
            logits[:, ~ok] = -np.inf
            m = logits.max(axis=1, keepdims=True)
            w = np.exp(logits - m)
            z = w.sum(axis=1, keepdims=True)
            out[l, :, qh, :] = (w / z) @ V
            lse[l, :, qh] = (m + np.log(z))[:, 0]
    return (out, lse) if return_lse else out


# ----------------------------------------------------------------------------------
# stochastic acceptance (T > 0)
# ----------------------------------------------------------------------------------
# The pages compare greedy decoding (Table 3, T = 0) with sampled decoding (Table 1) but
# print no acceptance rule for T > 0. The reading taken is standard speculative sampling
# (Leviathan, Kalman and Matias 2023; Chen et al. 2023), position by position over the
# block: draft i is kept when u_i * q_i(d_i) < p_i(d_i) (u_i uniform in [0, 1), the test
# made in fp32 as the GPU makes it: it decides an integer); at the first rejection the
# next token is drawn from the residual max(0, p_i - q_i) (from p_i itself when that
# residual has no mass), and after B acceptances from p_B. The draws u_0..u_{B-1} and the
# final draw v are inputs.
def accept_decisions(draft_ids, q_rows, p_rows, u):
    """fp32 acceptance tests of one sequence: draft i kept iff u_i * q_i(d_i) < p_i(d_i).

    q_rows [B][V], p_rows [B+1][V] (fp32 probabilities), u [B]. Returns a (leading kept
    count) and the per-position decisions.
    """
    B = len(draft_ids)
    keep = np.zeros(B, dtype=bool)
    for i in range(B):
        d = int(draft_ids[i])
        qd, pd = np.float32(q_rows[i, d]), np.float32(p_rows[i, d])
        keep[i] = np.float32(np.float32(u[i]) * qd) < pd
    a = B
    for i in range(B):
        if not keep[i]:
            a = i
            break
    return a, keep


def sampling_weights(q_rows, p_rows, a):
    """The distribution the next token is drawn from (unnormalised, fp64): the residual
    max(0, p_a - q_a) after a rejection at position a < B, else p_B."""
    B = q_rows.shape[0]
    if a < B:
        return np.maximum(0.0, p_rows[a].astype(np.float64) - q_rows[a].astype(np.float64))
    return p_rows[B].astype(np.float64)


def draw_weights(q_rows, p_rows, a):
    """The weights the next token is actually drawn from: ``sampling_weights``, except that
    a residual with no mass (p_a <= q_a everywhere, which exact arithmetic only reaches when
    the two rows are equal, so a rejection there comes from rounding or from a draft that q
    gives no mass) is replaced by the target's own row p_a. Speculative sampling emits
    samples of the target's distribution; p_a is that distribution at the rejected
    position, so the emitted token always lies in the target's support there.

    Raises ValueError when the row drawn from has no mass at all (not a probability row).
    """
    w = sampling_weights(q_rows, p_rows, a)
    if not (w > 0).any() and a < q_rows.shape[0]:
        w = p_rows[a].astype(np.float64)
    if not (w > 0).any():
        raise ValueError("the target's probability row has no mass")
    return w


def inverse_cdf(w, v):
    """Smallest t with sum(w[:t+1]) > v * sum(w), for weights w >= 0 with a positive sum
    and a draw 0 <= v < 1. The threshold is then below the total, so some running sum
    passes it, and the first that does ends on an entry with mass."""
    w = np.asarray(w, np.float64)
    if not (0.0 <= v < 1.0):
        raise ValueError("the draw must lie in [0, 1)")
    c = np.cumsum(w)
    if not c[-1] > 0:
        raise ValueError("weights without mass")
    return int(np.searchsorted(c, v * c[-1], side="right"))


def accept_sampled(draft_ids, q_rows, p_rows, u, v):
    """One sequence's stochastic acceptance: (a, next token), the next token drawn from
    ``draw_weights`` with the draw v."""
    a, _ = accept_decisions(draft_ids, q_rows, p_rows, u)
    return a, inverse_cdf(draw_weights(q_rows, p_rows, a), v)


# ----------------------------------------------------------------------------------
# drafter prologue: projections of the boundary and of the block inputs
# ----------------------------------------------------------------------------------
# The pages say only that the drafter uses the views (Figure 2 caption (c)); its learned
# projections are not described. The reading taken: per tapped layer l, the boundary
# key/value rows are linear maps of the boundary hidden vector, and the block's queries
# linear maps of the drafter's block inputs, with no bias or normalisation:
#   bkv[b][l][n] = sum_k W_kv[l][n][k] h[b][l][k]   (n < Hkv D: key of head n // D, then values)
#   q[b][l][i][n] = sum_k W_q[l][n][k] x[b][l][i][k]
def draft_prologue(w_kv, w_q, boundary, x):
    """fp64 projections: w_kv [L][2 Hkv D][hidden], w_q [L][Hq D][hidden], boundary
    [b][L][hidden], x [b][L][B][hidden] -> (bkv [b][L][2 Hkv D], q [b][L][B][Hq D])."""
    w_kv, w_q = np.asarray(w_kv, np.float64), np.asarray(w_q, np.float64)
    bkv = np.einsum("lnk,blk->bln", w_kv, np.asarray(boundary, np.float64))
    q = np.einsum("lnk,blik->blin", w_q, np.asarray(x, np.float64))
    return bkv, q


# ----------------------------------------------------------------------------------
# readout helpers (views in the same terms the device state uses)
# ----------------------------------------------------------------------------------
def segment_count(n: int, s: int) -> int:
    """Complete segments of scale s among n retained rows."""
    return n // s


def softmax_scale_for(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
