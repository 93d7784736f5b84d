"""A device runner for the synthetic workloads of the drafting round.

The workload recipes (``Workload``, ``CONFIGS``, the sweep) live in ``synth.workloads``
and are re-exported here. ``DeviceRun`` owns the torch allocations of one run (state arena, prefix chunks, all
rounds' inputs) and drives the library through the binding; it holds no arithmetic of
the method.
"""

from __future__ import annotations

import math
from dataclasses import replace

import numpy as np

import fixed_cost_drafter_b200 as F
from synth.workloads import (  # noqa: F401  (re-exported: the recipes live beside the generator)
    CONFIGS, QWEN3_8B, SWEEP_BATCHES, SWEEP_MEANS, SWEEP_PREFIXES, Workload, sweep_point)


class DeviceRun:
    """One workload on one GPU: state arena, generated inputs, calls into the library."""

    def __init__(self, wl: Workload, device="cuda", rounds: int | None = None,
                 prefill_chunk: int | None = None, prefix_override=None, accepts_override=None,
                 seq_offset: int = 0, kv_heads=None):
        """``kv_heads`` = (h0, h1): this run holds KV heads h0 .. h1 - 1 of every sequence (and
        their query heads), a KV-head shard of the workload; inputs are the same generated
        values as the whole run's, sliced by head."""
        import torch
        import synth
        self.torch, self.synth = torch, synth
        self.full_wl = wl
        self.h0 = 0
        if kv_heads is not None:
            h0, h1 = kv_heads
            if not 0 <= h0 < h1 <= wl.n_kv_heads:
                raise ValueError(f"KV heads {kv_heads} outside 0..{wl.n_kv_heads}")
            wl = replace(wl, n_kv_heads=h1 - h0, n_q_heads=(h1 - h0) * wl.group)
            self.h0 = h0
        self.wl = wl
        self.dev = torch.device(device)
        self.cfg = wl.config()
        self.layout = F.ls_get_layout(self.cfg)
        self.nbytes = F.ls_state_bytes(self.cfg)
        self.arena = torch.empty(self.nbytes, dtype=torch.uint8, device=self.dev)
        self.stream = torch.cuda.current_stream(self.dev)
        self.state = F.ls_init_state(self.cfg, self.arena, self.nbytes, self.stream)
        self.tdtype = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.rounds = wl.rounds if rounds is None else rounds
        self.b0 = int(seq_offset)  # generator coordinates of this run's first sequence
        self.prefix_len = (np.asarray(prefix_override, dtype=np.int64) if prefix_override is not None
                           else replace(wl, batch=self.b0 + wl.batch).prefix_lengths()[self.b0:])
        self.prefill_chunk = prefill_chunk
        # per-head scales of every KV head of the workload (a shard indexes them from h0)
        self.scale_host = (synth.head_scales(wl.seed, wl.n_layers, self.full_wl.n_kv_heads) if wl.head_scale
                           else None)
        self.scale_dev = (torch.from_numpy(self.scale_host).to(self.dev) if self.scale_host is not None
                          else None)
        nb = self.b0 + wl.batch
        acc = synth.accept_lengths(wl.seed, max(self.rounds, 1), nb, wl.block, wl.accept_mean)[:, self.b0:]
        if accepts_override is not None:
            acc = np.broadcast_to(np.asarray(accepts_override, dtype=np.int32).reshape(-1, 1),
                                  (max(self.rounds, 1), wl.batch)).copy() if np.ndim(accepts_override) == 1 \
                else np.asarray(accepts_override, dtype=np.int32)
        acc_all = np.zeros((max(self.rounds, 1), nb), dtype=np.int32)
        acc_all[:, self.b0:] = acc
        draft, target = synth.token_ids(wl.seed, max(self.rounds, 1), nb, wl.block, acc_all, wl.vocab)
        draft, target = draft[:, self.b0:], target[:, self.b0:]
        self.accept_host = acc[:self.rounds]
        self.draft = torch.from_numpy(draft[:self.rounds].copy()).to(self.dev)
        self.target = torch.from_numpy(target[:self.rounds].copy()).to(self.dev)
        self.accept_len = torch.zeros(wl.batch, dtype=torch.int32, device=self.dev)
        self.next_token = torch.zeros(wl.batch, dtype=torch.int32, device=self.dev)
        e = wl.elem()
        # boundary keys/values: this run's heads' slices [h0 D, ...) and [Hkv D + h0 D, ...)
        # of the (replicated) boundary hidden vector
        self.bk_off = self.h0 * wl.head_dim
        self.bv_off = (self.full_wl.n_kv_heads + self.h0) * wl.head_dim
        self.boundary_k = self.arena.data_ptr() + self.layout.off_boundary + self.bk_off * e
        self.boundary_v = self.arena.data_ptr() + self.layout.off_boundary + self.bv_off * e
        self.softmax_scale = 1.0 / math.sqrt(wl.head_dim)

    # ---- generated inputs -------------------------------------------------------
    def _fill(self, t, tensor_id, shape, head_dim, r0=0, b0=0, l0=0, p0=0, scaled=False, x0=0):
        self.synth.device_fill_normal(
            t.data_ptr(), self.wl.seed, tensor_id, shape, r0=r0, b0=self.b0 + b0, l0=l0, p0=p0,
            head_dim=head_dim,
            scale_ptr=self.scale_dev.data_ptr() if (scaled and self.scale_dev is not None) else None,
            scale_heads=self.full_wl.n_kv_heads, dtype=self.wl.dtype, stream=self.stream.cuda_stream, x0=x0,
            scale_layers=self.wl.n_layers)

    @property
    def kv_x0(self):
        """First K/V row column of this run's heads in the workload's rows."""
        return self.h0 * self.wl.head_dim

    @property
    def q_x0(self):
        """First query column of this run's query heads."""
        return self.h0 * self.wl.group * self.wl.head_dim

    def chunk_bounds(self):
        """[(row_begin, row_end)]: the prefill chunks, whole largest-scale segments each."""
        P = self.prefix_len
        pmax = int(P.max()) if len(P) else 0
        chunk = self.prefill_chunk or max(pmax, 1)
        smax = self.wl.scales[-1]
        chunk = max(smax, (chunk // smax) * smax) if pmax > chunk else chunk
        out, rb = [], 0
        while True:
            re_ = min(rb + chunk, pmax)
            out.append((rb, re_))
            if re_ >= pmax:
                return out
            rb = re_

    def prefix_chunks(self):
        """Yields (row_begin, row_end, k, v): the generated prefix chunk by chunk,
        k/v [b][L][rows][Hkv*D]."""
        torch, wl, S = self.torch, self.wl, self.synth
        rowel = wl.n_kv_heads * wl.head_dim
        for rb, re_ in self.chunk_bounds():
            n = max(re_ - rb, 0)
            k = torch.empty((wl.batch, wl.n_layers, max(n, 1), rowel), dtype=self.tdtype, device=self.dev)
            v = torch.empty_like(k)
            if n:
                self._fill(k, S.PREFIX_K, (1, wl.batch, wl.n_layers, n, rowel), wl.head_dim, p0=rb, scaled=True,
                           x0=self.kv_x0)
                self._fill(v, S.PREFIX_V, (1, wl.batch, wl.n_layers, n, rowel), wl.head_dim, p0=rb, scaled=True,
                           x0=self.kv_x0)
            yield rb, re_, k, v
            del k, v

    def _last_hidden(self):
        wl = self.wl
        last_hidden = self.torch.empty((wl.batch, wl.n_layers, wl.hidden), dtype=self.tdtype, device=self.dev)
        self._fill(last_hidden, self.synth.LAST_HIDDEN, (1, wl.batch, wl.n_layers, 1, wl.hidden), 0)
        return last_hidden

    def _prefill_bytes(self, rb, re_):
        wl = self.wl
        rows = int(np.maximum(np.minimum(self.prefix_len, re_) - rb, 0).sum())
        return rows * wl.n_layers * wl.n_kv_heads * wl.head_dim * 2 * wl.elem()

    def prefill(self, timer=None):
        """Generates the prefix (in chunks when asked) and runs ls_prefill_summary over it.

        ``timer``, if given, is called as ``timer(start_event, end_event, bytes)`` around each
        library call (generation excluded)."""
        torch, wl = self.torch, self.wl
        pmax = int(self.prefix_len.max()) if len(self.prefix_len) else 0
        plen = torch.from_numpy(self.prefix_len).to(self.dev)
        last_hidden = self._last_hidden()
        rowel = wl.n_kv_heads * wl.head_dim
        for rb, re_, k, v in self.prefix_chunks():
            n = max(re_ - rb, 0)
            wsb = F.ls_prefill_workspace_bytes(self.cfg, rb, re_)
            ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=self.dev)
            last = re_ >= pmax
            if timer is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
            F.ls_prefill_summary(self.state, k, v, max(n, 1) * rowel, rowel, plen, rb, re_,
                                 last_hidden if last else None, ws, wsb, self.stream)
            if timer is not None:
                e1.record(self.stream)
                timer(e0, e1, self._prefill_bytes(rb, re_))
            del ws
        self.last_hidden = last_hidden

    def fill_pages(self, cache):
        """Writes the generated prefix into a PagedCache (what the target's prefill leaves)."""
        for rb, re_, k, v in self.prefix_chunks():
            for b in range(self.wl.batch):
                hi = min(re_, int(self.prefix_len[b]))
                if hi > rb:
                    cache.write(b, rb, k[b, :, :hi - rb], v[b, :, :hi - rb])

    def prefill_paged(self, cache, timer=None, workspace=True):
        """ls_prefill_paged over the prefix already in ``cache`` (same chunks as ``prefill``;
        ``workspace`` False uses the library's fixed scratch)."""
        torch = self.torch
        pmax = int(self.prefix_len.max()) if len(self.prefix_len) else 0
        plen = torch.from_numpy(self.prefix_len).to(self.dev)
        last_hidden = self._last_hidden()
        kv = cache.descriptor()
        for rb, re_ in self.chunk_bounds():
            wsb = F.ls_prefill_workspace_bytes(self.cfg, rb, re_)
            ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=self.dev) if workspace else None
            last = re_ >= pmax
            if timer is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
            F.ls_prefill_paged(self.state, kv, plen, rb, re_, last_hidden if last else None, ws,
                               wsb if workspace else 0, self.stream)
            if timer is not None:
                e1.record(self.stream)
                timer(e0, e1, self._prefill_bytes(rb, re_))
        self.last_hidden = last_hidden
        self.paged_len = self.prefix_len.copy()

    def make_round_inputs(self, r0=0, n=None):
        """All inputs of rounds [r0, r0+n): verify K/V/hidden and drafter queries."""
        torch, wl, S = self.torch, self.wl, self.synth
        n = self.rounds - r0 if n is None else n
        B1 = wl.block + 1
        rowel = wl.n_kv_heads * wl.head_dim
        vk = torch.empty((n, wl.batch, wl.n_layers, B1, rowel), dtype=self.tdtype, device=self.dev)
        vv = torch.empty_like(vk)
        vh = torch.empty((n, wl.batch, wl.n_layers, B1, wl.hidden), dtype=self.tdtype, device=self.dev)
        q = torch.empty((n, wl.batch, wl.n_layers, wl.block, wl.n_q_heads * wl.head_dim),
                        dtype=self.tdtype, device=self.dev)
        self._fill(vk, S.VERIFY_K, (n, wl.batch, wl.n_layers, B1, rowel), wl.head_dim, r0=r0, scaled=True,
                   x0=self.kv_x0)
        self._fill(vv, S.VERIFY_V, (n, wl.batch, wl.n_layers, B1, rowel), wl.head_dim, r0=r0, scaled=True,
                   x0=self.kv_x0)
        self._fill(vh, S.VERIFY_HIDDEN, (n, wl.batch, wl.n_layers, B1, wl.hidden), 0, r0=r0)
        self._fill(q, S.QUERY, (n, wl.batch, wl.n_layers, wl.block, wl.n_q_heads * wl.head_dim),
                   wl.head_dim, r0=r0, x0=self.q_x0)
        return dict(vk=vk, vv=vv, vh=vh, q=q, r0=r0)

    def write_verify_pages(self, cache, inputs, r):
        """The target's verify pass of round r into ``cache``: its B + 1 K/V rows at the
        sequences' positions len .. len + B; len then advances by the round's a + 1."""
        i = r - inputs["r0"]
        for b in range(self.wl.batch):
            cache.write(b, int(self.paged_len[b]), inputs["vk"][i][b], inputs["vv"][i][b])
        if not hasattr(self, "verify_slots"):
            self.verify_slots = {}
        self.verify_slots[r] = cache.slots(self.paged_len, self.wl.block + 1)
        self.paged_len = self.paged_len + self.accept_host[r] + 1

    def paged_descriptor(self, cache, r, with_slots=False):
        """The cache's descriptor, with round r's verify slots when asked."""
        return cache.descriptor(self.verify_slots[r] if with_slots else None)

    def commit_paged(self, cache, inputs, r, with_slots=False):
        """ls_commit_round_paged of round r (its verify rows already written to ``cache``),
        reading them through the block table or, with_slots, at the slots the write used."""
        i = r - inputs["r0"]
        F.ls_commit_round_paged(self.state, self.draft[r], self.target[r], self.paged_descriptor(cache, r, with_slots),
                                inputs["vh"][i], self.accept_len, self.next_token, self.stream)

    def commit(self, inputs, r):
        i = r - inputs["r0"]
        F.ls_commit_round(self.state, self.draft[r], self.target[r], inputs["vk"][i], inputs["vv"][i],
                          inputs["vh"][i], self.accept_len, self.next_token, self.stream)

    def attend(self, inputs, r, out, layer_begin=0, layer_count=None, views=None):
        """ls_draft_attend (views None) or ls_draft_attend_views with an LS_VIEW_* mask."""
        wl = self.wl
        lc = wl.n_layers if layer_count is None else layer_count
        i = r - inputs["r0"]
        q = inputs["q"][i]
        if lc != wl.n_layers or layer_begin != 0:
            q = q[:, layer_begin:layer_begin + lc].contiguous()
        if views is None:
            F.ls_draft_attend(self.state, layer_begin, lc, q, self.boundary_k, self.boundary_v, wl.hidden,
                              self.softmax_scale, out, self.stream)
        else:
            F.ls_draft_attend_views(self.state, layer_begin, lc, q, self.boundary_k, self.boundary_v, wl.hidden,
                                    self.softmax_scale, views, out, self.stream)

    def round(self, inputs, r, out):
        """ls_round: commit and attention over all layers in one call (boundary keys and
        values are this run's heads' slices of [0, Hkv*D) and [Hkv*D, 2*Hkv*D) of the
        boundary hidden)."""
        i = r - inputs["r0"]
        F.ls_round(self.state, self.draft[r], self.target[r], inputs["vk"][i], inputs["vv"][i], inputs["vh"][i],
                   self.accept_len, self.next_token, inputs["q"][i], self.bk_off, self.bv_off,
                   self.softmax_scale, out, self.stream)

    def new_out(self, layer_count=None):
        wl = self.wl
        lc = wl.n_layers if layer_count is None else layer_count
        dt = self.torch.float32 if (wl.flags & F.LS_FLAG_OUT_F32) else self.tdtype
        return self.torch.empty((wl.batch, lc, wl.block, wl.n_q_heads * wl.head_dim), dtype=dt, device=self.dev)

    # ---- readout ----------------------------------------------------------------
    def read_state(self):
        """The arena as numpy views: counters, kv rows, fp32 summary, boundary."""
        torch, wl, y = self.torch, self.wl, self.layout
        host = torch.empty(self.nbytes, dtype=torch.uint8, pin_memory=True)
        F.ls_read_state(self.state, host, self.nbytes, self.stream)
        raw = host.numpy()
        b, L, H, D, nsc, sl = wl.batch, wl.n_layers, wl.n_kv_heads, wl.head_dim, len(wl.scales), wl.slots
        ed = np.uint16 if wl.dtype == "bf16" else np.float32

        def view(off, dt, shape):
            n = int(np.prod(shape)) * np.dtype(dt).itemsize
            return raw[off:off + n].view(dt).reshape(shape)

        return dict(
            counters=view(y.off_counters, np.int64, (b, L, 1 + nsc)).copy(),
            kv=view(y.off_kv, ed, (b, L, H, 2, y.kv_rows, D)).copy(),
            seg=view(y.off_seg_mean, np.float32, (b, L, H, nsc, sl, 2, D)).copy(),
            part=view(y.off_part_sum, np.float32, (b, L, H, nsc, 2, D)).copy(),
            glob=view(y.off_glob_sum, np.float32, (b, L, H, 2, D)).copy(),
            boundary=view(y.off_boundary, ed, (b, L, wl.hidden)).copy(),
        )

    def reset_state(self):
        """A fresh state in the same arena (ls_init_state zeroes it): nothing retained."""
        F.ls_destroy_state(self.state)
        self.state = F.ls_init_state(self.cfg, self.arena, self.nbytes, self.stream)

    def error(self):
        return F.ls_get_error(self.state)

    def close(self):
        if self.state:
            F.ls_destroy_state(self.state)
            self.state = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PagedCache:
    """A target's paged KV cache of the tapped layers, as an inference engine keeps it.

    Pages are handed out to the sequences from a seeded permutation of the pool, so a
    sequence's pages are scattered and interleaved with other sequences' pages. Layouts:
    ``packed``      per layer K and V tensors [num_pages][page_size][Hkv*D];
    ``interleaved`` per layer one tensor [num_pages][2][page_size][Hkv*D] (K then V per page);
    ``padded``      packed with each slot padded to Hkv*D + 64 elements (rows not back to back).
    Positions 0 .. capacity[b] - 1 of sequence b have pages; other block-table entries are -1.
    """

    def __init__(self, run: DeviceRun, page_size: int, capacity, layout: str = "packed", spare_pages: int = 3,
                 seed: int = 0):
        torch, wl = run.torch, run.wl
        self.torch, self.page_size, self.layout = torch, int(page_size), layout
        rowel = wl.n_kv_heads * wl.head_dim
        self.rowel = rowel
        cap = np.asarray(capacity, dtype=np.int64)
        n_b = -(-cap // page_size)
        self.max_blocks = max(int(n_b.max()), 1)
        self.num_pages = int(n_b.sum()) + spare_pages
        perm = np.random.default_rng(seed).permutation(self.num_pages)
        table = np.full((wl.batch, self.max_blocks), -1, dtype=np.int32)
        o = 0
        for b in range(wl.batch):
            table[b, :n_b[b]] = perm[o:o + n_b[b]]
            o += n_b[b]
        self.table_host = table
        self.block_table = torch.from_numpy(table).to(run.dev)
        NP, PS = self.num_pages, self.page_size
        self.k, self.v, self.bufs = [], [], []
        for _ in range(wl.n_layers):
            if layout == "interleaved":
                t = torch.zeros((NP, 2, PS, rowel), dtype=run.tdtype, device=run.dev)
                self.bufs.append(t)
                self.k.append(t[:, 0])
                self.v.append(t[:, 1])
            else:
                slot = rowel + (64 if layout == "padded" else 0)
                tk = torch.zeros((NP, PS, slot), dtype=run.tdtype, device=run.dev)
                tv = torch.zeros_like(tk)
                self.bufs += [tk, tv]
                self.k.append(tk[..., :rowel])
                self.v.append(tv[..., :rowel])
        self.slot_stride = self.k[0].stride(1)
        self.page_stride = self.k[0].stride(0)
        self._desc = F.make_paged_kv([t.data_ptr() for t in self.k], [t.data_ptr() for t in self.v],
                                     self.page_stride, self.slot_stride, self.block_table, self.max_blocks,
                                     self.page_size, self.num_pages)

    def descriptor(self, verify_slots=None):
        """The ls_paged_kv descriptor; with ``verify_slots`` (int64 [b][B+1]) set in a copy."""
        if verify_slots is None:
            return self._desc
        d = F.ls_paged_kv.from_buffer_copy(self._desc)
        d.verify_slots = verify_slots.data_ptr()
        return d

    def slots(self, lens, n):
        """int64 [b][n] device tensor: slots (page * page_size + offset) of positions
        lens[b] .. lens[b] + n - 1, as an engine's slot mapping holds them."""
        out = np.zeros((len(lens), n), dtype=np.int64)
        for b, p0 in enumerate(lens):
            pg, off = self.locate(b, int(p0), n)
            out[b] = pg * self.page_size + off
        return self.torch.from_numpy(out).to(self.block_table.device)

    def locate(self, b: int, p0: int, n: int):
        """(pages, offsets) of positions p0 .. p0 + n - 1 of sequence b (host arrays)."""
        pos = np.arange(p0, p0 + n)
        return self.table_host[b, pos // self.page_size].astype(np.int64), pos % self.page_size

    def write(self, b: int, p0: int, k_rows, v_rows):
        """Rows [L][n][Hkv*D] of sequence b at positions p0 .. p0 + n - 1, every layer."""
        n = k_rows.shape[1]
        pg, off = self.locate(b, p0, n)
        assert (pg >= 0).all(), "position beyond the sequence's pages"
        pg = self.torch.from_numpy(pg).to(k_rows.device)
        off = self.torch.from_numpy(off).to(k_rows.device)
        for l in range(len(self.k)):
            self.k[l][pg, off] = k_rows[l]
            self.v[l][pg, off] = v_rows[l]
