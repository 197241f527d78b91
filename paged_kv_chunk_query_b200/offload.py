"""Chunk schedule for KV and gradients resident in pinned host memory.

"Out of the Memory Barrier" ([pt] §2D "Offloading Assíncrono de KV Cache para
CPU": dedicated streams and pinned memory move data while computation runs;
for sparse attention the page ids are known early, so the transfer overlaps
other work; [es] §2B "Descarga Asíncrona a CPU": KV and its gradients are
offloaded; [it] §2C).  This module only orders calls into the C ABI on two
CUDA streams; every copy and every computation runs inside liboomb.so.

Pools: a pinned-host pool holds every page's K/V and fp32 gradients (its page
representatives stay on the device); a small device staging pool holds, per
chunk, the pages Top-K kept for each KV-head group and the chunk's own pages.
The staging pool has three parts used by chunks in turn, so chunk c+1's
prefetch fills one part while chunk c computes on another and chunk c-1's
gradients drain from the third.

Per chunk c (compute stream C, copy stream S; part = c % 3):
  C: wait for prefetch(c); append K_c, V_c into the part's current pages
     (page summaries, zeroed gradient blocks)
  S: store those pages and summaries into the host pool
  S: Top-K for chunk c+1 against the host pool's summaries; selection -> host
  C: forward + backward of chunk c on the staging part
  host: wait for the selection of c+1, build the block lists
  S: prefetch chunk c+1's selected blocks into part (c+1) % 3, then write
     back chunk c-1's gradient deltas (D2H, zero-fill; the host add runs on
     the library's worker thread)
Part (c+1) % 3 was last used by chunk c-2, whose write-back (issued in
iteration c-1, earlier on S) has drained and zeroed its gradient blocks.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


class OffloadRun:
    def __init__(self, w, device, host_pool=None):
        self.w, self.dev = w, device
        P, Hkv, d = w.page_size, w.num_kv_heads, w.head_dim
        self.sel_max = w.top_k + w.n_recent
        self.ppc = w.pages_per_chunk
        self.parts = 3
        self.half = self.sel_max + self.ppc           # staging pages per part
        self.host = host_pool or L.pool_create(w.num_pages, P, Hkv, d, L.LOC_PINNED_HOST, True,
                                               w.alloc_seed, device.index or 0)
        self.own_host = host_pool is None
        self.stage = L.pool_create(self.parts * self.half, P, Hkv, d, L.LOC_DEVICE, True, 0,
                                   device.index or 0)
        self.stage_pages = np.array([L.pool_alloc_page(self.stage)
                                     for _ in range(self.parts * self.half)], dtype=np.int64)
        self.table = np.array([L.pool_alloc_page(self.host) for _ in range(w.num_chunks * self.ppc)],
                              dtype=np.int64)
        self.table_dev = torch.tensor(self.table, dtype=torch.int32, device=device)
        self.copy = torch.cuda.Stream(device=device)
        C, Hq = w.chunk_len, w.num_q_heads
        self.sel_l = torch.zeros((Hkv, self.sel_max), dtype=torch.int32, device=device)
        self.sel_n = torch.zeros(Hkv, dtype=torch.int32, device=device)
        self.sel_host = torch.zeros((Hkv * self.sel_max + Hkv,), dtype=torch.int32).pin_memory()
        ws = L.page_topk_workspace_size(C, Hq, Hkv, d, max(1, (w.num_chunks - 1) * self.ppc))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.delta = torch.empty((Hq, C), dtype=torch.float32, device=device)
        n = self.parts
        self.cur_dev = [torch.tensor(self.stage_pages[b * self.half + self.sel_max:
                                                      (b + 1) * self.half],
                                     dtype=torch.int32, device=device) for b in range(n)]
        self.past_dev = [torch.zeros((Hkv, self.sel_max), dtype=torch.int32, device=device)
                         for _ in range(n)]
        # pinned upload buffers per part: rewritten three chunks after their last copy,
        # by which time the host has synchronised on later copy-stream events
        self.past_host = [torch.zeros((Hkv, self.sel_max), dtype=torch.int32).pin_memory()
                          for _ in range(n)]
        self.cnt_host = [torch.zeros(Hkv, dtype=torch.int32).pin_memory() for _ in range(n)]
        self.cnt_dev = [torch.zeros(Hkv, dtype=torch.int32, device=device) for _ in range(n)]
        self.h2d_bytes = 0
        self.d2h_bytes = 0
        self.selections = []

    def close(self):
        self.sync()
        L.pool_destroy(self.stage)
        if self.own_host:
            L.pool_destroy(self.host)

    # ---------------------------------------------------------------- helpers
    def _blocks_of_pages(self, pages):
        """Block ids (page * Hkv + head) of whole pages, page-major."""
        Hkv = self.w.num_kv_heads
        return (np.asarray(pages, dtype=np.int64)[:, None] * Hkv
                + np.arange(Hkv, dtype=np.int64)[None, :]).reshape(-1)

    def _select(self, c, q):
        """Top-K for chunk c on the copy stream; returns an event recorded after
        the selection was copied into pinned host memory."""
        w = self.w
        n_past = c * self.ppc
        Hkv = w.num_kv_heads
        ev = torch.cuda.Event()
        with torch.cuda.stream(self.copy):
            L.page_topk(self.host, q, self.table_dev[:n_past], n_past, w.top_k, w.n_recent,
                        self.sel_l, None, self.sel_n, self.ws, stream=self.copy)
            self.sel_host[:Hkv * self.sel_max].copy_(self.sel_l.view(-1), non_blocking=True)
            self.sel_host[Hkv * self.sel_max:].copy_(self.sel_n, non_blocking=True)
            ev.record(self.copy)
        return ev

    def _read_selection(self, ev):
        ev.synchronize()
        Hkv = self.w.num_kv_heads
        ids = self.sel_host[:Hkv * self.sel_max].view(Hkv, self.sel_max).numpy()
        cnt = self.sel_host[Hkv * self.sel_max:].numpy()
        return [ids[g, :cnt[g]].tolist() for g in range(Hkv)]

    def _prefetch(self, c, sel):
        """Selected blocks of chunk c into staging part c % 3 (copy stream)."""
        b = c % self.parts
        Hkv = self.w.num_kv_heads
        counts = np.array([len(x) for x in sel], dtype=np.int64)
        slots = self.stage_pages[b * self.half: b * self.half + self.sel_max]
        past = self.past_host[b].numpy()
        past[:] = 0
        # slot-major order: staging blocks (slot i, head g) are consecutive, so the
        # gradient write-back of these blocks is one large device->host copy
        src, dst = [], []
        for i in range(int(counts.max()) if len(counts) else 0):
            gs = np.nonzero(counts > i)[0]
            lp = np.array([sel[g][i] for g in gs], dtype=np.int64)
            src.append(self.table[lp] * Hkv + gs)
            dst.append(slots[i] * Hkv + gs)
            past[gs, i] = slots[i]
        src = np.concatenate(src) if src else np.zeros(0, dtype=np.int64)
        dst = np.concatenate(dst) if dst else np.zeros(0, dtype=np.int64)
        self.cnt_host[b].numpy()[:] = counts
        ev = torch.cuda.Event()
        with torch.cuda.stream(self.copy):
            self.past_dev[b].copy_(self.past_host[b], non_blocking=True)
            self.cnt_dev[b].copy_(self.cnt_host[b], non_blocking=True)
            L.page_prefetch(self.host, self.stage, src, dst, stream=self.copy, done_event=ev)
        self.h2d_bytes += len(src) * 2 * self.w.page_size * self.w.head_dim * 2
        return ev, (src, dst)

    def _writeback(self, c, blocks):
        """Gradient deltas of chunk c back into the host pool (copy stream)."""
        src, dst = blocks
        with torch.cuda.stream(self.copy):
            L.grad_writeback(self.stage, self.host, src, dst, stream=self.copy)
        self.d2h_bytes += len(src) * 2 * self.w.page_size * self.w.head_dim * 4

    # ---------------------------------------------------------------- run
    def run(self, chunks, outputs=None, backward=True):
        """chunks(c) -> dict of device tensors q, k, v, do; outputs(c) -> (o, lse,
        dq) device tensors to fill, or None to use scratch buffers."""
        w = self.w
        N, Hkv = w.num_chunks, w.num_kv_heads
        comp = torch.cuda.current_stream(self.dev)
        scratch = None
        pending = None          # (prefetch event, (host blocks, staging blocks)) of chunk c
        prev = None             # (computed event, gradient blocks) of chunk c-1
        self.selections = [[[] for _ in range(Hkv)]]
        empty = np.zeros(0, dtype=np.int64)
        for c in range(N):
            b = c % self.parts
            x = chunks(c)
            cur_pages = self.stage_pages[b * self.half + self.sel_max:(b + 1) * self.half]
            if outputs is not None:
                o, lse, dq = outputs(c)
            else:
                if scratch is None:
                    scratch = (torch.empty_like(x["q"]),
                               torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32,
                                           device=self.dev), torch.empty_like(x["q"]))
                o, lse, dq = scratch
            if pending is not None:
                comp.wait_event(pending[0])
            pf_blocks = pending[1] if pending is not None else (empty, empty)
            # append chunk c into the part's current pages; store them on the host
            L.kv_append(self.stage, self.cur_dev[b], x["k"], x["v"], comp)
            appended = torch.cuda.Event()
            appended.record(comp)
            store_src = self._blocks_of_pages(cur_pages)
            store_dst = self._blocks_of_pages(self.table[c * self.ppc:(c + 1) * self.ppc])
            self.copy.wait_event(appended)
            L.page_prefetch(self.stage, self.host, store_src, store_dst, stream=self.copy)
            self.d2h_bytes += len(store_src) * 2 * w.page_size * w.head_dim * 2
            # Top-K of chunk c+1 (every earlier page's summary is now on the host side)
            ev_sel = self._select(c + 1, chunks(c + 1)["q"]) if c + 1 < N else None
            past = self.past_dev[b] if c else None
            cnt = self.cnt_dev[b] if c else None
            L.chunk_attn_fwd(self.stage, x["q"], o, lse, past, cnt, self.cur_dev[b],
                             w.softmax_scale, comp)
            if backward:
                L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, self.delta, past, cnt,
                                 self.cur_dev[b], w.softmax_scale, comp)
            computed = torch.cuda.Event()
            computed.record(comp)
            # gradient blocks of chunk c: its selected past blocks and its own pages
            grads = (np.concatenate([pf_blocks[1], store_src]),
                     np.concatenate([pf_blocks[0], store_dst]))
            if ev_sel is not None:
                sel_next = self._read_selection(ev_sel)
                self.selections.append(sel_next)
                # part (c+1) % 3 last served chunk c-2, drained by its write-back
                # (issued in iteration c-1, earlier on the copy stream)
                pending = self._prefetch(c + 1, sel_next)
            if backward and prev is not None:
                self.copy.wait_event(prev[0])
                self._writeback(c - 1, prev[1])
            prev = (computed, grads)
        if backward and prev is not None:
            self.copy.wait_event(prev[0])
            self._writeback(N - 1, prev[1])
        comp.wait_stream(self.copy)

    def sync(self):
        """Waits for the device and for every queued host gradient addition."""
        torch.cuda.synchronize(self.dev)
        L.grad_writeback_sync(self.stage)
