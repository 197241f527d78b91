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

Nothing goes through the host between Top-K and the prefetch: the selection
stays on the device, oomb_prefetch_lists turns it into block lists, and
oomb_block_copy / oomb_grad_block_add move the blocks by reading and writing
the pinned pages in place (one launch per list).  The host only enqueues.

Per chunk c (compute stream C, copy stream S and write-back stream W with
higher priority; part = c % 3):
  C: wait for prefetch(c); append K_c, V_c into the part's current pages
     (page summaries, zeroed gradient blocks)
  S: store those pages and summaries into the host pool
  S: Top-K for chunk c+1 against the host pool's summaries, its block lists,
     and the prefetch of its blocks into part (c+1) % 3
  C: forward, backward preprocess and dK/dV of chunk c on the staging part;
     its dQ on a third stream D beside the dK/dV launch (each fills the
     other's last partial wave of CTAs, as in the device-resident step)
  W: once chunk c-1 has computed, add its gradient blocks into the host pool
     and zero them on the device
The write-backs have their own stream so that the prefetch chain of the next
chunk (store, Top-K, lists, gather on S) does not queue behind a write-back:
on one copy stream the compute stream waited about 0.3 ms per chunk for its
prefetch.  Part (c+1) % 3 was last used by chunk c-2: S waits for that
chunk's write-back (which reads the part's block lists and zeroes its
gradient blocks) before rebuilding the lists, and C waits for its dQ before
chunk c's append (after which S starts overwriting the part).  Delta, O, LSE
and dQ scratch are per part, since chunk c's dQ may still read its LSE and
delta while chunk c+1 runs on C.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


class OffloadRun:
    def __init__(self, w, device, host_pool=None):
        self.w, self.dev = w, device
        P, Hkv, d = w.page_size, w.num_kv_heads, w.head_dim
        N = w.num_chunks
        self.sel_max = w.top_k + w.n_recent
        self.ppc = w.pages_per_chunk
        self.parts = 3
        self.half = self.sel_max + self.ppc           # staging pages per part
        self.host = host_pool or L.pool_create(w.num_pages, P, Hkv, d, L.LOC_PINNED_HOST, True,
                                               w.alloc_seed, device.index or 0)
        self.own_host = host_pool is None
        self.stage = L.pool_create(self.parts * self.half, P, Hkv, d, L.LOC_DEVICE, True, 0,
                                   device.index or 0)
        stage_pages = np.array([L.pool_alloc_page(self.stage)
                                for _ in range(self.parts * self.half)], dtype=np.int64)
        self.table = np.array([L.pool_alloc_page(self.host) for _ in range(N * self.ppc)],
                              dtype=np.int64)
        i32 = dict(dtype=torch.int32, device=device)
        self.table_dev = torch.tensor(self.table, **i32)
        # a higher-priority copy stream: its short kernels take SMs as soon as
        # an attention CTA retires
        self.copy = torch.cuda.Stream(device=device, priority=-1)
        self.wb = torch.cuda.Stream(device=device, priority=-1)   # gradient write-backs
        self.side = torch.cuda.Stream(device=device)   # each chunk's dQ
        C, Hq = w.chunk_len, w.num_q_heads
        heads = np.arange(Hkv, dtype=np.int64)

        def blocks(pages):  # page-major block ids of whole pages
            return (np.asarray(pages, dtype=np.int64)[:, None] * Hkv + heads[None, :]).reshape(-1)

        n = self.parts
        slots = [stage_pages[b * self.half: b * self.half + self.sel_max] for b in range(n)]
        cur = [stage_pages[b * self.half + self.sel_max:(b + 1) * self.half] for b in range(n)]
        self.slots_dev = [torch.tensor(x, **i32) for x in slots]
        self.cur_dev = [torch.tensor(x, **i32) for x in cur]
        self.cur_blocks = [torch.tensor(blocks(x), **i32) for x in cur]
        # host blocks of every chunk's own pages, [N][ppc * Hkv]
        self.own_host_blocks = torch.tensor(blocks(self.table).reshape(N, -1), **i32)
        self.sel_l = [torch.zeros((Hkv, self.sel_max), **i32) for _ in range(n)]
        self.cnt_dev = [torch.zeros(Hkv, **i32) for _ in range(n)]
        self.past_dev = [torch.zeros((Hkv, self.sel_max), **i32) for _ in range(n)]
        self.pf_src = [torch.full((self.sel_max * Hkv,), -1, **i32) for _ in range(n)]
        self.pf_dst = [torch.full((self.sel_max * Hkv,), -1, **i32) for _ in range(n)]
        ws = L.page_topk_workspace_size(C, Hq, Hkv, d, max(1, (N - 1) * self.ppc))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.deltas = [torch.empty((Hq, C), dtype=torch.float32, device=device)
                       for _ in range(n)]
        # forward workspace (split last wave); every forward runs on the compute stream
        self.fwd_ws = L.fwd_workspace(d, device)
        # every chunk's selection, copied back for inspection (not on the schedule's path)
        self.sel_hist = torch.zeros((N, Hkv, self.sel_max), dtype=torch.int32).pin_memory()
        self.cnt_hist = torch.zeros((N, Hkv), dtype=torch.int32).pin_memory()

    def close(self):
        self.sync()
        L.pool_destroy(self.stage)
        if self.own_host:
            L.pool_destroy(self.host)

    # ---------------------------------------------------------------- run
    def run(self, chunks, outputs=None, backward=True):
        """chunks(c) -> dict of device tensors q, k, v, do; outputs(c) -> (o, lse,
        dq) device tensors to fill, or None to use scratch buffers."""
        w = self.w
        N = w.num_chunks
        comp = torch.cuda.current_stream(self.dev)
        S, D, W = self.copy, self.side, self.wb
        scratch = [None] * self.parts
        dq_done = [None] * self.parts   # event: the dQ of the part's last chunk has finished
        self.wb_done = [None] * self.parts  # event: the part's last write-back has finished
        prefetched = None       # event: chunk c's blocks are in its staging part
        prev_computed = None    # event: chunk c-1's backward has finished
        self.copy.wait_stream(comp)
        D.wait_stream(comp)
        W.wait_stream(comp)
        for c in range(N):
            b = c % self.parts
            x = chunks(c)
            if outputs is not None:
                o, lse, dq = outputs(c)
            else:
                if scratch[b] is None:
                    scratch[b] = (torch.empty_like(x["q"]),
                                  torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32,
                                              device=self.dev), torch.empty_like(x["q"]))
                o, lse, dq = scratch[b]
            if prefetched is not None:
                comp.wait_event(prefetched)
            b2 = (c + 1) % self.parts   # the part chunk c+1's prefetch overwrites (chunk c-2's)
            if dq_done[b2] is not None:
                comp.wait_event(dq_done[b2])
            L.kv_append(self.stage, self.cur_dev[b], x["k"], x["v"], comp)
            appended = torch.cuda.Event()
            appended.record(comp)
            S.wait_event(appended)
            # chunk c's pages (and their representatives) into the host pool
            L.block_copy(self.stage, self.host, self.cur_blocks[b], self.own_host_blocks[c],
                         stream=S)
            if c + 1 < N:
                b1 = (c + 1) % self.parts
                n_past = (c + 1) * self.ppc
                L.page_topk(self.host, chunks(c + 1)["q"], self.table_dev[:n_past], n_past,
                            w.top_k, w.n_recent, self.sel_l[b1], None, self.cnt_dev[b1], self.ws,
                            stream=S)
                if self.wb_done[b1] is not None:   # chunk c-2's write-back read these lists
                    S.wait_event(self.wb_done[b1])
                L.prefetch_lists(self.host, self.stage, self.sel_l[b1], self.cnt_dev[b1],
                                 self.table_dev[:n_past], self.slots_dev[b1], self.pf_src[b1],
                                 self.pf_dst[b1], self.past_dev[b1], stream=S)
                L.block_copy(self.host, self.stage, self.pf_src[b1], self.pf_dst[b1], stream=S)
                prefetched = torch.cuda.Event()
                prefetched.record(S)
                with torch.cuda.stream(S):
                    self.sel_hist[c + 1].copy_(self.sel_l[b1], non_blocking=True)
                    self.cnt_hist[c + 1].copy_(self.cnt_dev[b1], non_blocking=True)
            past = self.past_dev[b] if c else None
            cnt = self.cnt_dev[b] if c else None
            L.chunk_attn_fwd(self.stage, x["q"], o, lse, past, cnt, self.cur_dev[b],
                             w.softmax_scale, comp, fwd_ws=self.fwd_ws)
            if backward:
                delta = self.deltas[b]
                L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta, past, cnt,
                                 self.cur_dev[b], w.softmax_scale, comp, step=L.BWD_PREPROCESS)
                D.wait_stream(comp)
                L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta, past, cnt,
                                 self.cur_dev[b], w.softmax_scale, D, step=L.BWD_DQ)
                dq_done[b] = torch.cuda.Event()
                dq_done[b].record(D)
                L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta, past, cnt,
                                 self.cur_dev[b], w.softmax_scale, comp, step=L.BWD_DKDV)
                computed = torch.cuda.Event()
                computed.record(comp)
                if prev_computed is not None:
                    self._writeback(c - 1, prev_computed)
                prev_computed = computed
        if backward and prev_computed is not None:
            self._writeback(N - 1, prev_computed)
        comp.wait_stream(S)
        comp.wait_stream(D)
        comp.wait_stream(W)

    def _writeback(self, c, computed):
        """Chunk c's gradient blocks (its prefetched blocks and its own pages)
        added into the host pool on the write-back stream, zeroed on the
        device."""
        b = c % self.parts
        W = self.wb
        W.wait_event(computed)
        if c > 0:
            L.grad_block_add(self.stage, self.host, self.pf_dst[b], self.pf_src[b], True, stream=W)
        L.grad_block_add(self.stage, self.host, self.cur_blocks[b], self.own_host_blocks[c], True,
                         stream=W)
        self.wb_done[b] = torch.cuda.Event()
        self.wb_done[b].record(W)

    def sync(self):
        """Waits for the device (every copy and gradient addition is stream-ordered)."""
        torch.cuda.synchronize(self.dev)

    # ---------------------------------------------------------------- inspection
    @property
    def selections(self):
        """Per chunk, per group, the kept logical page ids (after sync())."""
        out = [[[] for _ in range(self.w.num_kv_heads)]]
        for c in range(1, self.w.num_chunks):
            cnt = self.cnt_hist[c].tolist()
            out.append([self.sel_hist[c, g, :cnt[g]].tolist() for g in range(len(cnt))])
        return out

    def link_bytes(self, backward=True):
        """(host->device, device->host) bytes one run moves over the host link
        (after sync()): prefetched KV blocks and the host gradients read for
        the additions; stored KV blocks and the gradients written back."""
        w = self.w
        kv_block = 2 * w.page_size * w.head_dim * 2
        g_block = 2 * w.page_size * w.head_dim * 4
        sel = int(self.cnt_hist[1:].sum())
        own = w.num_chunks * self.ppc * w.num_kv_heads
        h2d = sel * kv_block + ((sel + own) * g_block if backward else 0)
        d2h = own * kv_block + ((sel + own) * g_block if backward else 0)
        return h2d, d2h


def plan_segments(n_past, window):
    """The calls that take a chunk's past of n_past pages through a window of
    `window` pages: [(segment mode, first page, pages)], in order, covering
    [0, n_past) once; the last call also carries the chunk itself.  No past or
    a single segment is one whole-key-set call."""
    segs = [(a, min(window, n_past - a)) for a in range(0, n_past, window)]
    if len(segs) <= 1:
        return [(L.SEG_WHOLE,) + (segs[0] if segs else (0, 0))]
    modes = [L.SEG_FIRST] + [L.SEG_NEXT] * (len(segs) - 2) + [L.SEG_LAST]
    return [(m, a, n) for m, (a, n) in zip(modes, segs)]


class DenseOffloadRun:
    """Dense attention with KV and gradients in pinned host memory and a
    bounded device window ([pt] §2D: pages move between host and GPU on
    dedicated streams while computation runs; the pages' dense-model case).

    The device holds ``slots`` slots of ``window`` pages each plus two sets
    of the chunk's own pages.  A chunk's past is taken in segments of
    ``window`` pages: the forward merges them into an fp32 running output
    (oomb segment modes, FIRST / NEXT / LAST, the last with the chunk itself),
    then the backward streams the same segments again, and each segment's
    gradient blocks are added into the host pool (and zeroed) as soon as its
    backward is done.  Calls take the slots in turn, and each call's pages
    are fetched ``slots - 1`` calls ahead on a fetch stream (higher priority),
    while a write-back stream stores the chunk's own pages and returns the
    gradients, so the link's two directions run at once and a fetch never
    queues behind a gradient copy.  The chunk's own pages are appended on the
    device, stored to the host pool, and their gradients added back after the
    chunk's backward.

    Host pages are taken in logical order (and the slots' pages in order), so
    a segment is one contiguous range in both pools: its K/V travel as one
    copy-engine transfer (oomb_page_prefetch merges consecutive blocks), which
    takes no SM from the attention kernels; only the gradient additions run
    as (small) kernels over the host link.

    Ordering (events): a slot's next fetch waits for the slot's last compute
    (both streams of a backward call) and its gradient write-back; the
    fetches of chunk c+1 wait for chunk c's pages to be stored; chunk c+2's
    append waits for chunk c's own pages to be stored and written back.
    """

    def __init__(self, w, device, window, grad_path="host", slots=3):
        """grad_path "gpu": a kernel adds each segment's gradient blocks into the
        pinned host pages over the host link; "host": they are copied
        device -> host (copy engine) and a library worker thread adds them with
        CPU threads (oomb_grad_writeback), leaving the link's host -> device
        direction to the K/V.  slots >= 2: device slots of `window` pages (the
        fetch lead is slots - 1 calls)."""
        if slots < 2:
            raise ValueError("slots must be at least 2")
        self.w, self.dev, self.window, self.slots = w, device, window, slots
        self.grad_path = grad_path
        P, Hkv, d, N = w.page_size, w.num_kv_heads, w.head_dim, w.num_chunks
        C, Hq = w.chunk_len, w.num_q_heads
        self.ppc = w.pages_per_chunk
        self.host = L.pool_create(w.num_pages, P, Hkv, d, L.LOC_PINNED_HOST, True, 0,
                                  device.index or 0)
        # `slots` slots of `window` pages and two sets of the chunk's own pages
        # (used by chunks in turn, so chunk c+1 appends while chunk c's drain)
        n_stage = slots * window + 2 * self.ppc
        self.stage = L.pool_create(n_stage, P, Hkv, d, L.LOC_DEVICE, True, 0, device.index or 0)
        sp = np.array([L.pool_alloc_page(self.stage) for _ in range(n_stage)], dtype=np.int64)
        self.table = np.array([L.pool_alloc_page(self.host) for _ in range(N * self.ppc)],
                              dtype=np.int64)
        i32 = dict(dtype=torch.int32, device=device)
        heads = np.arange(Hkv, dtype=np.int64)

        def blocks(pages):
            return (np.asarray(pages, dtype=np.int64)[:, None] * Hkv + heads[None, :]).reshape(-1)

        slot_pages = [sp[i * window:(i + 1) * window] for i in range(slots)]
        base = slots * window
        curs = [sp[base:base + self.ppc], sp[base + self.ppc:]]
        self.slot_blocks = [torch.tensor(blocks(x), **i32) for x in slot_pages]
        self.slot_blocks_host = [blocks(x) for x in slot_pages]
        # the past list of a slot: its pages, the same for every group
        self.slot_lists = [torch.tensor(np.tile(x, (Hkv, 1)), **i32) for x in slot_pages]
        self.counts = torch.tensor(np.repeat(np.arange(window + 1)[:, None], Hkv, 1), **i32)
        self.cur_dev = [torch.tensor(x, **i32) for x in curs]
        self.cur_blocks = [torch.tensor(blocks(x), **i32) for x in curs]
        self.cur_blocks_host = [blocks(x) for x in curs]
        n_seg = max(1, -(-(N - 1) * self.ppc // window))
        # host blocks of segment s (logical pages [s W, (s + 1) W)), page-major
        self.seg_blocks, self.seg_blocks_host = [], []
        for s in range(n_seg):
            pages = self.table[s * window:(s + 1) * window]
            self.seg_blocks.append(torch.tensor(blocks(pages), **i32))
            self.seg_blocks_host.append(blocks(pages))
        self.own_blocks = torch.tensor(blocks(self.table).reshape(N, -1), **i32)
        self.own_blocks_host = blocks(self.table).reshape(N, -1)
        self.copy = torch.cuda.Stream(device=device, priority=-1)   # fetches (host -> device)
        self.wb = torch.cuda.Stream(device=device, priority=-1)     # stores and gradients back
        self.o_acc = torch.empty((C, Hq, d), dtype=torch.float32, device=device)
        self.dq_acc = torch.empty_like(self.o_acc)
        # dQ of each backward segment runs on its own stream beside that
        # segment's dK/dV; chunk c's dQ may still read its delta (and LSE)
        # while chunk c+1 runs, so these alternate by chunk parity
        self.side = torch.cuda.Stream(device=device)
        self.deltas = [torch.empty((Hq, C), dtype=torch.float32, device=device) for _ in range(2)]
        # forward workspace (split last wave of each segment call; one stream)
        self.fwd_ws = L.fwd_workspace(d, device)
        self.h2d_bytes = self.d2h_bytes = 0

    def close(self):
        self.sync()
        L.pool_destroy(self.stage)
        L.pool_destroy(self.host)

    def _grads_back(self, src_dev, dst_dev, src_host, dst_host, X):
        """Gradient blocks of the staging pool into the host pool (zeroed here)."""
        if self.grad_path == "host":
            L.grad_writeback(self.stage, self.host, src_host, dst_host, stream=X)
        else:
            L.grad_block_add(self.stage, self.host, src_dev, dst_dev, True, stream=X)

    def _segments(self, c):
        """(mode, first page, pages) of chunk c's calls; the last carries the chunk."""
        return plan_segments(c * self.ppc, self.window)

    def run(self, chunks, outputs=None, backward=True):
        w = self.w
        Hkv, N = w.num_kv_heads, w.num_chunks
        comp = torch.cuda.current_stream(self.dev)
        F, B, D = self.copy, self.wb, self.side
        kv_blk, g_blk = 2 * w.page_size * w.head_dim * 2, 2 * w.page_size * w.head_dim * 4
        lead = self.slots - 1
        slot_used = [() for _ in range(self.slots)]  # events a slot's next fetch waits for
        cur_free = [None, None]    # event: a chunk-page set's store and write-back are done
        dq_chunk = [None, None]    # event: the last dQ of the parity's previous chunk is done
        stored = [None] * N        # event: chunk c's own pages are in the host pool
        for st in (F, B, D):
            st.wait_stream(comp)
        scratch = [None, None]

        def calls_of(c):
            segs = self._segments(c)
            return [(c, "fwd") + sg for sg in segs] + \
                ([(c, "bwd") + sg for sg in segs] if backward else [])

        # every call of the run in order: (chunk, kind, segment mode, first page, pages)
        seq = [call for c in range(N) for call in calls_of(c)]
        fetched = {}               # call index -> (slot, event after its fetch)
        nxt = 0                    # the next call to fetch
        use = 0                    # calls take the slots in turn

        def fetch_upto(j_max, cur_chunk):
            """Fetches the calls up to j_max, stopping before any call of a chunk
            beyond cur_chunk + 1 (its past would hold pages not stored yet)."""
            nonlocal nxt, use
            while nxt <= min(j_max, len(seq) - 1):
                c2, _, _, a, n = seq[nxt]
                if c2 > cur_chunk + 1:
                    break
                slot = use % self.slots
                use += 1
                for ev_used in slot_used[slot]:
                    F.wait_event(ev_used)
                if c2 >= 1:
                    F.wait_event(stored[c2 - 1])
                if n:
                    sgi = a // self.window
                    L.page_prefetch(self.host, self.stage, self.seg_blocks_host[sgi][:n * Hkv],
                                    self.slot_blocks_host[slot][:n * Hkv], stream=F)
                    self.h2d_bytes += n * Hkv * kv_blk
                e = torch.cuda.Event()
                e.record(F)
                fetched[nxt] = (slot, e)
                nxt += 1

        i = 0
        for c in range(N):
            x = chunks(c)
            cb = c % 2
            if outputs is not None:
                o, lse, dq = outputs(c)
            else:
                if scratch[cb] is None:
                    scratch[cb] = (torch.empty_like(x["q"]),
                                   torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32,
                                               device=self.dev), torch.empty_like(x["q"]))
                o, lse, dq = scratch[cb]
            delta = self.deltas[cb]
            if dq_chunk[cb] is not None:
                comp.wait_event(dq_chunk[cb])   # chunk c-2's dQ read this delta / scratch
            cur = self.cur_dev[cb]
            if cur_free[cb] is not None:
                comp.wait_event(cur_free[cb])
            L.kv_append(self.stage, cur, x["k"], x["v"], comp)
            ev = torch.cuda.Event()
            ev.record(comp)
            B.wait_event(ev)
            L.page_prefetch(self.stage, self.host, self.cur_blocks_host[cb], self.own_blocks_host[c],
                            stream=B)
            self.d2h_bytes += self.ppc * Hkv * kv_blk
            stored[c] = torch.cuda.Event()
            stored[c].record(B)
            first_bwd = True
            last = ()
            while i < len(seq) and seq[i][0] == c:
                fetch_upto(i + lead, c)
                _, kind, mode, a, n = seq[i]
                slot, e = fetched.pop(i)
                comp.wait_event(e)
                past, cnt = (self.slot_lists[slot], self.counts[n]) if n else (None, None)
                if kind == "fwd":
                    L.chunk_attn_fwd(self.stage, x["q"], o, lse, past, cnt, cur,
                                     w.softmax_scale, comp, segment=mode, o_acc=self.o_acc,
                                     fwd_ws=self.fwd_ws)
                    done = torch.cuda.Event()
                    done.record(comp)
                    slot_used[slot] = (done,)
                else:
                    if first_bwd:
                        L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta,
                                         None, None, cur, w.softmax_scale, comp,
                                         step=L.BWD_PREPROCESS)
                        first_bwd = False
                    # dQ beside dK/dV: D after the slot's fetch and the preprocess
                    D.wait_stream(comp)
                    L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta,
                                     past, cnt, cur, w.softmax_scale, D,
                                     step=L.BWD_DQ, segment=mode, o_acc=self.o_acc,
                                     dq_acc=self.dq_acc)
                    L.chunk_attn_bwd(self.stage, x["q"], o, lse, x["do"], dq, delta,
                                     past, cnt, cur, w.softmax_scale, comp,
                                     step=L.BWD_DKDV, segment=mode, o_acc=self.o_acc,
                                     dq_acc=self.dq_acc)
                    done = torch.cuda.Event()
                    done.record(comp)
                    done_dq = torch.cuda.Event()
                    done_dq.record(D)
                    last = (done, done_dq)
                    slot_used[slot] = last
                    if n:
                        # the segment's gradients into the host pool, zeroed here
                        B.wait_event(done)
                        sgi = a // self.window
                        self._grads_back(self.slot_blocks[slot][:n * Hkv],
                                         self.seg_blocks[sgi][:n * Hkv],
                                         self.slot_blocks_host[slot][:n * Hkv],
                                         self.seg_blocks_host[sgi][:n * Hkv], B)
                        gb = torch.cuda.Event()
                        gb.record(B)
                        slot_used[slot] = last + (gb,)
                        if self.grad_path == "gpu":
                            self.h2d_bytes += n * Hkv * g_blk
                        self.d2h_bytes += n * Hkv * g_blk
                i += 1
            if backward:
                # the chunk's own gradients (final after its last dK/dV)
                B.wait_event(last[0])
                self._grads_back(self.cur_blocks[cb], self.own_blocks[c], self.cur_blocks_host[cb],
                                 self.own_blocks_host[c], B)
                if self.grad_path == "gpu":
                    self.h2d_bytes += self.ppc * Hkv * g_blk
                self.d2h_bytes += self.ppc * Hkv * g_blk
                dq_chunk[cb] = last[1]   # its dQ read the chunk's pages, delta and LSE
            cur_free[cb] = torch.cuda.Event()
            cur_free[cb].record(B)
        comp.wait_stream(F)
        comp.wait_stream(B)
        comp.wait_stream(D)

    def sync(self):
        """Waits for the device and, on the host path, every queued addition."""
        torch.cuda.synchronize(self.dev)
        if self.grad_path == "host":
            L.grad_writeback_sync(self.stage)
