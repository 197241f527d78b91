"""Throughput of paged chunk attention (fwd+bwd) on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over a 256K-token context of the
Qwen2.5-7B attention shape (Hq=28, Hkv=4, d=128, 64-token pages, 64 chunks of
4096, shuffled page table): for every chunk, append K/V into its pages, the
forward, and the backward (preprocess, dK/dV added in place into the gradient
pool, dQ).  The headline value is the dense run's algorithmic TFLOP/s; the
same line carries the Top-K sparse run (Top-64 + 2 recent pages per chunk and
KV-head group, Top-K selection included in the timed step), tokens/s for
both, an end-to-end figure with host buffers, the roofline of the dominant
kernel, the 1M-token offloaded Top-K run (KV and gradients in pinned host
memory), the memory-bound kernels in batched launches (append, Top-K, block
gather and gradient scatter-add, over HBM and over the host link) and the CPU
oracle's throughput on a bounded sample.

Inputs are synthetic (seeded), drawn on the device before timing; the
working set (Q, dO, KV pool, gradient pool) is far larger than L2.  Under
torchrun each rank runs the same workload on its own GPU (independent
replicas, weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk-attn fwd+bwd TFLOP/s and context tokens/s at 256K (dense; Top-K sparse)"


# ------------------------------------------------------------------ helpers
def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs", 6650.0), "bf16": d.get("bf16_tflops", 1590.0),
                "bf16_sustained": d.get("bf16_tflops_sustained", 1400.0),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def clock_scaled_peak(burst, sm_mhz, sm_max_mhz):
    """The burst tensor peak scaled to the SM clock a run actually held: the
    tensor pipe's rate is proportional to the SM clock, so this is what the
    same GEMM would reach at that clock (None without a clock record)."""
    if not burst or not sm_mhz or not sm_max_mhz:
        return None
    return burst * sm_mhz / sm_max_mhz


def step_fractions(tflops, peaks, sm_mhz):
    """A step's TFLOP/s as fractions of the sustained, burst and clock-scaled
    burst bf16 peaks."""
    cp = clock_scaled_peak(peaks["bf16"], sm_mhz, peaks.get("sm_max_mhz"))
    return {"of_sustained": tflops / peaks["bf16_sustained"], "of_burst": tflops / peaks["bf16"],
            "of_clock_normalised": tflops / cp if cp else None}


def pairs_of_chunk(C, n_past_keys):
    """(query row, key) pairs of one head of one chunk: every past key plus the
    causal part of the chunk itself."""
    return C * n_past_keys + C * (C + 1) // 2


def chunk_past_keys(w, c, sparse):
    """Past keys each row of chunk c attends to: every earlier token (dense),
    the kept pages (Top-K: min(K, n_past - R) + min(R, n_past) pages, per
    chunk or per query tile alike), or the last `window` pages (recent-only)."""
    ppc, P = w.pages_per_chunk, w.page_size
    if sparse and c:
        return (min(w.top_k, max(0, c * ppc - w.n_recent)) + min(w.n_recent, c * ppc)) * P
    if w.window > 0:
        return min(w.window, c * ppc) * P
    return c * w.chunk_len


def step_pairs(w, sparse):
    """(query row, key) pairs of one step over all chunks and query heads."""
    return sum(pairs_of_chunk(w.chunk_len, chunk_past_keys(w, c, sparse)) * w.num_q_heads
               for c in range(w.num_chunks))


class Clocks:
    """Samples nvidia-smi every 200 ms while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        return self.summary()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in self.rows if num(r[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        loaded = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(self.rows)}


# ------------------------------------------------------------------ our path
class Run:
    """All device state of one workload: pool, page tables, inputs, outputs."""

    def __init__(self, w, sparse, device, inputs=None):
        """inputs: per chunk a dict of device tensors q, k, v, dO (default: the
        workload's shapes and distributions drawn on the device)."""
        import paged_kv_chunk_query_b200 as pk
        from paged_kv_chunk_query_b200 import synth
        self.pk, self.w, self.sparse, self.dev = pk, w, sparse, device
        N, C, P, Hq, Hkv, d = (w.num_chunks, w.chunk_len, w.page_size, w.num_q_heads,
                               w.num_kv_heads, w.head_dim)
        self.pool = pk.pool_create(w.num_pages, P, Hkv, d, pk.LOC_DEVICE, True, w.alloc_seed,
                                   device.index or 0)
        ppc = w.pages_per_chunk
        self.page_table = [pk.pool_alloc_page(self.pool) for _ in range(N * ppc)]
        pt = torch.tensor(self.page_table, dtype=torch.int32, device=device)
        self.page_table_dev = pt
        self.cur = [pt[c * ppc:(c + 1) * ppc].contiguous() for c in range(N)]
        self.inputs = inputs if inputs is not None else \
            [synth.device_chunk_inputs(w, c, device) for c in range(N)]
        self.o = [torch.empty((C, Hq, d), dtype=torch.bfloat16, device=device) for _ in range(N)]
        self.dq = [torch.empty_like(x) for x in self.o]
        self.lse = [torch.empty((Hq, C), dtype=torch.float32, device=device) for _ in range(N)]
        # one delta workspace per chunk: chunk c's dQ launch may still read its
        # delta while chunk c+1's preprocess runs
        self.deltas = [torch.empty((Hq, C), dtype=torch.float32, device=device) for _ in range(N)]
        # forward workspace (partial O/LSE of a split last wave); every forward
        # of a step runs on one stream, so one workspace serves them all
        self.fwd_ws = pk.fwd_workspace(d, device)
        self.side = torch.cuda.Stream(device=device)
        # selections of the next chunk run here, beside the current chunk's attention
        self.sel_stream = torch.cuda.Stream(device=device)
        self.early_select = True
        self.fwd_stream = torch.cuda.Stream(device=device)
        self.concurrent_bwd = True
        self.fwd_overlap = False
        self.dense_past = [None] + [pt[:c * ppc].repeat(Hkv, 1).contiguous() for c in range(1, N)]
        self.dense_cnt = [None] + [torch.full((Hkv,), c * ppc, dtype=torch.int32, device=device)
                                   for c in range(1, N)]
        self.local = w.window > 0
        if self.local:
            self.loc_p = [torch.zeros((Hkv, w.window), dtype=torch.int32, device=device)
                          for _ in range(N)]
            self.loc_n = [torch.zeros((Hkv,), dtype=torch.int32, device=device) for _ in range(N)]
        self.qtile = sparse and w.qtile_topk
        self.qpage = sparse and w.qpage_topk
        self.masks = [None] * N
        if sparse:
            ms = w.top_k + w.n_recent
            nq = (C + 127) // 128
            # selection problems per chunk: query tiles, query pages, or the chunk
            nprob = nq if self.qtile else (C // P if self.qpage else None)
            rows = 128 if self.qtile else P
            lead = (nprob, Hkv) if nprob else (Hkv,)
            self.sel_l = [torch.zeros(lead + (ms,), dtype=torch.int32, device=device)
                          for _ in range(N)]
            self.sel_p = [torch.zeros(lead + (ms,), dtype=torch.int32, device=device)
                          for _ in range(N)]
            self.sel_n = [torch.zeros(lead, dtype=torch.int32, device=device) for _ in range(N)]
            if nprob:
                ws = pk.page_topk_batched_workspace_size(nprob, Hkv, d, (N - 1) * ppc)
                self.sel_rows = rows
                self.row_start = torch.arange(0, (nprob + 1) * rows, rows, dtype=torch.int32,
                                              device=device).clamp_(max=C)
                self.npast = [torch.full((nprob,), c * ppc, dtype=torch.int32, device=device)
                              for c in range(N)]
            else:
                ws = pk.page_topk_workspace_size(C, Hq, Hkv, d, (N - 1) * ppc)
            self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
            if self.qpage:
                # per query tile: the union of its query pages' lists + membership masks
                mu = min(128 // P, C // P) * ms
                self.u_pages = [torch.zeros((nq, Hkv, mu), dtype=torch.int32, device=device)
                                for _ in range(N)]
                self.masks = [torch.zeros((nq, Hkv, mu), dtype=torch.uint8, device=device)
                              for _ in range(N)]
                self.u_cnt = [torch.zeros((nq, Hkv), dtype=torch.int32, device=device)
                              for _ in range(N)]
        # algorithmic FLOPs per chunk (per kernel class) and per step
        self.flops = {"fwd": [], "dkdv": [], "dq": []}
        for c in range(N):
            pairs = pairs_of_chunk(C, chunk_past_keys(w, c, sparse)) * Hq
            self.flops["fwd"].append(4.0 * pairs * d)
            self.flops["dkdv"].append(8.0 * pairs * d)
            self.flops["dq"].append(2.0 * pairs * d)
        self.step_flops = sum(sum(v) for v in self.flops.values())
        # per chunk: append, forward (+ merge), preprocess, dK/dV, dQ; Top-K adds its two
        # launches (query mean; scores with the select) per chunk with a past
        # (per-query-tile lists: and a second dK/dV launch; per-query-page
        # lists: that and the union-list launch); local lists one
        # the forward's merge launch when its last wave of (query tile, head)
        # units is split over the free SMs (the launcher's rule)
        ns = torch.cuda.get_device_properties(device).multi_processor_count
        tail = ((C + 127) // 128 * Hq) % ns
        self.fwd_merge = tail > 0 and min(ns // tail, 256 // tail) >= 2
        self.launches_per_step = N * (5 + int(self.fwd_merge)) + ((N - 1) * 2 if sparse else 0) + \
            ((N - 1) if self.local else 0) + ((N - 1) if self.qtile else 0) + \
            ((N - 1) * 2 if self.qpage else 0)

    def select(self, c, st, timed):
        """Chunk c's past lists on stream st: (pages, counts, masks)."""
        pk, w = self.pk, self.w
        ppc = w.pages_per_chunk
        x = self.inputs[c]
        if c == 0:
            return None, None, None
        n_past = c * ppc
        if self.local:
            timed("lists", lambda: pk.local_pages(self.pool, self.page_table_dev[:n_past], n_past,
                                                  self.loc_p[c], self.loc_n[c], stream=st), st)
            return self.loc_p[c], self.loc_n[c], None
        if self.qtile or self.qpage:
            timed("topk", lambda: pk.page_topk_batched(
                self.pool, x["q"], self.row_start, self.sel_rows, self.npast[c], n_past,
                self.page_table_dev[:n_past], w.top_k, w.n_recent, self.sel_l[c], self.sel_p[c],
                self.sel_n[c], self.ws, stream=st), st)
            if self.qtile:
                return self.sel_p[c], self.sel_n[c], None
            timed("lists", lambda: pk.qpage_lists(
                self.pool, self.sel_l[c], self.sel_p[c], self.sel_n[c], w.chunk_len,
                self.u_pages[c], self.masks[c], self.u_cnt[c], stream=st), st)
            return self.u_pages[c], self.u_cnt[c], self.masks[c]
        if self.sparse:
            timed("topk", lambda: pk.page_topk(
                self.pool, x["q"], self.page_table_dev[:n_past], n_past, w.top_k, w.n_recent,
                self.sel_l[c], self.sel_p[c], self.sel_n[c], self.ws, stream=st), st)
            return self.sel_p[c], self.sel_n[c], None
        return self.dense_past[c], self.dense_cnt[c], None

    def step(self, timers=None):
        if self.fwd_overlap and self.concurrent_bwd:
            return self._step3(timers)
        return self._step2(timers)

    def _step3(self, timers=None):
        """One pass over all chunks on three streams: the forward stream runs
        chunk c's selection, forward and preprocess; then chunk c's dQ (side
        stream) and dK/dV (main stream) run while the forward stream already
        takes chunk c+1 (its forward reads only K/V, which no backward writes).
        Appends stay on the main stream."""
        pk, w = self.pk, self.w
        M = torch.cuda.current_stream()
        S, F = self.side, self.fwd_stream

        def timed(name, fn, st):
            if timers is None:
                fn()
                return
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            timers.setdefault(name, []).append((a, b))

        S.wait_stream(M)
        F.wait_stream(M)
        timed("append", lambda: pk.kv_append(self.pool, self.cur[0], self.inputs[0]["k"],
                                             self.inputs[0]["v"], M), M)
        appended = torch.cuda.Event()
        appended.record(M)
        for c in range(w.num_chunks):
            x = self.inputs[c]
            F.wait_event(appended)    # chunk c's pages (and earlier summaries) appended
            past, cnt, msk = self.select(c, F, timed)
            o, lse, dq = self.o[c], self.lse[c], self.dq[c]
            sc = w.softmax_scale
            delta = self.deltas[c]
            timed("fwd", lambda: pk.chunk_attn_fwd(self.pool, x["q"], o, lse, past, cnt,
                                                   self.cur[c], sc, F, past_masks=msk,
                                                   fwd_ws=self.fwd_ws), F)
            timed("preprocess", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], sc, F,
                step=pk.BWD_PREPROCESS, past_masks=msk), F)
            if c + 1 < w.num_chunks:
                xn = self.inputs[c + 1]
                timed("append", lambda: pk.kv_append(self.pool, self.cur[c + 1], xn["k"], xn["v"],
                                                     M), M)
                appended = torch.cuda.Event()
                appended.record(M)
            S.wait_stream(F)
            M.wait_stream(F)
            timed("dq", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], sc, S,
                step=pk.BWD_DQ, past_masks=msk), S)
            timed("dkdv", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], sc, M,
                step=pk.BWD_DKDV, past_masks=msk), M)
        M.wait_stream(S)
        M.wait_stream(F)

    def _step2(self, timers=None):
        """One pass over all chunks.  With concurrent_bwd, chunk c's dQ launch
        runs on a second stream next to its dK/dV launch (the two only read
        what the forward and preprocess wrote and write disjoint outputs), so
        each fills the other's last partial wave of CTAs.  With early_select,
        chunk c+1's past lists (Top-K or recent pages) are made on a third
        stream as soon as chunk c's pages are appended: they read only chunk
        c+1's queries and the page means of chunks 0..c, which the backward
        does not change, so they run beside chunk c's attention instead of
        between chunk c's dK/dV and chunk c+1's forward.  All selections share
        one workspace and so stay in order on that stream."""
        pk, w = self.pk, self.w
        stream = torch.cuda.current_stream()
        side = self.side if self.concurrent_bwd else stream

        def timed(name, fn, st=None):
            st = st or stream
            if timers is None:
                fn()
                return
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            timers.setdefault(name, []).append((a, b))

        if side is not stream:
            side.wait_stream(stream)
        early = self.early_select and (self.sparse or self.local)
        sel = self.sel_stream
        if early:
            sel.wait_stream(stream)
        lists = {}

        def select_next(c):
            # chunk c's lists on the selection stream, once chunks 0..c-1 are appended
            appended = torch.cuda.Event()
            appended.record(stream)
            sel.wait_event(appended)
            lists[c] = self.select(c, sel, timed)
            done = torch.cuda.Event()
            done.record(sel)
            lists[c] = lists[c] + (done,)

        for c in range(w.num_chunks):
            x = self.inputs[c]
            if c == 0:
                timed("append", lambda: pk.kv_append(self.pool, self.cur[0], x["k"], x["v"],
                                                     stream))
            if early:
                if c + 1 < w.num_chunks:
                    select_next(c + 1)
                if c == 0:
                    past, cnt, msk = None, None, None
                else:
                    past, cnt, msk, done = lists.pop(c)
                    stream.wait_event(done)
            else:
                past, cnt, msk = self.select(c, stream, timed)
            o, lse, dq = self.o[c], self.lse[c], self.dq[c]
            s = w.softmax_scale
            delta = self.deltas[c]
            timed("fwd", lambda: pk.chunk_attn_fwd(self.pool, x["q"], o, lse, past, cnt,
                                                   self.cur[c], s, stream, past_masks=msk,
                                                   fwd_ws=self.fwd_ws))
            timed("preprocess", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], s, stream,
                step=pk.BWD_PREPROCESS, past_masks=msk))
            if c + 1 < w.num_chunks:
                # chunk c+1's pages: nothing of chunk c reads or writes them
                xn = self.inputs[c + 1]
                timed("append", lambda: pk.kv_append(self.pool, self.cur[c + 1], xn["k"], xn["v"],
                                                     stream))
            if side is not stream:
                side.wait_stream(stream)
            timed("dq", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], s, side,
                step=pk.BWD_DQ, past_masks=msk), side)
            timed("dkdv", lambda: pk.chunk_attn_bwd(
                self.pool, x["q"], o, lse, x["do"], dq, delta, past, cnt, self.cur[c], s, stream,
                step=pk.BWD_DKDV, past_masks=msk))
        if side is not stream:
            stream.wait_stream(side)
        if early:
            stream.wait_stream(sel)

    def time_topk_alone(self, reps=3):
        """Every chunk's Top-K selection back to back (no attention launches in
        between): ms for one pass over chunks 1..N-1, (two-launch form from Q,
        one-launch form from per-group Q sums).  Each pass is captured once in
        a CUDA graph and replayed (a loop of microsecond launches is bound by
        host launch cost otherwise).  The chunks' queries (1.8 GiB together)
        rotate, so L2 does not hold them.  The Q sums are made beforehand, as
        the projection's epilogue makes them in a full layer."""
        pk, w = self.pk, self.w
        ppc = w.pages_per_chunk
        C, Hq, Hkv, d = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.head_dim
        qsums = [x["q"].float().reshape(C, Hkv, Hq // Hkv, d).sum(dim=(0, 2)).contiguous()
                 for x in self.inputs]
        ws_q = torch.zeros(pk.page_topk_qsum_workspace_size(Hkv, (w.num_chunks - 1) * ppc),
                           dtype=torch.uint8, device=self.dev)

        def from_q(st):
            for c in range(1, w.num_chunks):
                n_past = c * ppc
                pk.page_topk(self.pool, self.inputs[c]["q"], self.page_table_dev[:n_past], n_past,
                             w.top_k, w.n_recent, self.sel_l[c], self.sel_p[c], self.sel_n[c],
                             self.ws, stream=st)

        def from_qsum(st):
            for c in range(1, w.num_chunks):
                n_past = c * ppc
                pk.page_topk_qsum(self.pool, qsums[c], C, Hq, self.page_table_dev[:n_past],
                                  n_past, w.top_k, w.n_recent, self.sel_l[c], self.sel_p[c],
                                  self.sel_n[c], ws_q, stream=st)

        def graph_ms(one_pass):
            s = torch.cuda.Stream(device=self.dev)
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                one_pass(s)
            torch.cuda.current_stream().wait_stream(s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one_pass(torch.cuda.current_stream())
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                g.replay()
            b.record()
            torch.cuda.synchronize()
            del g
            return a.elapsed_time(b) / reps

        return graph_ms(from_q), graph_ms(from_qsum)

    def close(self):
        self.pk.pool_destroy(self.pool)


def _barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()


def whole_job_rate(units_per_rank, ms_max, world):
    """Whole-job throughput of `world` replicas: every rank processes
    `units_per_rank`, the job takes the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def _max_over_ranks(x, dist_on, device):
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_steps(run, steps, warmup, dist_on, device, kernel_timers=True):
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize()
    _barrier(dist_on)
    torch.cuda.synchronize()
    timers = {} if kernel_timers else None
    stream = torch.cuda.current_stream()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        run.step(timers)
    b.record(stream)
    torch.cuda.synchronize()
    _barrier(dist_on)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    per_kernel = {}
    if timers:
        for name, ev in timers.items():
            per_kernel[name] = sum(x.elapsed_time(y) for x, y in ev) / steps  # ms per step
    return _max_over_ranks(ms, dist_on, device), per_kernel


def e2e_dense(w, steps, device):
    """Same dense workload through the public API with host buffers: every
    chunk's Q, K, V, dO are copied from pinned host memory and O, LSE, dQ plus
    the final gradient pool are read back, inside the timed region.  Copies run
    on a copy stream, overlapped with the previous chunk's compute; each
    chunk's dQ runs beside its dK/dV on a second stream (the backward's
    step calls), as in the device-timed step."""
    import paged_kv_chunk_query_b200 as pk
    from paged_kv_chunk_query_b200 import synth
    N, C, Hq, Hkv, d, P = (w.num_chunks, w.chunk_len, w.num_q_heads, w.num_kv_heads,
                           w.head_dim, w.page_size)
    ppc = w.pages_per_chunk
    pool = pk.pool_create(w.num_pages, P, Hkv, d, pk.LOC_DEVICE, True, w.alloc_seed,
                          device.index or 0)
    try:
        table = [pk.pool_alloc_page(pool) for _ in range(N * ppc)]
        pt = torch.tensor(table, dtype=torch.int32, device=device)
        host_in = []
        for c in range(N):
            x = synth.device_chunk_inputs(w, c, device)
            host_in.append({k: v.cpu().pin_memory() for k, v in x.items()})
        host_o = [torch.empty((C, Hq, d), dtype=torch.bfloat16).pin_memory() for _ in range(N)]
        host_dq = [torch.empty_like(t) for t in host_o]
        host_dq = [t.pin_memory() for t in host_dq]
        host_lse = [torch.empty((Hq, C), dtype=torch.float32).pin_memory() for _ in range(N)]
        _, grad, _ = pk.pool_views(pool)
        host_grad = torch.empty(grad.shape, dtype=torch.float32).pin_memory()
        dev_in = [{k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in host_in[0].items()}
                  for _ in range(2)]
        dev_out = [(torch.empty((C, Hq, d), dtype=torch.bfloat16, device=device),
                    torch.empty((Hq, C), dtype=torch.float32, device=device),
                    torch.empty((C, Hq, d), dtype=torch.bfloat16, device=device)) for _ in range(2)]
        # one delta per buffer parity: chunk c's dQ (side stream) may still read its
        # delta while chunk c+1's preprocess runs
        deltas = [torch.empty((Hq, C), dtype=torch.float32, device=device) for _ in range(2)]
        fwd_ws = pk.fwd_workspace(d, device)
        past = [None] + [pt[:c * ppc].repeat(Hkv, 1).contiguous() for c in range(1, N)]
        cnt = [None] + [torch.full((Hkv,), c * ppc, dtype=torch.int32, device=device)
                        for c in range(1, N)]
        comp = torch.cuda.current_stream()
        copy = torch.cuda.Stream(device=device)
        side = torch.cuda.Stream(device=device)   # each chunk's dQ beside its dK/dV
        h2d = sum(t.numel() * t.element_size() for t in host_in[0].values()) * N
        d2h = (sum(t.numel() * t.element_size() for t in (host_o[0], host_lse[0], host_dq[0])) * N
               + host_grad.numel() * 4)

        def one_step():
            in_ready = [torch.cuda.Event() for _ in range(N)]
            out_ready = [torch.cuda.Event() for _ in range(N)]
            dq_done = [torch.cuda.Event() for _ in range(N)]
            out_free = [torch.cuda.Event() for _ in range(N)]
            with torch.cuda.stream(copy):
                for k, v in host_in[0].items():
                    dev_in[0][k].copy_(v, non_blocking=True)
                in_ready[0].record(copy)
            for c in range(N):
                buf = c % 2
                if c + 1 < N:
                    with torch.cuda.stream(copy):
                        if c >= 1:  # inputs buffer (c+1)%2 was chunk c-1's
                            copy.wait_event(out_ready[c - 1])
                            copy.wait_event(dq_done[c - 1])
                        for k, v in host_in[c + 1].items():
                            dev_in[(c + 1) % 2][k].copy_(v, non_blocking=True)
                        in_ready[c + 1].record(copy)
                comp.wait_event(in_ready[c])
                if c >= 2:
                    comp.wait_event(out_free[c - 2])
                x = dev_in[buf]
                o, lse, dq = dev_out[buf]
                cur = pt[c * ppc:(c + 1) * ppc]
                pk.kv_append(pool, cur, x["k"], x["v"], comp)
                pk.chunk_attn_fwd(pool, x["q"], o, lse, past[c], cnt[c], cur, w.softmax_scale, comp,
                                  fwd_ws=fwd_ws)
                delta = deltas[buf]
                bwd = (pool, x["q"], o, lse, x["do"], dq, delta, past[c], cnt[c], cur,
                       w.softmax_scale)
                pk.chunk_attn_bwd(*bwd, comp, step=pk.BWD_PREPROCESS)
                side.wait_stream(comp)
                pk.chunk_attn_bwd(*bwd, side, step=pk.BWD_DQ)
                dq_done[c].record(side)
                pk.chunk_attn_bwd(*bwd, comp, step=pk.BWD_DKDV)
                out_ready[c].record(comp)
                with torch.cuda.stream(copy):
                    copy.wait_event(out_ready[c])
                    copy.wait_event(dq_done[c])
                    host_o[c].copy_(o, non_blocking=True)
                    host_lse[c].copy_(lse, non_blocking=True)
                    host_dq[c].copy_(dq, non_blocking=True)
                    out_free[c].record(copy)
            comp.wait_stream(copy)
            host_grad.copy_(grad, non_blocking=True)

        one_step()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(comp)
        for _ in range(steps):
            one_step()
        b.record(comp)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps, h2d, d2h
    finally:
        pk.pool_destroy(pool)


def offload_run(w, steps, device, dist_on):
    """1M-token Top-K run with every page's KV and gradients in pinned host
    memory (selected pages prefetched into an HBM staging pool on a copy
    stream, gradient deltas written back asynchronously).  One step = all
    chunks, timed with CUDA events on the compute stream, max over ranks."""
    from paged_kv_chunk_query_b200 import synth
    from paged_kv_chunk_query_b200.offload import OffloadRun
    ins = [synth.device_chunk_inputs(w, c, device) for c in range(w.num_chunks)]
    run = OffloadRun(w, device)
    try:
        run.run(lambda c: ins[c])  # warm-up pass (also fills the host pools)
        run.sync()
        _barrier(dist_on)
        comp = torch.cuda.current_stream()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        a.record(comp)
        for _ in range(steps):
            run.run(lambda c: ins[c])
        b.record(comp)
        run.sync()  # every gradient addition is stream-ordered on the device
        wall = (time.perf_counter() - t0) * 1e3 / steps
        ev_ms = a.elapsed_time(b) / steps
        ms = _max_over_ranks(ev_ms, dist_on, device)
        import paged_kv_chunk_query_b200 as pk
        status = pk.get_device_status(run.stage) | pk.get_device_status(run.host)
        h2d, d2h = run.link_bytes()
    finally:
        run.close()
        del ins
        torch.cuda.empty_cache()
    return {"workload": w.name, "context": w.context, "ms_per_step": ms,
            "ms_per_step_wall": wall,
            "ms_per_chunk": ms / w.num_chunks, "tokens_per_s": w.context / (ms / 1e3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "h2d_gbs": h2d / (ms / 1e3) / 1e9, "d2h_gbs": d2h / (ms / 1e3) / 1e9,
            "link_bytes_note": "host link: prefetched KV + host gradients read for the "
                               "additions (h2d); stored KV + gradients written back (d2h)",
            "device_status": status}


def dense_offload_run(w, window, device, dist_on, grad_path="host"):
    """Dense 256K with KV and gradients in pinned host memory and a window of
    `window` past pages per slot (three slots) on the device; one step = all chunks,
    timed with CUDA events on the compute stream (1 warm-up step)."""
    from paged_kv_chunk_query_b200 import synth
    from paged_kv_chunk_query_b200.offload import DenseOffloadRun
    ins = [synth.device_chunk_inputs(w, c, device) for c in range(w.num_chunks)]
    run = DenseOffloadRun(w, device, window, grad_path)
    try:
        run.run(lambda c: ins[c])
        run.sync()
        run.h2d_bytes = run.d2h_bytes = 0
        _barrier(dist_on)
        comp = torch.cuda.current_stream()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(comp)
        run.run(lambda c: ins[c])
        b.record(comp)
        run.sync()
        ms = _max_over_ranks(a.elapsed_time(b), dist_on, device)
        import paged_kv_chunk_query_b200 as pk
        status = pk.get_device_status(run.stage) | pk.get_device_status(run.host)
        P, Hkv, d = w.page_size, w.num_kv_heads, w.head_dim
        dev_bytes = (run.slots * window + 2 * w.pages_per_chunk) * Hkv * 2 * P * d * (2 + 4)
        full_bytes = w.num_pages * Hkv * 2 * P * d * (2 + 4)
        h2d, d2h = run.h2d_bytes, run.d2h_bytes
    finally:
        run.close()
        del ins
        torch.cuda.empty_cache()
    return {"workload": w.name, "window_pages": window, "slots": run.slots,
            "grad_path": grad_path,
            "ms_per_step": ms,
            "tokens_per_s": w.context / (ms / 1e3),
            "device_window_bytes": dev_bytes, "full_pool_bytes": full_bytes,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "h2d_gbs": h2d / (ms / 1e3) / 1e9, "d2h_gbs": d2h / (ms / 1e3) / 1e9,
            "device_status": status}


def projection_run(w, device, peaks, hidden=3584):
    """The Q/K/V projection of one chunk at the attention's shape (hidden 3584
    as in Qwen2.5-7B; random weights) through oomb_qkv_project: the GEMM's
    throughput, and a chunk's Top-K prefetch (66 pages x Hkv blocks from
    pinned host memory) run on a copy stream beside the K/V part."""
    import paged_kv_chunk_query_b200 as pk
    C, Hq, Hkv, d, P = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size
    n_out = (Hq + 2 * Hkv) * d
    gen = torch.Generator(device=device).manual_seed(w.seed)
    x = torch.randn((C, hidden), generator=gen, device=device).to(torch.bfloat16)
    wt = (torch.randn((n_out, hidden), generator=gen, device=device) / hidden ** 0.5).to(
        torch.bfloat16)
    ppc = C // P
    dev_i = device.index or 0
    pool = pk.pool_create(ppc + 128, P, Hkv, d, pk.LOC_DEVICE, True, 0, dev_i)
    host = pk.pool_create(4096, P, Hkv, d, pk.LOC_PINNED_HOST, True, 0, dev_i)
    try:
        pages = torch.tensor([pk.pool_alloc_page(pool) for _ in range(ppc)], dtype=torch.int32,
                             device=device)
        slots = [pk.pool_alloc_page(pool) for _ in range(66)]
        q = torch.empty((C, Hq, d), dtype=torch.bfloat16, device=device)
        qsum = torch.empty((Hkv, d), dtype=torch.float32, device=device)
        flops = 2.0 * C * hidden * n_out
        ms_qkv = _event_ms(lambda: pk.qkv_project(pool, x, wt, Hq, pk.PROJ_QKV, q=q, qsum=qsum,
                                                  page_ids=pages), reps=20, warmup=3)
        ms_q = _event_ms(lambda: pk.qkv_project(pool, x, wt, Hq, pk.PROJ_Q, q=q, qsum=qsum),
                         reps=20, warmup=3)
        ms_kv = _event_ms(lambda: pk.qkv_project(pool, x, wt, Hq, pk.PROJ_KV, page_ids=pages),
                          reps=20, warmup=3)
        # a chunk's selection: 66 random pages of the host pool, every group
        rng = torch.Generator().manual_seed(5)
        sel = torch.randperm(4096, generator=rng)[:66]
        src = (sel[:, None] * Hkv + torch.arange(Hkv)[None, :]).reshape(-1).to(torch.int32)
        dst = (torch.tensor(slots)[:, None] * Hkv + torch.arange(Hkv)[None, :]).reshape(-1)
        src, dst = src.to(device), dst.to(torch.int32).to(device)
        side = torch.cuda.Stream(device=device, priority=-1)
        ms_pf = _event_ms(lambda: pk.block_copy(host, pool, src, dst), reps=20, warmup=3)
        comp = torch.cuda.current_stream()

        def both():
            side.wait_stream(comp)
            pk.block_copy(host, pool, src, dst, stream=side)
            pk.qkv_project(pool, x, wt, Hq, pk.PROJ_KV, page_ids=pages, stream=comp)
            comp.wait_stream(side)
        ms_both = _event_ms(both, reps=20, warmup=3)
        status = pk.get_device_status(pool) | pk.get_device_status(host)
    finally:
        pk.pool_destroy(pool)
        pk.pool_destroy(host)
        torch.cuda.empty_cache()
    tf = flops / (ms_qkv / 1e3) / 1e12
    return {"shape": f"X [{C}][{hidden}] x W^T [{n_out}][{hidden}] bf16 (random weights)",
            "qkv": {"ms": ms_qkv, "tflops": tf, "frac_of_sustained": tf / peaks["bf16_sustained"],
                    "frac_of_burst": tf / peaks["bf16"]},
            "q_part_ms": ms_q, "kv_part_ms": ms_kv,
            "prefetch_one_selection_ms": ms_pf, "kv_part_with_prefetch_beside_ms": ms_both,
            # share of the shorter of the two that ran under the other
            "overlap_fraction": max(0.0, min(1.0, (ms_kv + ms_pf - ms_both) / min(ms_kv, ms_pf))),
            "note": "inputs resident in L2 (compute-bound GEMM, 2.2 kFLOP/B)",
            "device_status": status}


# ------------------------------------------------------------------ HBM / host-link kernels
def _event_ms(fn, reps=5, warmup=2):
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def hbm_kernels(w, device, peaks):
    """The memory-bound kernels measured in batched launches (per-chunk
    launches are microseconds long): the append of a whole 256K context in
    one launch, every chunk's Top-K in one batched launch, a gather and a
    gradient scatter-add of every (page, head) block of a shuffled 4096-page
    pool, and the same moves over the host link against a measured pinned
    memcpy peak.  Inputs are larger than L2 (512 MiB pools, 1.75 GiB of Q)."""
    import paged_kv_chunk_query_b200 as pk
    P, Hkv, d, Hq, C, N = (w.page_size, w.num_kv_heads, w.head_dim, w.num_q_heads, w.chunk_len,
                           w.num_chunks)
    T, npg = w.context, w.num_pages
    dev_i = device.index or 0
    hbm = peaks["hbm_gbs"]
    out = {}

    def entry(nbytes, ms, peak, what):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"ms": ms, "bytes": nbytes, "gbs": gbs, "frac": gbs / peak, "what": what}

    a = pk.pool_create(npg, P, Hkv, d, pk.LOC_DEVICE, True, w.alloc_seed or 1, dev_i)
    b = pk.pool_create(npg, P, Hkv, d, pk.LOC_DEVICE, True, 0, dev_i)
    h = None
    try:
        table = torch.tensor([pk.pool_alloc_page(a) for _ in range(npg)], dtype=torch.int32,
                             device=device)
        gen = torch.Generator(device=device).manual_seed(w.seed)
        k = torch.randn((T, Hkv, d), generator=gen, device=device).to(torch.bfloat16)
        v = torch.randn((T, Hkv, d), generator=gen, device=device).to(torch.bfloat16)
        ms = _event_ms(lambda: pk.kv_append(a, table, k, v))
        nb = 2 * T * Hkv * d * 2 * 2 + 2 * T * Hkv * d * 4 + npg * Hkv * d * 4
        out["kv_append_whole_context"] = entry(
            nb, ms, hbm, f"{T} tokens into {npg} shuffled pages in one launch: K,V read + "
            "written, fp32 page means written, fp32 gradient blocks zeroed")
        del k, v
        # every chunk's Top-K in one batched launch
        q_all = torch.randn((N * C, Hq, d), generator=gen, device=device).to(torch.bfloat16)
        n_past = torch.tensor([c * w.pages_per_chunk for c in range(N)], dtype=torch.int32,
                              device=device)
        row_start = torch.tensor([c * C for c in range(N + 1)], dtype=torch.int32, device=device)
        K, R = 64, 2
        max_past = (N - 1) * w.pages_per_chunk
        out_l = torch.empty((N, Hkv, K + R), dtype=torch.int32, device=device)
        out_c = torch.empty((N, Hkv), dtype=torch.int32, device=device)
        ws = torch.empty(pk.page_topk_batched_workspace_size(N, Hkv, d, max_past),
                         dtype=torch.uint8, device=device)
        ms = _event_ms(lambda: pk.page_topk_batched(a, q_all, row_start, C, n_past, max_past,
                                                    table, K, R, out_l, None, out_c, ws))
        n_scored = int(n_past.sum())
        nb = N * C * Hq * d * 2 + n_scored * (Hkv * d * 4 + 4) + N * Hkv * (K + R) * 4
        out["topk_batched_all_chunks"] = entry(
            nb, ms, hbm, f"{N} chunks x {Hkv} groups in one batched call (query means of "
            f"{N * C} rows, {n_scored} page scores per group, K={K}, R={R})")
        del q_all
        # gather / scatter-add of every block of the shuffled pool
        nblk = npg * Hkv
        perm = torch.randperm(nblk, device=device, generator=gen).to(torch.int32)
        ident = torch.arange(nblk, dtype=torch.int32, device=device)
        ms = _event_ms(lambda: pk.block_copy(a, b, perm, ident))
        nb = nblk * (2 * P * d * 2 * 2 + d * 4 * 2)
        out["block_gather_all_pages"] = entry(nb, ms, hbm, f"{nblk} shuffled (page, head) "
                                              "blocks (K, V, page mean) device -> device")
        ms = _event_ms(lambda: pk.grad_block_add(a, b, perm, ident, zero_src=False))
        nb = nblk * 2 * P * d * 4 * 3
        out["grad_scatter_add_all_pages"] = entry(nb, ms, hbm, f"{nblk} shuffled fp32 gradient "
                                                  "blocks added into another pool (read src, "
                                                  "read + write dst)")
        # host link: memcpy peak, then the same moves to / from pinned pages
        big = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
        dbig = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        ms_h2d = _event_ms(lambda: dbig.copy_(big, non_blocking=True), reps=3)
        ms_d2h = _event_ms(lambda: big.copy_(dbig, non_blocking=True), reps=3)
        peak_h2d = (256 << 20) / (ms_h2d / 1e3) / 1e9
        peak_d2h = (256 << 20) / (ms_d2h / 1e3) / 1e9
        del big, dbig
        h = pk.pool_create(npg, P, Hkv, d, pk.LOC_PINNED_HOST, True, 0, dev_i)
        blk_kv = 2 * P * d * 2
        ms = _event_ms(lambda: pk.block_copy(a, h, perm, ident), reps=3)
        link = {"memcpy_h2d_gbs": peak_h2d, "memcpy_d2h_gbs": peak_d2h}
        link["store_all_blocks_d2h"] = entry(nblk * blk_kv, ms, peak_d2h,
                                             f"{nblk} shuffled KV blocks device -> pinned host")
        ms = _event_ms(lambda: pk.block_copy(h, b, ident, perm), reps=3)
        link["gather_all_blocks_h2d"] = entry(nblk * blk_kv, ms, peak_h2d,
                                              f"{nblk} KV blocks pinned host -> shuffled device")
        sel = perm[:(K + R) * Hkv].contiguous()
        ms = _event_ms(lambda: pk.block_copy(h, b, sel, ident[:sel.numel()].contiguous()))
        link["gather_one_chunk_selection_h2d"] = entry(
            sel.numel() * blk_kv, ms, peak_h2d, f"{sel.numel()} KV blocks (one chunk's "
            "selection) pinned host -> device")
        ms = _event_ms(lambda: pk.grad_block_add(a, h, perm, ident, zero_src=False), reps=3)
        link["grad_add_all_blocks_to_host"] = entry(
            nblk * 2 * P * d * 4, ms, min(peak_h2d, peak_d2h), f"{nblk} fp32 gradient blocks "
            "added into pinned host pages (each byte crosses the link both ways)")
        out["host_link"] = link
        torch.cuda.synchronize()
        out["device_status"] = (pk.get_device_status(a) | pk.get_device_status(b) |
                                pk.get_device_status(h))
    finally:
        for pool in (a, b, h):
            if pool:
                pk.pool_destroy(pool)
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w, rows, seed_chunk=None):
    """Bounded sample of the same workload for the CPU oracle: the first `rows`
    query rows of chunk N/2 (all heads), as a chunk of their own, against every
    past key of that chunk, forward and backward.  Returns (seconds,
    algorithmic FLOPs, threads used, description)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle.attention import chunk_backward, chunk_forward
    from paged_kv_chunk_query_b200 import synth
    c = w.num_chunks // 2 if seed_chunk is None else seed_chunk
    C = w.chunk_len
    ch = synth.chunk_inputs(w, c)
    q = ch["q"][:rows].float().numpy().astype(np.float64)
    do = ch["do"][:rows].float().numpy().astype(np.float64)
    kc, vc = ch["k"][:rows].float().numpy(), ch["v"][:rows].float().numpy()
    past_k, past_v = [], []
    for cc in range(c):  # past keys of chunk c, drawn chunk by chunk (not timed)
        x = synth.chunk_inputs(w, cc, which=("k", "v"))
        past_k.append(x["k"].float().numpy())
        past_v.append(x["v"].float().numpy())
    pk_ = np.concatenate(past_k).astype(np.float64)
    pv_ = np.concatenate(past_v).astype(np.float64)
    Hkv = w.num_kv_heads
    kp = [pk_[:, g, :] for g in range(Hkv)]
    vp = [pv_[:, g, :] for g in range(Hkv)]
    t0 = time.perf_counter()
    chunk_forward(q, kp, vp, kc, vc, w.softmax_scale)
    chunk_backward(q, kp, vp, kc, vc, do, w.softmax_scale)
    dt = time.perf_counter() - t0
    pairs = pairs_of_chunk(rows, c * C) * w.num_q_heads
    flops = 14.0 * pairs * w.head_dim
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    desc = (f"{w.name}: first {rows} rows of chunk {c} (all {w.num_q_heads} heads) against its "
            f"{c * C} past keys + causal self, fp64 numpy fwd+bwd")
    return dt, flops, threads, desc


def oracle_tiny_full():
    """The tiny workload (L 512, Hq 4, Hkv 1, d 64, 16-token pages, 8 chunks of
    64) run in full by the oracle, fwd+bwd: (seconds, algorithmic FLOPs)."""
    from oracle.recurrent import run_sequence
    from paged_kv_chunk_query_b200 import synth
    w = synth.WORKLOADS["tiny"]
    inp = synth.sequence_inputs(w)
    t0 = time.perf_counter()
    run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                 w.softmax_scale)
    dt = time.perf_counter() - t0
    return dt, 14.0 * step_pairs(w, False) * w.head_dim


def cpu_baseline_obj(w, rows):
    """The oracle as it stands on a bounded sample of the headline workload,
    plus the tiny workload in full and the sample's rate extrapolated (and
    labelled as such) to one whole step."""
    dt, fl, threads, desc = oracle_sample(w, rows)
    rate = fl / dt
    tdt, tfl = oracle_tiny_full()
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": desc, "seconds": dt,
            "tiny_full_run": {"seconds": tdt, "tflops": tfl / tdt / 1e12,
                              "what": "tiny workload (L 512) fwd+bwd in full, fp64"},
            "extrapolated_full_step_seconds": step_pairs(w, False) * 14.0 * w.head_dim / rate,
            "extrapolation_note": "the sample's TFLOP/s applied to the whole dense step's "
                                  "algorithmic FLOPs; an estimate, not a measurement"}


# ------------------------------------------------------------------ roofline bits
def _traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e:
        return None
    # the kernel's source and the headers it includes, hashed in order
    h = hashlib.sha256()
    for rel in e.get("sources", [e.get("source")]):
        src = os.path.join(ROOT, rel) if rel else ""
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    if h.hexdigest() != e["sha256"]:
        return None
    return e


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen256k")
    ap.add_argument("--sparse-workload", default=None,
                    help="sparse run's workload (default: the Top-K variant of --workload)")
    ap.add_argument("--no-sparse", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-offload", action="store_true")
    ap.add_argument("--no-hbm", action="store_true", help="skip the batched HBM/host-link kernels")
    ap.add_argument("--no-local", action="store_true", help="skip the recent-only page-list run")
    ap.add_argument("--local-workload", default="qwen256k_local")
    ap.add_argument("--no-qtile", action="store_true", help="skip the per-query-tile Top-K run")
    ap.add_argument("--no-projection", action="store_true",
                    help="skip the Q/K/V projection GEMM measurement")
    ap.add_argument("--no-dense-offload", action="store_true",
                    help="skip the dense run with host-resident KV and a device window")
    ap.add_argument("--dense-window", type=int, default=512, help="window pages (two slots)")
    ap.add_argument("--dense-grad-path", choices=["gpu", "host"], default="host",
                    help="gradient write-back of the dense offload run")
    ap.add_argument("--qtile-workload", default="qwen256k_topk_qtile")
    ap.add_argument("--no-qpage", action="store_true", help="skip the per-query-page Top-K run")
    ap.add_argument("--qpage-workload", default="qwen256k_topk_qpage")
    ap.add_argument("--fwd-overlap", action="store_true",
                    help="run each chunk's forward on a third stream beside the previous backward")
    ap.add_argument("--serial-bwd", action="store_true",
                    help="run each chunk's dQ launch after its dK/dV launch on one stream")
    ap.add_argument("--offload-workload", default="qwen1m_topk_offload")
    ap.add_argument("--cpu-rows", type=int, default=0, help="oracle sample rows (0: auto)")
    ap.add_argument("--no-32k", action="store_true", help="skip the 32K dense throughput line")
    ap.add_argument("--small-workload", default="qwen32k")
    a = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from paged_kv_chunk_query_b200 import synth
    w = synth.WORKLOADS[a.workload]
    ws_name = a.sparse_workload or (a.workload + "_topk" if a.workload + "_topk" in synth.WORKLOADS
                                    else a.workload)

    if a.impl == "reference":
        # The reference arm is the CPU oracle as it stands, rank 0 only.
        if rank != 0:
            return
        # the sample shrinks with the number of steps so the whole run stays
        # near two minutes (64 rows for 8 steps; rate units are per second)
        rows = a.cpu_rows or max(16, min(64, 64 * 8 // max(1, a.steps + a.warmup)))
        for _ in range(a.warmup):
            oracle_sample(w, rows)
        secs, flops = [], 0.0
        threads, desc = 1, ""
        for _ in range(a.steps):
            dt, flops, threads, desc = oracle_sample(w, rows)
            secs.append(dt)
        dt = sum(secs) / len(secs)
        val = flops / dt / 1e12
        line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": 0, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": {"workload": w.name, "sample": desc},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads,
                                 "kind": "oracle", "sample": desc},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import paged_kv_chunk_query_b200 as pk  # noqa: F401  (fails loudly without the library)

    clocks = Clocks(local)
    dense = Run(w, False, device)
    dense.concurrent_bwd = not a.serial_bwd
    dense.fwd_overlap = a.fwd_overlap
    clocks.start()
    ms, kt = time_steps(dense, a.steps, a.warmup, dist_on, device)
    clk = clocks.stop()
    dense_status = pk.get_device_status(dense.pool)
    step_flops = dense.step_flops
    launches_dense = dense.launches_per_step
    fwd_merge = dense.fwd_merge
    value = whole_job_rate(step_flops, ms, world) / 1e12
    tokens = whole_job_rate(w.context, ms, world)
    kernel_flops = {k: sum(v) for k, v in dense.flops.items()}
    kt_serial = None
    if dense.concurrent_bwd:
        # one more step, untimed as a whole, in the serial schedule: per-kernel
        # event times without co-scheduled launches of the other stream
        dense.concurrent_bwd = False
        timers = {}
        dense.step(timers)
        torch.cuda.synchronize()
        kt_serial = {n: sum(x.elapsed_time(y) for x, y in ev) for n, ev in timers.items()}
    dense.close()
    del dense
    torch.cuda.empty_cache()

    peaks = _peaks()
    # dominant kernel: the one credited with the most algorithmic work (dK/dV;
    # it also has the largest share of the serial launch list).  With the
    # two-stream backward, event times of a launch include co-scheduled CTAs.
    dom = max(kernel_flops, key=kernel_flops.get)
    dom_ms = kt[dom]
    tr = _traffic(dom)
    clock_peak = clock_scaled_peak(peaks["bf16"], clk.get("sm_mhz"), peaks.get("sm_max_mhz"))
    if dom in kernel_flops:
        achieved = kernel_flops[dom] / (dom_ms / 1e3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved,
                "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_sustained"],
                "frac_of_burst": achieved / peaks["bf16"],
                "frac_clock_normalised": achieved / clock_peak if clock_peak else None,
                "clock_normalised_peak": clock_peak,
                "peak_source": f"bf16_tflops_sustained ({peaks['source']}); burst "
                               f"{peaks['bf16']:.1f}; clock-normalised = burst x median SM MHz "
                               "of this run / max SM MHz",
                "traffic": tr["bytes_per_launch"] if tr else None,
                "launch_share": dom_ms / ms}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": None, "traffic": tr["bytes_per_launch"] if tr else None}
    kernels = {k: {"ms_per_step": v, "share": v / ms,
                   "tflops": (kernel_flops[k] / (v / 1e3) / 1e12) if k in kernel_flops else None}
               for k, v in kt.items()}

    sparse_obj = None
    if not a.no_sparse:
        ws = synth.WORKLOADS[ws_name]
        sp = Run(ws, True, device)
        sp.concurrent_bwd = not a.serial_bwd
        sp.fwd_overlap = a.fwd_overlap
        ms_s, kt_s = time_steps(sp, a.steps, a.warmup, dist_on, device)
        sparse_status = pk.get_device_status(sp.pool)
        topk_bytes = 0.0
        C, Hq, Hkv, d = ws.chunk_len, ws.num_q_heads, ws.num_kv_heads, ws.head_dim
        for c in range(1, ws.num_chunks):
            n_past = c * ws.pages_per_chunk
            topk_bytes += C * Hq * d * 2 + n_past * (Hkv * d * 4 + 4) + Hkv * (ws.top_k + ws.n_recent) * 8
        topk_in_step_ms = kt_s.get("topk", 0.0)
        topk_ms, topk_qsum_ms = sp.time_topk_alone()
        n_sel = ws.num_chunks - 1
        topk_qsum_bytes = topk_bytes - n_sel * C * Hq * d * 2
        sparse_obj = {"workload": ws.name, "value": sp.step_flops * world / (ms_s / 1e3) / 1e12,
                      "gpu_launches": sp.launches_per_step * a.steps,
                      "unit": "TFLOP/s", "ms_per_step": ms_s,
                      "tokens_per_s": ws.context * world / (ms_s / 1e3),
                      "dense_over_sparse_time": ms / ms_s,
                      "kernels": {k: {"ms_per_step": v, "share": v / ms_s} for k, v in kt_s.items()},
                      "topk_hbm": {"bound": "hbm", "achieved": topk_bytes / (topk_ms / 1e3) / 1e9
                                   if topk_ms else None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                   "frac": (topk_bytes / (topk_ms / 1e3) / 1e9) / peaks["hbm_gbs"]
                                   if topk_ms else None,
                                   "ms_per_step_alone": topk_ms,
                                   "us_per_chunk_alone": topk_ms * 1e3 / n_sel,
                                   "ms_per_step_in_step": topk_in_step_ms,
                                   "from_qsum": {
                                       "ms_per_step_alone": topk_qsum_ms,
                                       "us_per_chunk_alone": topk_qsum_ms * 1e3 / n_sel,
                                       "achieved": topk_qsum_bytes / (topk_qsum_ms / 1e3) / 1e9,
                                       "frac": topk_qsum_bytes / (topk_qsum_ms / 1e3) / 1e9
                                       / peaks["hbm_gbs"],
                                       "note": "one launch per chunk (scores + select) from "
                                       "per-group Q sums such as the projection's epilogue "
                                       "writes; reads the page summaries only"},
                                   "note": "all chunks' selections timed back to back, alone, "
                                   "replayed from a CUDA graph (query mean, page scores, radix "
                                   "select per chunk); in the "
                                   "step chunk c+1's selection runs on its own stream beside "
                                   "chunk c's attention, and ms_per_step_in_step is its event "
                                   "time there (overlapped, off the critical path)"},
                      "device_status": sparse_status}
        sp.close()
        del sp
        torch.cuda.empty_cache()

    small_obj = None
    if not a.no_32k:
        w32 = synth.WORKLOADS[a.small_workload]
        r32 = Run(w32, False, device)
        r32.concurrent_bwd = not a.serial_bwd
        r32.fwd_overlap = a.fwd_overlap
        clk32 = Clocks(local)
        clk32.start()
        ms_32, kt_32 = time_steps(r32, max(a.steps, 5), a.warmup, dist_on, device)
        c32 = clk32.stop()
        tf32 = r32.step_flops / (ms_32 / 1e3) / 1e12
        small_obj = {"workload": w32.name, "context": w32.context,
                     "value": tf32 * world, "unit": "TFLOP/s", "ms_per_step": ms_32,
                     "steps": max(a.steps, 5), "tokens_per_s": w32.context * world / (ms_32 / 1e3),
                     "tflop_per_step": r32.step_flops / 1e12,
                     "fractions_of_bf16_peak": step_fractions(tf32, _peaks(), c32.get("sm_mhz")),
                     "clocks": c32,
                     "kernels": {k: {"ms_per_step": v} for k, v in kt_32.items()},
                     "device_status": pk.get_device_status(r32.pool)}
        r32.close()
        del r32
        torch.cuda.empty_cache()

    local_obj = None
    if not a.no_local:
        wl = synth.WORKLOADS[a.local_workload]
        lr = Run(wl, False, device)
        lr.concurrent_bwd = not a.serial_bwd
        lr.fwd_overlap = a.fwd_overlap
        ms_l, kt_l = time_steps(lr, a.steps, a.warmup, dist_on, device)
        local_obj = {"workload": wl.name, "window_pages": wl.window,
                     "value": lr.step_flops * world / (ms_l / 1e3) / 1e12, "unit": "TFLOP/s",
                     "ms_per_step": ms_l, "tokens_per_s": wl.context * world / (ms_l / 1e3),
                     "kernels": {k: {"ms_per_step": v} for k, v in kt_l.items()},
                     "device_status": pk.get_device_status(lr.pool)}
        lr.close()
        del lr
        torch.cuda.empty_cache()

    qtile_obj = None
    if not a.no_qtile:
        wq = synth.WORKLOADS[a.qtile_workload]
        qr = Run(wq, True, device)
        qr.concurrent_bwd = not a.serial_bwd
        qr.fwd_overlap = a.fwd_overlap
        ms_q, kt_q = time_steps(qr, a.steps, a.warmup, dist_on, device)
        qtile_obj = {"workload": wq.name, "selection": "Top-K per 128-row query tile",
                     "value": qr.step_flops * world / (ms_q / 1e3) / 1e12, "unit": "TFLOP/s",
                     "ms_per_step": ms_q, "tokens_per_s": wq.context * world / (ms_q / 1e3),
                     "kernels": {k: {"ms_per_step": v} for k, v in kt_q.items()},
                     "device_status": pk.get_device_status(qr.pool)}
        qr.close()
        del qr
        torch.cuda.empty_cache()

    qpage_obj = None
    if not a.no_qpage:
        wp = synth.WORKLOADS[a.qpage_workload]
        qp = Run(wp, True, device)
        qp.concurrent_bwd = not a.serial_bwd
        qp.fwd_overlap = a.fwd_overlap
        ms_p, kt_p = time_steps(qp, a.steps, a.warmup, dist_on, device)
        qpage_obj = {"workload": wp.name,
                     "selection": f"Top-K per {wp.page_size}-token query page; per 128-row "
                                  "query tile the union of its query pages' lists with "
                                  "membership masks",
                     "value": qp.step_flops * world / (ms_p / 1e3) / 1e12, "unit": "TFLOP/s",
                     "ms_per_step": ms_p, "tokens_per_s": wp.context * world / (ms_p / 1e3),
                     "kernels": {k: {"ms_per_step": v} for k, v in kt_p.items()},
                     "device_status": pk.get_device_status(qp.pool)}
        qp.close()
        del qp
        torch.cuda.empty_cache()

    offload_obj = None
    if not a.no_offload:
        offload_obj = offload_run(synth.WORKLOADS[a.offload_workload], max(1, min(a.steps, 2)),
                                  device, dist_on)
        if sparse_obj and offload_obj:
            # per-chunk time against the device-resident Top-K run of the same shape
            per_chunk_dev = sparse_obj["ms_per_step"] / synth.WORKLOADS[ws_name].num_chunks
            offload_obj["ms_per_chunk_device_resident"] = per_chunk_dev
            offload_obj["overhead_vs_device_resident"] = (
                offload_obj["ms_per_chunk"] / per_chunk_dev - 1.0)
        offload_obj["tokens_per_s"] *= world

    dense_off_obj = None
    if not a.no_dense_offload:
        dense_off_obj = dense_offload_run(w, a.dense_window, device, dist_on, a.dense_grad_path)
        dense_off_obj["ms_per_step_device_resident"] = ms
        dense_off_obj["overhead_vs_device_resident"] = dense_off_obj["ms_per_step"] / ms - 1.0
        dense_off_obj["tokens_per_s"] *= world

    proj_obj = None
    if not a.no_projection:
        proj_obj = projection_run(w, device, peaks)

    hbm_obj = None
    if not a.no_hbm:
        hbm_obj = hbm_kernels(w, device, peaks)

    e2e = None
    if not a.no_e2e:
        _barrier(dist_on)
        ms_e, h2d, d2h = e2e_dense(w, max(1, min(a.steps, 2)), device)
        ms_e = _max_over_ranks(ms_e, dist_on, device)   # every rank runs this line
        e2e = {"value": step_flops * world / (ms_e / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu:
        cpu = cpu_baseline_obj(w, a.cpu_rows or 64)

    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "context": w.context, "chunk_len": w.chunk_len,
                   "num_chunks": w.num_chunks, "page_size": w.page_size,
                   "heads": f"{w.num_q_heads}q/{w.num_kv_heads}kv", "head_dim": w.head_dim,
                   "page_table": "shuffled" if w.shuffle_pages else "identity",
                   "parallelism": f"replicas{world}",
                   "fwd_schedule": "one CTA per (128-row query tile, head); the last partial "
                   "wave split along its key tiles over the idle SMs, merged by a second launch"
                   if fwd_merge else "one CTA per (128-row query tile, head)",
                   "bwd_schedule": "serial" if a.serial_bwd else
                   "dQ on a second stream beside dK/dV; next chunk's append issued early",
                   "l2": "inputs larger than L2 (Q+dO 3.5 GiB, KV pool 512 MiB, grad pool 1 GiB)"},
        "tokens_per_s": tokens,
        "kernels": kernels,
        "kernels_serial_step": None if kt_serial is None else {
            k: {"ms_per_step": v, "tflops": (kernel_flops[k] / (v / 1e3) / 1e12)
                if k in kernel_flops else None} for k, v in kt_serial.items()},
        "roofline": roof,
        "step_fractions_of_bf16_peak": step_fractions(value / world, peaks, clk.get("sm_mhz")),
        "ms_x_median_sm_mhz": ms * clk["sm_mhz"] if clk.get("sm_mhz") else None,
        "qwen32k": small_obj,
        "sparse": sparse_obj,
        "local": local_obj,
        "qtile_topk": qtile_obj,
        "qpage_topk": qpage_obj,
        "offload": offload_obj,
        "dense_offload": dense_off_obj,
        "projection": proj_obj,
        "hbm_kernels": hbm_obj,
        "e2e": e2e,
        "cpu_baseline": cpu,
        # launches of this library's kernels inside the headline's timed region
        "gpu_launches": launches_dense * a.steps,
        "clocks": clk,
        "device_status": dense_status,
        "peaks": peaks,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
