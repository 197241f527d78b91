"""GPU parity at the full workload sizes, in the schedule the benchmark times.

The attention of a chunk's queries against a paged KV cache of every earlier
chunk, forward and backward with gradients added in place into the paged pool
([pt] §2B "Kernels Personalizados"; [it] §2B), and its page-level Top-K
variant ([pt] §2C; [es] §2B "Atención Escasa a Nivel de Página"), run here at
the sizes the throughput figures are quoted on: 4096-token chunks of the
Qwen2.5-7B attention shape (28 query heads, 4 KV heads, d 128, 64-token
pages), over 32K and 256K contexts (dense and Top-K), and the 1M-token
offloaded Top-K run.

Every run goes through ``bench.Run.step`` — the very launches, streams and
arguments the benchmark times — on inputs drawn on the CPU by the seeded
generator, so the fp64 oracle sees the same bytes.  A whole chunk in fp64 is
out of reach at these sizes, so the oracle is evaluated on samples:

* O, LSE (rel L2 <= 5e-3, max abs <= 1e-2) and dQ (rel L2 <= 1e-2) of 256
  rows of every query head (first and last row of the chunk included) of
  sampled chunks, against every key the row sees;
* one chunk's dK / dV on 8 sampled pages per KV-head group (rel L2 <= 1e-2):
  the gradient pool is zeroed and that chunk's backward launches re-run, so
  the pool holds that chunk's contribution alone;
* on the gradient pool the whole step accumulated, two sums the softmax fixes
  exactly: sum over keys of dK_g = 0 (each row's dS sums to zero over its
  keys) and sum over keys of dV_g = sum of dO over the group's rows (each
  row's P sums to one).  The GPU forms P and dS in bf16, so the first holds
  to the size of the per-key error: |sum dK_g| <= 1e-2 ||dK_g||_F, and the
  second to rel L2 <= 1e-2 (the backward tolerance);
* Top-K page ids of every chunk bit for bit, except pages whose fp64 score
  lies within 1e-5 of the K-th score.

The per-query-page Top-K workload (one selection per 64-token query page)
is checked on its selections, sampled rows (each against its own query
page's pages), the gradient-pool sums, and one chunk's dK / dV on sampled
pages (each block of rows contributing through its own key set).

The 1M offloaded run (KV and gradients in pinned host memory, selected pages
prefetched into a staging pool) is checked against the same workload with
every page in HBM: identical selections, bit-equal forward outputs and dQ on
sampled chunks, and host gradient pool against device pool within rel L2
1e-3.  Its inputs are drawn on the device (values are compared GPU against
GPU; the kernels' agreement with the oracle at this shape is what the 256K
Top-K case shows).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import bench
import paged_kv_chunk_query_b200 as pk
from oracle.attention import chunk_keys_backward, chunk_rows_backward
from oracle.sparse import group_query_means, kth_score, page_key_means, page_scores, select_pages
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import rel_l2, to64

pytestmark = pytest.mark.gpu

ROWS = 256            # sampled query rows per head and chunk
PAGES = 8             # sampled key pages per group for the single-chunk dK/dV
TIE = 1e-5
FWD_REL, FWD_ABS, BWD_REL = 5e-3, 1e-2, 1e-2


def _dev():
    return torch.device("cuda", 0)


def _draw(w):
    """Every chunk's q, k, v, dO from the seeded CPU generator (threads:
    each chunk and tensor has its own generator, so the values do not depend
    on the order)."""
    with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        return list(ex.map(lambda c: synth.chunk_inputs(w, c), range(w.num_chunks)))


def _keys(cpu):
    """K and V of the whole sequence, [L][Hkv][d] fp32 numpy (bf16 values)."""
    k = torch.cat([x["k"] for x in cpu]).float().numpy()
    v = torch.cat([x["v"] for x in cpu]).float().numpy()
    return k, v


def _run(w, sparse, cpu):
    dev = _dev()
    ins = [{key: t.to(dev) for key, t in x.items()} for x in cpu]
    run = bench.Run(w, sparse, dev, inputs=ins)
    run.step()
    torch.cuda.synchronize()
    assert pk.get_device_status(run.pool) == 0
    return run


def _close(run):
    run.close()
    torch.cuda.empty_cache()


def _selected(run, c):
    """Per group, the kept logical pages of chunk c (sparse runs)."""
    cnt = run.sel_n[c].cpu().tolist()
    sel = run.sel_l[c].cpu()
    return [sel[g, :cnt[g]].tolist() for g in range(len(cnt))]


def _tokens(w, c, pages):
    """Absolute token positions a chunk-c row may see: the tokens of `pages`
    (None: every earlier token) followed by the chunk's own tokens."""
    C, P = w.chunk_len, w.page_size
    if pages is None:
        past = np.arange(c * C)
    elif len(pages):
        past = (np.asarray(pages, dtype=np.int64)[:, None] * P + np.arange(P)[None, :]).reshape(-1)
    else:
        past = np.zeros(0, dtype=np.int64)
    return np.concatenate([past, np.arange(c * C, (c + 1) * C)]).astype(np.int64)


def _sample_rows(C, seed):
    rng = np.random.default_rng(seed)
    inner = rng.choice(np.arange(1, C - 1), size=ROWS - 2, replace=False)
    return np.sort(np.concatenate([[0, C - 1], inner]))


def _check_rows(w, run, cpu, kf, vf, c, selected=None, block_rows=None):
    """O, LSE, dQ of ROWS sampled rows of every head of chunk c against the
    oracle over every key those rows see.  `selected`: per group the kept
    pages (None: dense); with `block_rows`, per block of that many rows a
    per-group selection (the rows of block b see selected[b][g])."""
    C, Hq, Hkv = w.chunk_len, w.num_q_heads, w.num_kv_heads
    G = Hq // Hkv
    rows = _sample_rows(C, 9000 + c)
    idx = torch.tensor(rows, device=run.o[c].device)
    o_gpu = to64(run.o[c][idx])                       # [R][Hq][d]
    lse_gpu = to64(run.lse[c][:, idx])                # [Hq][R]
    dq_gpu = to64(run.dq[c][idx])
    q = cpu[c]["q"][rows].double().numpy()
    do = cpu[c]["do"][rows].double().numpy()
    o_ref, lse_ref, dq_ref = np.zeros_like(o_gpu), np.zeros_like(lse_gpu), np.zeros_like(dq_gpu)
    if block_rows is None:
        groups = [(np.arange(len(rows)), selected)]
    else:
        blk = rows // block_rows
        groups = [(np.nonzero(blk == b)[0], selected[b]) for b in np.unique(blk)]
    for sel_rows, sel in groups:
        for g in range(Hkv):
            tok = _tokens(w, c, None if sel is None else sel[g])
            kk = kf[tok, g].astype(np.float64)
            vv = vf[tok, g].astype(np.float64)
            for h in range(g * G, (g + 1) * G):
                o_ref[sel_rows, h], lse_ref[h, sel_rows], dq_ref[sel_rows, h] = \
                    chunk_rows_backward(q[sel_rows, h], do[sel_rows, h], c * C + rows[sel_rows],
                                        kk, vv, tok, w.softmax_scale)
    assert rel_l2(o_gpu, o_ref) <= FWD_REL, (c, rel_l2(o_gpu, o_ref))
    assert np.max(np.abs(o_gpu - o_ref)) <= FWD_ABS, c
    assert rel_l2(lse_gpu, lse_ref) <= FWD_REL, c
    assert np.max(np.abs(lse_gpu - lse_ref)) <= FWD_ABS, c
    assert rel_l2(dq_gpu, dq_ref) <= BWD_REL, (c, rel_l2(dq_gpu, dq_ref))


def _check_sums(w, run):
    """Sum over keys of dK_g = 0 and of dV_g = sum of dO over the group's rows,
    on the gradient pool the whole step accumulated."""
    Hq, Hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim
    G = Hq // Hkv
    _, grad, _ = pk.pool_views(run.pool)
    ids = run.page_table_dev.long()
    dk_sum = torch.zeros((Hkv, d), dtype=torch.float64, device=grad.device)
    dv_sum = torch.zeros_like(dk_sum)
    dk_sq = torch.zeros(Hkv, dtype=torch.float64, device=grad.device)
    for part in ids.split(1024):                       # pages in slices (fp64 copies)
        g = grad[part].double()                        # [pages][Hkv][2][P][d]
        dk_sum += g[:, :, 0].sum(dim=(0, 2))
        dv_sum += g[:, :, 1].sum(dim=(0, 2))
        dk_sq += g[:, :, 0].pow(2).sum(dim=(0, 2, 3))
    do_sum = torch.zeros_like(dk_sum)
    for x in run.inputs:
        do_sum += x["do"].double().view(-1, Hkv, G, d).sum(dim=(0, 2))
    for g in range(Hkv):
        assert float(dk_sum[g].norm()) <= 1e-2 * float(dk_sq[g].sqrt()), g
        assert float((dv_sum[g] - do_sum[g]).norm()) <= 1e-2 * float(do_sum[g].norm()), g


def _check_single_chunk_grads(w, run, cpu, kf, vf, c, selected=None):
    """Zero the gradient pool, re-run chunk c's backward launches as the step
    issues them, and compare dK / dV of PAGES sampled pages per group with
    the oracle's one-chunk contribution."""
    C, Hq, Hkv, P = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.page_size
    G = Hq // Hkv
    _, grad, _ = pk.pool_views(run.pool)
    grad.zero_()
    x = run.inputs[c]
    if selected is None:
        past, cnt = run.dense_past[c], run.dense_cnt[c]
    else:
        past, cnt = run.sel_p[c], run.sel_n[c]
    for step in (pk.BWD_PREPROCESS, pk.BWD_DKDV):
        pk.chunk_attn_bwd(run.pool, x["q"], run.o[c], run.lse[c], x["do"], run.dq[c],
                          run.deltas[c], past, cnt, run.cur[c], w.softmax_scale, step=step)
    torch.cuda.synchronize()
    assert pk.get_device_status(run.pool) == 0
    q = cpu[c]["q"].double().numpy()
    do = cpu[c]["do"].double().numpy()
    rng = np.random.default_rng(9500 + c)
    ppc = w.pages_per_chunk
    for g in range(Hkv):
        past_pages = list(range(c * ppc)) if selected is None else list(selected[g])
        pages = past_pages + list(range(c * ppc, (c + 1) * ppc))
        # first and last listed page, the chunk's first page, the rest at random
        must = sorted({pages[0], pages[-1], c * ppc})
        rest = [p for p in pages if p not in must]
        pick = sorted(must + rng.choice(rest, size=PAGES - len(must), replace=False).tolist())
        tok = _tokens(w, c, None if selected is None else selected[g])
        pos_in = {int(t): i for i, t in enumerate(tok)}
        key_idx = np.array([pos_in[p * P + t] for p in pick for t in range(P)])
        dk_ref, dv_ref = chunk_keys_backward(
            q[:, g * G:(g + 1) * G], do[:, g * G:(g + 1) * G], c * C + np.arange(C),
            kf[tok, g].astype(np.float64), vf[tok, g].astype(np.float64), tok, key_idx,
            w.softmax_scale)
        phys = torch.tensor([run.page_table[p] for p in pick], dtype=torch.long,
                            device=grad.device)
        blk = to64(grad[phys, g])                      # [PAGES][2][P][d]
        dk_gpu = blk[:, 0].reshape(-1, w.head_dim)
        dv_gpu = blk[:, 1].reshape(-1, w.head_dim)
        assert rel_l2(dk_gpu, dk_ref) <= BWD_REL, (g, rel_l2(dk_gpu, dk_ref))
        assert rel_l2(dv_gpu, dv_ref) <= BWD_REL, (g, rel_l2(dv_gpu, dv_ref))


def _check_topk(w, run, cpu, kf, chunks):
    """Kept pages of the given chunks against the oracle's selection (tie band)."""
    P, Hkv, C = w.page_size, w.num_kv_heads, w.chunk_len
    kbar_all = page_key_means(kf, P)                  # [pages][Hkv][d]
    for c in chunks:
        n_past = c * w.pages_per_chunk
        ref_scores = page_scores(group_query_means(cpu[c]["q"], Hkv), kbar_all[:n_past])
        want = select_pages(ref_scores, n_past, w.top_k, w.n_recent)
        got = _selected(run, c)
        for g in range(Hkv):
            assert got[g] == sorted(set(got[g])), (c, g)
            assert len(got[g]) == min(w.top_k, max(0, n_past - w.n_recent)) + \
                min(w.n_recent, n_past), (c, g)
            assert set(range(max(0, n_past - w.n_recent), n_past)) <= set(got[g]), (c, g)
            kth = kth_score(ref_scores[g], n_past, w.top_k, w.n_recent)
            for p in set(got[g]) ^ set(want[g]):
                assert kth is not None and abs(ref_scores[g, p] - kth) <= TIE, (c, g, p)
        # the physical ids are the page table's
        phys = run.sel_p[c].cpu()
        cnt = run.sel_n[c].cpu().tolist()
        for g in range(Hkv):
            assert phys[g, :cnt[g]].tolist() == [run.page_table[p] for p in got[g]]


def test_fullsize_qwen32k_dense():
    """32K context, 8 chunks of 4096, dO ~ N(0, 1e-2^2): every chunk's sampled
    rows, the single-chunk dK / dV of the last chunk, the gradient-pool sums."""
    w = synth.WORKLOADS["qwen32k"]
    cpu = _draw(w)
    kf, vf = _keys(cpu)
    run = _run(w, False, cpu)
    try:
        _check_sums(w, run)
        for c in range(w.num_chunks):
            _check_rows(w, run, cpu, kf, vf, c)
        _check_single_chunk_grads(w, run, cpu, kf, vf, w.num_chunks - 1)
    finally:
        _close(run)


def test_fullsize_qwen256k_dense():
    """256K context over a shuffled page table: chunks 0, 1, N/2 and N-1
    (262,144 keys), the gradient-pool sums after 64 chunks, and one chunk's
    dK / dV on sampled pages."""
    w = synth.WORKLOADS["qwen256k"]
    cpu = _draw(w)
    kf, vf = _keys(cpu)
    run = _run(w, False, cpu)
    try:
        _check_sums(w, run)
        N = w.num_chunks
        for c in (0, 1, N // 2, N - 1):
            _check_rows(w, run, cpu, kf, vf, c)
        _check_single_chunk_grads(w, run, cpu, kf, vf, 4)
    finally:
        _close(run)


def test_fullsize_qwen256k_topk():
    """256K Top-64 + 2 recent pages per chunk and group: every chunk's
    selection, sampled rows of chunks 1, N/2 and N-1 on the GPU's selection,
    the gradient-pool sums, and the last chunk's dK / dV on sampled pages."""
    w = synth.WORKLOADS["qwen256k_topk"]
    cpu = _draw(w)
    kf, vf = _keys(cpu)
    run = _run(w, True, cpu)
    try:
        N = w.num_chunks
        _check_topk(w, run, cpu, kf, range(1, N))
        _check_sums(w, run)
        for c in (1, N // 2, N - 1):
            _check_rows(w, run, cpu, kf, vf, c, _selected(run, c))
        _check_single_chunk_grads(w, run, cpu, kf, vf, N - 1, _selected(run, N - 1))
    finally:
        _close(run)


def test_fullsize_qwen256k_topk_per_query_page():
    """256K Top-64 + 2 recent pages per 64-token query page and group: the
    selections of chunks 1, N/2 and N-1 (every query page), sampled rows of
    those chunks each against its own query page's pages, the gradient-pool
    sums, and the last chunk's dK / dV on sampled pages."""
    w = synth.WORKLOADS["qwen256k_topk_qpage"]
    cpu = _draw(w)
    kf, vf = _keys(cpu)
    run = _run(w, True, cpu)
    try:
        N, P, Hkv = w.num_chunks, w.page_size, w.num_kv_heads
        kbar_all = page_key_means(kf, P)
        _check_sums(w, run)
        for c in (1, N // 2, N - 1):
            n_past = c * w.pages_per_chunk
            cnt = run.sel_n[c].cpu().numpy()
            lg = run.sel_l[c].cpu().numpy()
            sel = [[lg[b, g, :cnt[b, g]].tolist() for g in range(Hkv)] for b in range(len(cnt))]
            for b in range(len(cnt)):
                ref = page_scores(group_query_means(cpu[c]["q"][b * P:(b + 1) * P], Hkv),
                                  kbar_all[:n_past])
                want = select_pages(ref, n_past, w.top_k, w.n_recent)
                for g in range(Hkv):
                    kth = kth_score(ref[g], n_past, w.top_k, w.n_recent)
                    for p in set(sel[b][g]) ^ set(want[g]):
                        assert kth is not None and abs(ref[g, p] - kth) <= TIE, (c, b, g, p)
            _check_rows(w, run, cpu, kf, vf, c, sel, block_rows=P)
        _check_single_chunk_grads_qpage(w, run, cpu, kf, vf, N - 1)
    finally:
        _close(run)


def _check_single_chunk_grads_qpage(w, run, cpu, kf, vf, c):
    """As _check_single_chunk_grads, for per-query-page lists: each block of
    page_size rows has its own key set, so the oracle's contribution to a
    sampled key is summed over the blocks whose set holds it."""
    C, Hq, Hkv, P = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.page_size
    G = Hq // Hkv
    _, grad, _ = pk.pool_views(run.pool)
    grad.zero_()
    x = run.inputs[c]
    for step in (pk.BWD_PREPROCESS, pk.BWD_DKDV):
        pk.chunk_attn_bwd(run.pool, x["q"], run.o[c], run.lse[c], x["do"], run.dq[c],
                          run.deltas[c], run.u_pages[c], run.u_cnt[c], run.cur[c],
                          w.softmax_scale, step=step, past_masks=run.masks[c])
    torch.cuda.synchronize()
    assert pk.get_device_status(run.pool) == 0
    cnt = run.sel_n[c].cpu().numpy()
    lg = run.sel_l[c].cpu().numpy()
    nb = C // P
    sel = [[lg[b, g, :cnt[b, g]].tolist() for g in range(Hkv)] for b in range(nb)]
    q = cpu[c]["q"].double().numpy()
    do = cpu[c]["do"].double().numpy()
    rng = np.random.default_rng(9700 + c)
    ppc = w.pages_per_chunk
    for g in range(Hkv):
        listed = sorted(set().union(*[set(sel[b][g]) for b in range(nb)]))
        rest = [p for p in listed if p not in (listed[0], listed[-1])]
        pick = sorted({listed[0], listed[-1], c * ppc, (c + 1) * ppc - 1} |
                      set(rng.choice(rest, size=PAGES - 4, replace=False).tolist()))
        ptok = {p: np.arange(p * P, (p + 1) * P) for p in pick}
        dk_ref = {p: np.zeros((P, w.head_dim)) for p in pick}
        dv_ref = {p: np.zeros((P, w.head_dim)) for p in pick}
        for b in range(nb):
            tok = _tokens(w, c, sel[b][g])
            pos_in = {int(t): i for i, t in enumerate(tok)}
            seen = [p for p in pick if int(ptok[p][0]) in pos_in]
            if not seen:
                continue
            key_idx = np.array([pos_in[int(t)] for p in seen for t in ptok[p]])
            rows = np.arange(b * P, (b + 1) * P)
            dk_b, dv_b = chunk_keys_backward(
                q[rows, g * G:(g + 1) * G], do[rows, g * G:(g + 1) * G], c * C + rows,
                kf[tok, g].astype(np.float64), vf[tok, g].astype(np.float64), tok, key_idx,
                w.softmax_scale)
            for i, p in enumerate(seen):
                dk_ref[p] += dk_b[i * P:(i + 1) * P]
                dv_ref[p] += dv_b[i * P:(i + 1) * P]
        phys = torch.tensor([run.page_table[p] for p in pick], dtype=torch.long,
                            device=grad.device)
        blk = to64(grad[phys, g])                      # [pages][2][P][d]
        dk_gpu = blk[:, 0].reshape(-1, w.head_dim)
        dv_gpu = blk[:, 1].reshape(-1, w.head_dim)
        want_k = np.concatenate([dk_ref[p] for p in pick])
        want_v = np.concatenate([dv_ref[p] for p in pick])
        assert rel_l2(dk_gpu, want_k) <= BWD_REL, (g, rel_l2(dk_gpu, want_k))
        assert rel_l2(dv_gpu, want_v) <= BWD_REL, (g, rel_l2(dv_gpu, want_v))


class _TokenKeys:
    """K or V of a long sequence kept as one bf16 CPU tensor [L][Hkv][d];
    indexing [tokens, g] gives those rows of KV head g as fp32 numpy."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, idx):
        tok, g = idx
        return self.t[torch.as_tensor(tok, dtype=torch.long), g].float().numpy()


def test_fullsize_qwen1m_offload_matches_device_resident():
    """1M tokens (16,384 pages, 256 chunks): the offloaded schedule (pinned
    host pools, staging prefetch, gradient write-back) against the same
    workload with every page in HBM, and the last chunk against the oracle.

    Every chunk's K and V, and the last chunk's Q and dO, come from the seeded
    CPU generator (the other chunks' Q and dO are drawn on the device: they
    do not enter the last chunk's selection or outputs), so the last chunk's
    Top-K ids and 256 sampled rows of every head are checked against the
    oracle over all 16,320 past pages.  The host gradient pool must also
    hold the two softmax sums (sum over keys of dK_g = 0, of dV_g = sum of dO)."""
    from paged_kv_chunk_query_b200.offload import OffloadRun
    w = synth.WORKLOADS["qwen1m_topk_offload"]
    dev = _dev()
    N, C, Hq, Hkv, P, d = (w.num_chunks, w.chunk_len, w.num_q_heads, w.num_kv_heads,
                           w.page_size, w.head_dim)
    G = Hq // Hkv
    with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        kv_cpu = list(ex.map(lambda c: synth.chunk_inputs(w, c, which=("k", "v")), range(N)))
    last_cpu = synth.chunk_inputs(w, N - 1, which=("q", "do"))
    ins = []
    for c in range(N):
        x = synth.device_chunk_inputs(w, c, dev)
        x["k"], x["v"] = kv_cpu[c]["k"].to(dev), kv_cpu[c]["v"].to(dev)
        if c == N - 1:
            x["q"], x["do"] = last_cpu["q"].to(dev), last_cpu["do"].to(dev)
        ins.append(x)
    sample = (1, N // 2, N - 1)
    outs = {c: (torch.empty_like(ins[c]["q"]), torch.empty((Hq, C), dtype=torch.float32,
                                                           device=dev),
                torch.empty_like(ins[c]["q"])) for c in sample}
    scratch = (torch.empty_like(ins[0]["q"]), torch.empty((Hq, C), dtype=torch.float32, device=dev),
               torch.empty_like(ins[0]["q"]))
    off = OffloadRun(w, dev)
    try:
        off.run(lambda c: ins[c], lambda c: outs.get(c, scratch))
        off.sync()
        assert pk.get_device_status(off.stage) == 0 and pk.get_device_status(off.host) == 0
        sels = off.selections
        _, gh, _ = pk.pool_views(off.host)
        run = bench.Run(w, True, dev, inputs=ins)
        try:
            run.step()
            torch.cuda.synchronize()
            assert pk.get_device_status(run.pool) == 0
            for c in range(1, N):
                assert _selected(run, c) == sels[c], c
            for c in sample:
                assert torch.equal(outs[c][0], run.o[c]), c
                assert torch.equal(outs[c][1], run.lse[c]), c
                assert torch.equal(outs[c][2], run.dq[c]), c
            _, gd, _ = pk.pool_views(run.pool)
            err = ref = 0.0
            host_ids = torch.tensor(off.table, dtype=torch.long)
            dev_ids = run.page_table_dev.long()
            for a, b in zip(host_ids.split(512), dev_ids.split(512)):   # same logical pages
                h = gh[a].to(dev).double()
                dd = gd[b].double()
                err += float((h - dd).pow(2).sum())
                ref += float(dd.pow(2).sum())
            assert (err / ref) ** 0.5 <= 1e-3, (err / ref) ** 0.5
        finally:
            run.close()
        # the softmax sums on the host gradient pool the offloaded run built
        dk_sum = torch.zeros((Hkv, d), dtype=torch.float64, device=dev)
        dv_sum = torch.zeros_like(dk_sum)
        dk_sq = torch.zeros(Hkv, dtype=torch.float64, device=dev)
        for a in torch.tensor(off.table, dtype=torch.long).split(512):
            gg = gh[a].to(dev).double()
            dk_sum += gg[:, :, 0].sum(dim=(0, 2))
            dv_sum += gg[:, :, 1].sum(dim=(0, 2))
            dk_sq += gg[:, :, 0].pow(2).sum(dim=(0, 2, 3))
        do_sum = torch.zeros_like(dk_sum)
        for x in ins:
            do_sum += x["do"].double().view(-1, Hkv, G, d).sum(dim=(0, 2))
        for g in range(Hkv):
            assert float(dk_sum[g].norm()) <= 1e-2 * float(dk_sq[g].sqrt()), g
            assert float((dv_sum[g] - do_sum[g]).norm()) <= 1e-2 * float(do_sum[g].norm()), g
    finally:
        off.close()
    # the last chunk against the oracle: its selection over 16,320 past pages
    # and 256 sampled rows of every head on that selection
    c = N - 1
    kbar = np.concatenate([page_key_means(x["k"], P) for x in kv_cpu[:c]])
    n_past = c * w.pages_per_chunk
    ref = page_scores(group_query_means(last_cpu["q"], Hkv), kbar)
    want = select_pages(ref, n_past, w.top_k, w.n_recent)
    for g in range(Hkv):
        got = sels[c][g]
        assert len(got) == w.top_k + w.n_recent and got == sorted(got), g
        kth = kth_score(ref[g], n_past, w.top_k, w.n_recent)
        for pg in set(got) ^ set(want[g]):
            assert kth is not None and abs(ref[g, pg] - kth) <= TIE, (g, pg)
    kf = _TokenKeys(torch.cat([x["k"] for x in kv_cpu]))
    vf = _TokenKeys(torch.cat([x["v"] for x in kv_cpu]))
    cpu = {c: last_cpu}
    fake = type("R", (), {})()
    fake.o, fake.lse, fake.dq = ({c: outs[c][0]}, {c: outs[c][1]}, {c: outs[c][2]})
    _check_rows(w, fake, cpu, kf, vf, c, sels[c])
    del ins
    torch.cuda.empty_cache()
