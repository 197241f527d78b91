"""GPU parity: page representatives, Top-K page selection and page-sparse
attention vs the oracle.

Selection is compared bit for bit, except for pages whose fp64 oracle score
lies within 1e-5 of the K-th candidate score (fp32 vs fp64 rounding may order
those differently); the kept list must still be valid (right count, recent
pages present, ascending).  Sparse attention is then compared with the oracle
evaluated on the GPU's own selection.
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.recurrent import run_sequence
from oracle.sparse import (group_query_means, kth_score, page_key_means, page_scores,
                           select_pages)
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu

TIE = 1e-5


def _topk(run, q, n_past, K, R, scores=True):
    Hkv = run.w.num_kv_heads
    dev = run.dev
    ms = K + R
    out_l = torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev)
    out_p = torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(Hkv, dtype=torch.int32, device=dev)
    sc = torch.zeros((Hkv, max(n_past, 1)), dtype=torch.float32, device=dev)
    C, Hq, d = q.shape
    ws = torch.empty(pk.page_topk_workspace_size(C, Hq, Hkv, d, n_past), dtype=torch.uint8, device=dev)
    pt = torch.tensor(run.page_table[:n_past] or [0], dtype=torch.int32, device=dev)
    pk.page_topk(run.pool, q.to(dev).contiguous(), pt, n_past, K, R, out_l, out_p, cnt, ws,
                 out_scores=sc if scores else None)
    torch.cuda.synchronize()
    c = cnt.cpu().tolist()
    lists = [out_l[g, :c[g]].cpu().tolist() for g in range(Hkv)]
    phys = [out_p[g, :c[g]].cpu().tolist() for g in range(Hkv)]
    return lists, phys, sc[:, :n_past].double().cpu().numpy()


def _check_selection(gpu_lists, ref_scores, n_past, K, R):
    ref = select_pages(ref_scores, n_past, K, R)
    for g, (got, want) in enumerate(zip(gpu_lists, ref)):
        assert got == sorted(got) and len(set(got)) == len(got)
        assert len(got) == min(K, max(0, n_past - R)) + min(R, n_past)
        assert set(range(max(0, n_past - R), n_past)) <= set(got)
        kth = kth_score(ref_scores[g], n_past, K, R)
        for p in set(got) ^ set(want):  # disagreements only inside the tie band
            assert kth is not None and abs(ref_scores[g, p] - kth) <= TIE, (g, p)


def _topk_qsum(run, qsum, C, Hq, n_past, K, R, ws):
    """oomb_page_topk_qsum on a caller's workspace (counters zero at first use)."""
    Hkv = run.w.num_kv_heads
    dev = run.dev
    ms = K + R
    out_l = torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev)
    out_p = torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(Hkv, dtype=torch.int32, device=dev)
    sc = torch.zeros((Hkv, max(n_past, 1)), dtype=torch.float32, device=dev)
    pt = torch.tensor(run.page_table[:n_past] or [0], dtype=torch.int32, device=dev)
    pk.page_topk_qsum(run.pool, qsum, C, Hq, pt, n_past, K, R, out_l, out_p, cnt, ws,
                      out_scores=sc)
    torch.cuda.synchronize()
    c = cnt.cpu().tolist()
    lists = [out_l[g, :c[g]].cpu().tolist() for g in range(Hkv)]
    phys = [out_p[g, :c[g]].cpu().tolist() for g in range(Hkv)]
    return lists, phys, sc[:, :n_past].double().cpu().numpy()


def test_summaries_are_page_means():
    w = synth.Workload("sum", 8, 2, 128, 64, 256, 2, seed=21, page_direction=0.5)
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            r.append(**{k: v for k, v in synth.chunk_inputs(w, c).items() if k in ("k", "v")})
        torch.cuda.synchronize()
        _, _, summ = pk.pool_views(r.pool)
        got = summ[torch.tensor(r.page_table, device=r.dev)].double().cpu().numpy()
    k = synth.sequence_inputs(w)["k"]
    want = page_key_means(k, w.page_size)
    assert np.max(np.abs(got - want)) <= 1e-6 * max(1.0, np.max(np.abs(want)))


@pytest.mark.parametrize("K,R", [(3, 2), (1, 0), (0, 2), (50, 2), (5, 7)])
def test_topk_matches_oracle_small(K, R):
    w = synth.Workload("tk", 14, 2, 128, 64, 256, 5, seed=31, page_direction=0.5)
    inp = synth.sequence_inputs(w)
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            if c:
                n_past = c * w.pages_per_chunk
                lists, phys, sc = _topk(r, ch["q"], n_past, K, R)
                qbar = group_query_means(ch["q"], w.num_kv_heads)
                ref = page_scores(qbar, page_key_means(inp["k"][: c * w.chunk_len], w.page_size))
                assert np.max(np.abs(sc - ref)) <= 1e-6 + 1e-5 * np.max(np.abs(ref))
                _check_selection(lists, ref, n_past, K, R)
                for g in range(w.num_kv_heads):
                    assert phys[g] == [r.page_table[p] for p in lists[g]]
            r.append(ch["k"], ch["v"])
        assert r.status() == 0


def test_topk_many_candidates_and_exact_ties():
    """4096 past pages in one pool (radix select over many keys); groups of
    pages with identical keys make exact score ties at the K-th boundary."""
    Hq, Hkv, d, P, n_pages = 8, 2, 128, 16, 4096
    w = synth.Workload("big", Hq, Hkv, d, P, P * n_pages, 1, seed=41, page_direction=0.5,
                       shuffle_pages=True)
    gen = torch.Generator().manual_seed(5)
    k = torch.randn(n_pages * P, Hkv, d, generator=gen)
    k += 0.5 * torch.randn(n_pages, 1, Hkv, d, generator=gen).expand(n_pages, P, Hkv, d).reshape(-1, Hkv, d)
    for dup in range(1, 40):                    # page 100 + dup is a copy of page 100
        k[(100 + dup) * P:(101 + dup) * P] = k[100 * P:101 * P]
    k = k.to(torch.bfloat16)
    v = torch.randn(n_pages * P, Hkv, d, generator=gen).to(torch.bfloat16)
    q = torch.randn(256, Hq, d, generator=gen).to(torch.bfloat16)
    kbar = page_key_means(k, P)
    qbar = group_query_means(q, Hkv)
    ref = page_scores(qbar, kbar)
    # make the tied block straddle the K-th boundary of group 0
    order = np.argsort(-ref[0, :n_pages - 2], kind="stable")
    K = min(int(np.where(order == 100)[0][0]) + 20, 4090)
    with PagedRun(w, num_pages=n_pages) as r:
        r.append(k, v)
        lists, phys, sc = _topk(r, q, n_pages, K, 2)
        assert r.status() == 0
    _check_selection(lists, ref, n_pages, K, 2)
    # exact ties resolve to the lower logical id
    tied = set(range(100, 140))
    kept_tied = sorted(tied & set(lists[0]))
    if 0 < len(kept_tied) < len(tied):
        assert kept_tied == sorted(tied)[:len(kept_tied)]


def test_sparse_chunks_match_oracle_on_gpu_selection():
    w = synth.Workload("sp", 14, 2, 128, 64, 256, 6, seed=51, shuffle_pages=True,
                       page_direction=0.5, top_k=3, n_recent=2)
    inp = synth.sequence_inputs(w)
    sels, outs = [], []
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            n_past = c * w.pages_per_chunk
            if c:
                lists, _, sc = _topk(r, ch["q"], n_past, w.top_k, w.n_recent)
                ref = page_scores(group_query_means(ch["q"], w.num_kv_heads),
                                  page_key_means(inp["k"][: c * w.chunk_len], w.page_size))
                _check_selection(lists, ref, n_past, w.top_k, w.n_recent)
            else:
                lists = [[] for _ in range(w.num_kv_heads)]
            sels.append(lists)
            outs.append(r.chunk(c, ch, selected=lists if c else None))
        torch.cuda.synchronize()
        assert r.status() == 0
        dk, dv = r.grads_by_token(w.context)
    ref = run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                       w.softmax_scale, selections=sels)
    C = w.chunk_len
    o = np.concatenate([to64(x["o"]) for x in outs])
    lse = np.concatenate([to64(x["lse"]) for x in outs], axis=1)
    dq = np.concatenate([to64(x["dq"]) for x in outs])
    assert rel_l2(o, ref["o"]) <= 5e-3 and np.max(np.abs(o - ref["o"])) <= 1e-2
    assert rel_l2(lse, ref["lse"]) <= 5e-3
    assert rel_l2(dq, ref["dq"]) <= 1e-2
    assert rel_l2(dk, ref["dk"]) <= 1e-2
    assert rel_l2(dv, ref["dv"]) <= 1e-2
    # unselected pages of a chunk got nothing from it: compare per-token grad mass
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


@pytest.mark.parametrize("K,R,d", [(3, 2, 128), (0, 2, 128), (50, 2, 128), (1, 0, 128),
                                   (3, 2, 64), (20, 2, 64)])
def test_topk_from_qsum_matches_oracle(K, R, d):
    """Selection from per-group Q sums (one launch).  The sums are formed in
    fp32 by torch from the chunk's bf16 Q (another summation order than the
    library's own query mean), so scores match the oracle to fp32 rounding and
    the kept set matches outside the tie band; the same holds against the
    two-launch path.  One workspace serves every chunk (growing n_past), so
    each call must leave its counters at zero for the next."""
    w = synth.Workload("tq", 14, 2, d, 64, 256, 6, seed=33, page_direction=0.5)
    Hq, Hkv, d, C = w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len
    G = Hq // Hkv
    inp = synth.sequence_inputs(w)
    with PagedRun(w) as r:
        max_past = (w.num_chunks - 1) * w.pages_per_chunk
        ws = torch.zeros(pk.page_topk_qsum_workspace_size(Hkv, max_past), dtype=torch.uint8,
                         device=r.dev)
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            if c:
                n_past = c * w.pages_per_chunk
                qsum = ch["q"].to(r.dev).float().reshape(C, Hkv, G, d).sum(dim=(0, 2))
                lists, phys, sc = _topk_qsum(r, qsum.contiguous(), C, Hq, n_past, K, R, ws)
                ref = page_scores(group_query_means(ch["q"], Hkv),
                                  page_key_means(inp["k"][: c * C], w.page_size))
                assert np.max(np.abs(sc - ref)) <= 1e-6 + 1e-5 * np.max(np.abs(ref))
                _check_selection(lists, ref, n_past, K, R)
                for g in range(Hkv):
                    assert phys[g] == [r.page_table[p] for p in lists[g]]
                lists2, _, _ = _topk(r, ch["q"], n_past, K, R, scores=False)
                for g in range(Hkv):
                    kth = kth_score(ref[g], n_past, K, R)
                    for p in set(lists[g]) ^ set(lists2[g]):
                        assert kth is not None and abs(ref[g, p] - kth) <= TIE, (c, g, p)
            r.append(ch["k"], ch["v"])
        assert r.status() == 0
        assert int(ws[:4 * Hkv].view(torch.int32).abs().sum()) == 0  # counters back at zero


def test_topk_from_qsum_many_candidates():
    """4,096 past pages (radix select from registers at its largest) and then
    4,100 (the select that re-reads the keys), from Q sums."""
    Hq, Hkv, d, P = 8, 2, 128, 16
    for n_pages in (4096, 4100):
        w = synth.Workload("bigq", Hq, Hkv, d, P, P * n_pages, 1, seed=43, page_direction=0.5,
                           shuffle_pages=True)
        gen = torch.Generator().manual_seed(n_pages)
        k = torch.randn(n_pages * P, Hkv, d, generator=gen)
        k += 0.5 * torch.randn(n_pages, 1, Hkv, d, generator=gen).expand(
            n_pages, P, Hkv, d).reshape(-1, Hkv, d)
        k = k.to(torch.bfloat16)
        v = torch.randn(n_pages * P, Hkv, d, generator=gen).to(torch.bfloat16)
        q = torch.randn(192, Hq, d, generator=gen).to(torch.bfloat16)
        ref = page_scores(group_query_means(q, Hkv), page_key_means(k, P))
        with PagedRun(w, num_pages=n_pages) as r:
            r.append(k, v)
            ws = torch.zeros(pk.page_topk_qsum_workspace_size(Hkv, n_pages), dtype=torch.uint8,
                             device=r.dev)
            qsum = q.to(r.dev).float().reshape(192, Hkv, Hq // Hkv, d).sum(dim=(0, 2))
            for K in (64, 1000):
                lists, _, _ = _topk_qsum(r, qsum.contiguous(), 192, Hq, n_pages, K, 2, ws)
                _check_selection(lists, ref, n_pages, K, 2)
            assert r.status() == 0


def test_topk_from_projection_qsum():
    """Q and its per-group sums from the projection GEMM's epilogue feed the
    one-launch selection; the oracle selects from its own bf16-rounded
    projection of the same X and W.  X and W are small integers (W scaled by
    2^-5), so every fp32 partial sum of the GEMM is exact (|sum| <= 64 in
    steps of 2^-5) and both sides round the same exact value: the GPU's Q
    equals the oracle's bit for bit, and the per-group sums (|sum| <= 2^17 in
    steps of 2^-5) are exact in any order.  What remains is the fp32 scoring,
    inside the tie band."""
    from oracle.projection import qkv_projection
    C, hidden, Hq, Hkv, d, P, n_past = 256, 512, 14, 2, 128, 64, 48
    gen = torch.Generator().manual_seed(77)
    x = torch.randint(-2, 3, (C, hidden), generator=gen).to(torch.bfloat16)
    wt = (torch.randint(-2, 3, ((Hq + 2 * Hkv) * d, hidden), generator=gen) / 32.0).to(
        torch.bfloat16)
    k = (torch.randn(n_past * P, Hkv, d, generator=gen)
         + 0.5 * torch.randn(n_past, 1, Hkv, d, generator=gen).expand(
             n_past, P, Hkv, d).reshape(-1, Hkv, d)).to(torch.bfloat16)
    v = torch.randn(n_past * P, Hkv, d, generator=gen).to(torch.bfloat16)
    q_ref = qkv_projection(x.float().numpy(), wt.float().numpy(), Hq, Hkv, d)[0]
    q_ref = torch.tensor(q_ref).to(torch.bfloat16).double().numpy()
    ref = page_scores(group_query_means(q_ref, Hkv), page_key_means(k, P))
    w = synth.Workload("pq", Hq, Hkv, d, P, n_past * P, 1, seed=78, shuffle_pages=True)
    with PagedRun(w, num_pages=n_past) as r:
        r.append(k, v)
        q = torch.zeros((C, Hq, d), dtype=torch.bfloat16, device=r.dev)
        qsum = torch.zeros((Hkv, d), dtype=torch.float32, device=r.dev)
        pk.qkv_project(r.pool, x.to(r.dev), wt.to(r.dev), Hq, pk.PROJ_Q, q=q, qsum=qsum)
        torch.cuda.synchronize()
        assert np.array_equal(q.double().cpu().numpy(), q_ref)
        ws = torch.zeros(pk.page_topk_qsum_workspace_size(Hkv, n_past), dtype=torch.uint8,
                         device=r.dev)
        for K, R in ((8, 2), (20, 0)):
            lists, phys, sc = _topk_qsum(r, qsum, C, Hq, n_past, K, R, ws)
            assert np.max(np.abs(sc - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref)))
            _check_selection(lists, ref, n_past, K, R)
            for g in range(Hkv):
                assert phys[g] == [r.page_table[p] for p in lists[g]]
        assert r.status() == 0


def test_topk_replayed_from_cuda_graph_equals_eager():
    """The selections are dependent launches (the scores kernel after the
    query mean, the batch's kernels after one another): captured in a CUDA
    graph and replayed, the per-chunk, batched and Q-sum forms give the same
    lists, counts and scores as eager calls, bit for bit."""
    w = synth.Workload("tg", 14, 2, 128, 64, 256, 6, seed=35, page_direction=0.5,
                       shuffle_pages=True)
    Hq, Hkv, d, C, ppc = w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len, w.pages_per_chunk
    K, R = 5, 2
    ms = K + R
    dev = torch.device("cuda", 0)
    with PagedRun(w) as r:
        qs = []
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            r.append(ch["k"], ch["v"])
            qs.append(ch["q"].to(dev).contiguous())
        n_past = (w.num_chunks - 1) * ppc
        pt = torch.tensor(r.page_table[:n_past], dtype=torch.int32, device=dev)
        q_all = torch.cat(qs[1:]).contiguous()
        nb = w.num_chunks - 1
        rs = torch.arange(0, (nb + 1) * C, C, dtype=torch.int32, device=dev)
        npast_b = torch.tensor([c * ppc for c in range(1, w.num_chunks)], dtype=torch.int32,
                               device=dev)
        qsum = qs[-1].float().reshape(C, Hkv, Hq // Hkv, d).sum(dim=(0, 2)).contiguous()

        def buffers():
            return {"l": torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev),
                    "p": torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev),
                    "n": torch.zeros(Hkv, dtype=torch.int32, device=dev),
                    "s": torch.zeros((Hkv, n_past), dtype=torch.float32, device=dev),
                    "bl": torch.full((nb, Hkv, ms), -1, dtype=torch.int32, device=dev),
                    "bp": torch.full((nb, Hkv, ms), -1, dtype=torch.int32, device=dev),
                    "bn": torch.zeros((nb, Hkv), dtype=torch.int32, device=dev),
                    "ql": torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev),
                    "qn": torch.zeros(Hkv, dtype=torch.int32, device=dev)}

        ws = torch.empty(pk.page_topk_workspace_size(C, Hq, Hkv, d, n_past), dtype=torch.uint8,
                         device=dev)
        wsb = torch.empty(pk.page_topk_batched_workspace_size(nb, Hkv, d, n_past),
                          dtype=torch.uint8, device=dev)
        wsq = torch.zeros(pk.page_topk_qsum_workspace_size(Hkv, n_past), dtype=torch.uint8,
                          device=dev)

        def run(b, st):
            pk.page_topk(r.pool, qs[-1], pt, n_past, K, R, b["l"], b["p"], b["n"], ws,
                         out_scores=b["s"], stream=st)
            pk.page_topk_batched(r.pool, q_all, rs, C, npast_b, n_past, pt, K, R, b["bl"],
                                 b["bp"], b["bn"], wsb, stream=st)
            pk.page_topk_qsum(r.pool, qsum, C, Hq, pt, n_past, K, R, b["ql"], None, b["qn"],
                              wsq, stream=st)

        eager = buffers()
        for v in eager.values():
            v.fill_(-7)               # the sentinel the graphed buffers get too
        run(eager, torch.cuda.current_stream())
        torch.cuda.synchronize()
        graphed = buffers()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run(graphed, s)           # warm-up outside the capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for v in graphed.values():
            v.fill_(-7)               # whatever the replays do not write stays -7, as in eager
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run(graphed, torch.cuda.current_stream())
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        assert r.status() == 0
        for key in eager:
            assert torch.equal(eager[key], graphed[key]), key
        del g
