"""GPU tests of the device-list block moves (block copy, gradient
scatter-add, prefetch lists) and of the batched Top-K.

Block copies are byte moves: bit-exact.  A gradient addition into pinned
host pages is one fp32 add per element: bit-exact against torch's fp32 add.
Into a device pool the adds are atomics (a destination may repeat): with
integer-valued inputs every order of fp32 additions is exact, so that too is
compared bit for bit.  The batched Top-K must equal one oomb_page_topk call
per problem bit for bit, and one selection per query page must match the
oracle's selection for those rows (up to the 1e-5 tie band).
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.sparse import group_query_means, kth_score, page_key_means, page_scores, select_pages
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
TIE = 1e-5


def _i32(x):
    return torch.tensor(x, dtype=torch.int32, device=DEV)


def _fill_pool(pool, seed):
    kv, _, summ = pk.pool_views(pool)
    gen = torch.Generator().manual_seed(seed)
    src = torch.randn(kv.shape, generator=gen).to(torch.bfloat16)
    s = torch.randn(summ.shape, generator=gen)
    if kv.is_cuda:
        kv.copy_(src.to(DEV))
    else:
        kv.copy_(src)
    summ.copy_(s.to(DEV))
    torch.cuda.synchronize()


@pytest.mark.parametrize("P,d", [(64, 128), (16, 64)])
def test_block_copy_device_gather_bit_exact(P, d):
    Hkv = 2
    a = pk.pool_create(40, P, Hkv, d, pk.LOC_DEVICE, False, 0, 0)
    b = pk.pool_create(24, P, Hkv, d, pk.LOC_DEVICE, False, 0, 0)
    try:
        _fill_pool(a, 1)
        _fill_pool(b, 2)
        kv_b0 = pk.pool_views(b)[0].clone()
        s_b0 = pk.pool_views(b)[2].clone()
        rng = np.random.default_rng(3)
        src = rng.permutation(40 * Hkv)[:30].tolist()
        dst = rng.permutation(24 * Hkv)[:30].tolist()
        src[5] = -1                       # padding entries are skipped
        dst[9] = -1
        pk.block_copy(a, b, _i32(src), _i32(dst))
        torch.cuda.synchronize()
        assert pk.get_device_status(b) == 0
        kv_a, _, s_a = pk.pool_views(a)
        kv_b, _, s_b = pk.pool_views(b)
        want_kv = kv_b0.clone().view(-1, 2, P, d)
        want_s = s_b0.clone().view(-1, d)
        for s_, d_ in zip(src, dst):
            if s_ >= 0 and d_ >= 0:
                want_kv[d_] = kv_a.view(-1, 2, P, d)[s_]
                want_s[d_] = s_a.view(-1, d)[s_]
        assert torch.equal(kv_b.view(-1, 2, P, d), want_kv)
        assert torch.equal(s_b.view(-1, d), want_s)
        # an id beyond the pool: skipped, flagged; the other entries still move
        pk.block_copy(a, b, _i32([0, 1]), _i32([24 * Hkv, 3]))
        torch.cuda.synchronize()
        assert pk.get_device_status(b) & 1
        assert torch.equal(pk.pool_views(b)[0].view(-1, 2, P, d)[3], kv_a.view(-1, 2, P, d)[1])
        with pytest.raises(ValueError):          # list lengths differ: refused before the call
            pk.block_copy(a, b, _i32([0, 1]), _i32([0]))
    finally:
        pk.pool_destroy(a)
        pk.pool_destroy(b)


def test_block_copy_over_the_host_link_round_trip():
    P, Hkv, d = 64, 4, 128
    a = pk.pool_create(16, P, Hkv, d, pk.LOC_DEVICE, False, 0, 0)
    h = pk.pool_create(32, P, Hkv, d, pk.LOC_PINNED_HOST, False, 0, 0)
    c = pk.pool_create(16, P, Hkv, d, pk.LOC_DEVICE, False, 0, 0)
    try:
        _fill_pool(a, 4)
        rng = np.random.default_rng(5)
        src = rng.permutation(16 * Hkv)[:48]
        mid = rng.permutation(32 * Hkv)[:48]
        back = rng.permutation(16 * Hkv)[:48]
        pk.block_copy(a, h, _i32(src), _i32(mid))          # device -> pinned host
        pk.block_copy(h, c, _i32(mid), _i32(back))         # pinned host -> device
        torch.cuda.synchronize()
        assert pk.get_device_status(h) == 0 and pk.get_device_status(c) == 0
        kv_a, _, s_a = pk.pool_views(a)
        kv_h, _, s_h = pk.pool_views(h)
        kv_c, _, s_c = pk.pool_views(c)
        A = kv_a.view(-1, 2, P, d).cpu()
        for s_, m_, b_ in zip(src, mid, back):
            assert torch.equal(kv_h.view(-1, 2, P, d)[m_], A[s_])
            assert torch.equal(kv_c.view(-1, 2, P, d)[b_].cpu(), A[s_])
            assert torch.equal(s_c.view(-1, d)[b_], s_a.view(-1, d)[s_])
            assert torch.equal(s_h.view(-1, d)[m_], s_a.view(-1, d)[s_])
    finally:
        for p in (a, h, c):
            pk.pool_destroy(p)


def test_grad_block_add_into_pinned_host_bit_exact_and_zeroes():
    P, Hkv, d = 32, 2, 64
    a = pk.pool_create(6, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    h = pk.pool_create(10, P, Hkv, d, pk.LOC_PINNED_HOST, True, 0, 0)
    try:
        _, ga, _ = pk.pool_views(a)
        _, gh, _ = pk.pool_views(h)
        gen = torch.Generator().manual_seed(6)
        ga.copy_(torch.randn(ga.shape, generator=gen).to(DEV))
        gh.copy_(torch.randn(gh.shape, generator=gen))
        bh = gh.clone().view(-1, 2 * P * d)
        ba = ga.cpu().view(-1, 2 * P * d)
        src = [0, 1, 2, 3, 7, 9, 10, -1]
        dst = [19, 18, 4, 5, 6, 0, 11, 3]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            pk.grad_block_add(a, h, _i32(src), _i32(dst), zero_src=True, stream=stream)
        stream.synchronize()
        assert pk.get_device_status(h) == 0
        want = bh.clone()
        for s_, d_ in zip(src, dst):
            if s_ >= 0:
                want[d_] = bh[d_] + ba[s_]
        assert torch.equal(gh.view(-1, 2 * P * d), want)
        now = ga.cpu().view(-1, 2 * P * d)
        for blk in range(now.shape[0]):
            if blk in src:
                assert float(now[blk].abs().max()) == 0.0
            else:
                assert torch.equal(now[blk], ba[blk])
    finally:
        pk.pool_destroy(a)
        pk.pool_destroy(h)


def test_grad_block_add_device_atomics_with_repeated_destinations():
    P, Hkv, d = 64, 2, 128
    a = pk.pool_create(8, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    b = pk.pool_create(8, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    try:
        _, ga, _ = pk.pool_views(a)
        _, gb, _ = pk.pool_views(b)
        gen = torch.Generator().manual_seed(7)
        # small integers: every order of fp32 additions gives the exact sum
        ga.copy_(torch.randint(-50, 50, ga.shape, generator=gen).float().to(DEV))
        gb.copy_(torch.randint(-50, 50, gb.shape, generator=gen).float().to(DEV))
        A = ga.cpu().view(-1, 2 * P * d)
        B = gb.cpu().view(-1, 2 * P * d)
        src = list(range(16))
        dst = [3, 3, 3, 5, 0, 1, 2, 4, 6, 7, 8, 9, 10, 11, 12, 3]
        pk.grad_block_add(a, b, _i32(src), _i32(dst), zero_src=False)
        torch.cuda.synchronize()
        want = B.clone()
        for s_, d_ in zip(src, dst):
            want[d_] += A[s_]
        assert torch.equal(gb.cpu().view(-1, 2 * P * d), want)
        assert torch.equal(ga.cpu().view(-1, 2 * P * d), A)   # zero_src off
    finally:
        pk.pool_destroy(a)
        pk.pool_destroy(b)


def test_prefetch_lists_match_host_construction():
    P, Hkv, d = 16, 4, 64
    host = pk.pool_create(64, P, Hkv, d, pk.LOC_PINNED_HOST, False, 11, 0)
    stage = pk.pool_create(20, P, Hkv, d, pk.LOC_DEVICE, False, 0, 0)
    try:
        table = [pk.pool_alloc_page(host) for _ in range(50)]
        slots = [pk.pool_alloc_page(stage) for _ in range(9)]
        rng = np.random.default_rng(8)
        counts = [9, 0, 4, 7]
        sel = np.zeros((Hkv, 9), dtype=np.int32)
        for g, n in enumerate(counts):
            sel[g, :n] = np.sort(rng.permutation(50)[:n])
        src = torch.empty(9 * Hkv, dtype=torch.int32, device=DEV)
        dst = torch.empty_like(src)
        past = torch.empty((Hkv, 9), dtype=torch.int32, device=DEV)
        pk.prefetch_lists(host, stage, _i32(sel), _i32(counts), _i32(table), _i32(slots),
                          src, dst, past)
        torch.cuda.synchronize()
        assert pk.get_device_status(stage) == 0
        ws, wd, wp = [], [], np.zeros((Hkv, 9), dtype=np.int64)
        for i in range(9):
            for g in range(Hkv):
                if i < counts[g]:
                    ws.append(table[sel[g, i]] * Hkv + g)
                    wd.append(slots[i] * Hkv + g)
                    wp[g, i] = slots[i]
                else:
                    ws.append(-1)
                    wd.append(-1)
        assert src.cpu().tolist() == ws and dst.cpu().tolist() == wd
        assert past.cpu().numpy().tolist() == wp.tolist()
        # a count above max_sel is clamped and flagged
        pk.prefetch_lists(host, stage, _i32(sel), _i32([10, 0, 0, 0]), _i32(table), _i32(slots),
                          src, dst, past)
        torch.cuda.synchronize()
        assert pk.get_device_status(stage) & 4
    finally:
        pk.pool_destroy(host)
        pk.pool_destroy(stage)


def _batched(pool, q, row_start, n_past, max_rows, max_past, table, K, R, Hkv):
    B = len(n_past)
    ms = K + R
    out_l = torch.full((B, Hkv, ms), -1, dtype=torch.int32, device=DEV)
    out_p = torch.full_like(out_l, -1)
    cnt = torch.zeros((B, Hkv), dtype=torch.int32, device=DEV)
    sc = torch.zeros((B, Hkv, max(max_past, 1)), dtype=torch.float32, device=DEV)
    d = q.shape[2]
    ws = torch.empty(pk.page_topk_batched_workspace_size(B, Hkv, d, max_past), dtype=torch.uint8,
                     device=DEV)
    pk.page_topk_batched(pool, q, _i32(row_start), max_rows, _i32(n_past), max_past,
                         _i32(table), K, R, out_l, out_p, cnt, ws, out_scores=sc)
    torch.cuda.synchronize()
    return out_l.cpu(), out_p.cpu(), cnt.cpu(), sc.cpu()


@pytest.mark.parametrize("d", [128, 64])
def test_batched_topk_equals_per_chunk_calls(d):
    """All chunks' selections in one batch == one oomb_page_topk per chunk
    (the batch reduces its query means once per problem and selects in a
    kernel of its own; the bits must not change)."""
    w = synth.Workload("bt", 14, 2, d, 64, 512, 8, seed=71, page_direction=0.5,
                       shuffle_pages=True)
    K, R = 3, 2
    Hkv, ppc, C = w.num_kv_heads, w.pages_per_chunk, w.chunk_len
    with PagedRun(w) as r:
        qs = []
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            r.append(ch["k"], ch["v"])
            qs.append(ch["q"])
        q_all = torch.cat(qs).to(DEV).contiguous()
        n_past = [c * ppc for c in range(w.num_chunks)]
        row_start = [c * C for c in range(w.num_chunks + 1)]
        max_past = (w.num_chunks - 1) * ppc
        bl, bp, bc, bs = _batched(r.pool, q_all, row_start, n_past, C, max_past, r.page_table,
                                  K, R, Hkv)
        for c in range(1, w.num_chunks):
            out_l = torch.full((Hkv, K + R), -1, dtype=torch.int32, device=DEV)
            out_p = torch.full_like(out_l, -1)
            cnt = torch.zeros(Hkv, dtype=torch.int32, device=DEV)
            sc = torch.zeros((Hkv, n_past[c]), dtype=torch.float32, device=DEV)
            ws = torch.empty(pk.page_topk_workspace_size(C, w.num_q_heads, Hkv, w.head_dim,
                                                         n_past[c]), dtype=torch.uint8, device=DEV)
            pk.page_topk(r.pool, q_all[c * C:(c + 1) * C], _i32(r.page_table[:n_past[c]]),
                         n_past[c], K, R, out_l, out_p, cnt, ws, out_scores=sc)
            torch.cuda.synchronize()
            n = cnt.cpu()
            assert torch.equal(bc[c], n), c
            for g in range(Hkv):
                assert torch.equal(bl[c, g, :n[g]], out_l.cpu()[g, :n[g]]), (c, g)
                assert torch.equal(bp[c, g, :n[g]], out_p.cpu()[g, :n[g]]), (c, g)
            assert torch.equal(bs[c, :, :n_past[c]], sc.cpu()), c
        assert bc[0].tolist() == [0] * Hkv     # chunk 0: no past pages
        assert r.status() == 0


def test_per_query_page_topk_matches_oracle():
    """One selection per query page of the last chunk (64 rows each)."""
    w = synth.Workload("qp", 14, 2, 128, 64, 1024, 4, seed=81, page_direction=0.5)
    K, R = 4, 2
    Hkv, P, C = w.num_kv_heads, w.page_size, w.chunk_len
    inp = synth.sequence_inputs(w)
    last = w.num_chunks - 1
    n_past = last * w.pages_per_chunk
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            r.append(ch["k"], ch["v"])
        q = synth.chunk_inputs(w, last)["q"]
        nq = C // P
        bl, _, bc, bs = _batched(r.pool, q.to(DEV).contiguous(), [i * P for i in range(nq + 1)],
                                 [n_past] * nq, P, n_past, r.page_table, K, R, Hkv)
        assert r.status() == 0
    kbar = page_key_means(inp["k"][: last * C], P)
    for i in range(nq):
        ref = page_scores(group_query_means(q[i * P:(i + 1) * P], Hkv), kbar)
        got_s = bs[i, :, :n_past].double().numpy()
        assert np.max(np.abs(got_s - ref)) <= 1e-6 + 1e-5 * np.max(np.abs(ref))
        want = select_pages(ref, n_past, K, R)
        for g in range(Hkv):
            got = bl[i, g, :int(bc[i, g])].tolist()
            assert got == sorted(got) and len(got) == len(want[g])
            kth = kth_score(ref[g], n_past, K, R)
            for p in set(got) ^ set(want[g]):
                assert kth is not None and abs(ref[g, p] - kth) <= TIE, (i, g, p)
