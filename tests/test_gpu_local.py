"""GPU parity: recent-only (local window) page lists and attention over them.

The list builder must equal the oracle's lists mapped through the page table
bit for bit; attention over those lists must match the oracle evaluated on
the same key sets (forward O/LSE relative L2 <= 5e-3 and max abs <= 1e-2,
dQ/dK/dV relative L2 <= 1e-2); a window that covers the whole past must give
exactly the dense result (same kernels, same pages in the same order).
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.recurrent import run_sequence
from oracle.sparse import local_pages
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS, BWD_REL = 5e-3, 1e-2, 1e-2
DEV = torch.device("cuda", 0)


def _lists(r, n_past, window):
    Hkv = r.w.num_kv_heads
    pages = torch.full((Hkv, window), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((Hkv,), -1, dtype=torch.int32, device=DEV)
    pt = torch.tensor(r.page_table[:max(n_past, 1)] or [0], dtype=torch.int32, device=DEV)
    pk.local_pages(r.pool, pt, n_past, pages, cnt)
    return pages, cnt


@pytest.mark.parametrize("n_past,window", [(0, 3), (2, 3), (3, 3), (17, 3), (17, 1), (17, 40)])
def test_local_lists_match_oracle(n_past, window):
    w = synth.Workload("ll", 4, 3, 64, 16, 320, 1, seed=51, shuffle_pages=True)
    with PagedRun(w) as r:
        r.page_table = [pk.pool_alloc_page(r.pool) for _ in range(20)]
        pages, cnt = _lists(r, n_past, window)
        torch.cuda.synchronize()
        assert r.status() == 0
        want = local_pages(n_past, window, w.num_kv_heads)
        got_p, got_c = pages.cpu().numpy(), cnt.cpu().tolist()
        for g in range(w.num_kv_heads):
            n = len(want[g])
            assert got_c[g] == n
            assert got_p[g, :n].tolist() == [r.page_table[p] for p in want[g]]
            assert (got_p[g, n:] == 0).all()


def _run_local(w, window, backward=True):
    outs = []
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            inp = synth.chunk_inputs(w, c)
            n_past = c * w.pages_per_chunk
            cur = r.append(inp["k"], inp["v"])
            past, cnt = _lists(r, n_past, window) if n_past else (None, None)
            q = inp["q"].to(DEV).contiguous()
            o = torch.empty_like(q)
            lse = torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32, device=DEV)
            pk.chunk_attn_fwd(r.pool, q, o, lse, past, cnt, cur, w.softmax_scale, fwd_ws=r.fwd_ws)
            out = {"o": o, "lse": lse}
            if backward:
                do = inp["do"].to(DEV).contiguous()
                dq = torch.empty_like(q)
                pk.chunk_attn_bwd(r.pool, q, o, lse, do, dq, torch.empty_like(lse), past, cnt,
                                  cur, w.softmax_scale)
                out["dq"] = dq
            outs.append(out)
        torch.cuda.synchronize()
        assert r.status() == 0
        grads = r.grads_by_token(w.context) if backward else None
    return outs, grads


@pytest.mark.parametrize("window", [1, 3])
def test_local_attention_matches_oracle(window):
    w = synth.Workload("lw", 14, 2, 128, 64, 256, 5, seed=52, shuffle_pages=True)
    inp = synth.sequence_inputs(w)
    sels = [local_pages(c * w.pages_per_chunk, window, w.num_kv_heads)
            for c in range(w.num_chunks)]
    ref = run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                       w.softmax_scale, selections=sels)
    outs, (dk, dv) = _run_local(w, window)
    C = w.chunk_len
    for c, out in enumerate(outs):
        o, lse = to64(out["o"]), to64(out["lse"])
        o_ref, lse_ref = ref["o"][c * C:(c + 1) * C], ref["lse"][:, c * C:(c + 1) * C]
        assert rel_l2(o, o_ref) <= FWD_REL and np.max(np.abs(o - o_ref)) <= FWD_ABS, c
        assert rel_l2(lse, lse_ref) <= FWD_REL and np.max(np.abs(lse - lse_ref)) <= FWD_ABS, c
    dq = np.concatenate([to64(o["dq"]) for o in outs], axis=0)
    assert rel_l2(dq, ref["dq"]) <= BWD_REL
    assert rel_l2(dk, ref["dk"]) <= BWD_REL
    assert rel_l2(dv, ref["dv"]) <= BWD_REL


def test_window_covering_the_past_equals_dense_bit_for_bit():
    w = synth.Workload("lwd", 8, 2, 128, 32, 256, 3, seed=53, shuffle_pages=True)
    outs, (dk, dv) = _run_local(w, w.num_pages)
    with PagedRun(w) as r:
        dense = [r.chunk(c, synth.chunk_inputs(w, c)) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        dk_d, dv_d = r.grads_by_token(w.context)
    for a, b in zip(outs, dense):
        assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
        assert torch.equal(a["dq"], b["dq"])
    # the gradient pool is summed with atomics: equal up to fp32 summation order
    assert rel_l2(dk, dk_d) <= 1e-6 and rel_l2(dv, dv_d) <= 1e-6
