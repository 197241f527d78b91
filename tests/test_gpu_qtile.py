"""GPU parity: one past-page list per 128-row query tile (the coarser form
of per-query-page selection: two 64-token query pages share a list) vs the
oracle's per-row-block attention.

Tolerances as for the chunk-wide lists: forward O/LSE relative L2 <= 5e-3 and
max abs <= 1e-2, dQ/dK/dV relative L2 <= 1e-2.  Lists that are the same for
every query tile must reproduce the chunk-wide result: forward and dQ bit
for bit, the gradient pool up to fp32 summation order.  Selections made on
the GPU by the batched Top-K (one problem per query tile) must match the
oracle's per-block Top-K outside the 1e-5 tie band.
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.recurrent import run_sequence_blocks
from oracle.sparse import group_query_means, kth_score, page_key_means, page_scores, select_pages
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS, BWD_REL = 5e-3, 1e-2, 1e-2
DEV = torch.device("cuda", 0)
TILE = 128


def _qtile_lists(r, sel_c):
    """Device [n_qtiles][Hkv][max] physical ids and [n_qtiles][Hkv] counts."""
    nq, Hkv = len(sel_c), r.w.num_kv_heads
    m = max(1, max(len(s) for blk in sel_c for s in blk))
    ids = torch.zeros((nq, Hkv, m), dtype=torch.int32)
    cnt = torch.zeros((nq, Hkv), dtype=torch.int32)
    for t in range(nq):
        for g in range(Hkv):
            s = sel_c[t][g]
            if s:
                ids[t, g, :len(s)] = torch.tensor([r.page_table[p] for p in s], dtype=torch.int32)
            cnt[t, g] = len(s)
    return ids.to(DEV), cnt.to(DEV)


def _run(w, sels, backward=True):
    outs = []
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            inp = synth.chunk_inputs(w, c)
            cur = r.append(inp["k"], inp["v"])
            past, cnt = _qtile_lists(r, sels[c]) if c else (None, None)
            q = inp["q"].to(DEV).contiguous()
            o = torch.empty_like(q)
            lse = torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32, device=DEV)
            pk.chunk_attn_fwd(r.pool, q, o, lse, past, cnt, cur, w.softmax_scale, fwd_ws=r.fwd_ws)
            out = {"o": o, "lse": lse}
            if backward:
                dq = torch.empty_like(q)
                pk.chunk_attn_bwd(r.pool, q, o, lse, inp["do"].to(DEV).contiguous(), dq,
                                  torch.empty_like(lse), past, cnt, cur, w.softmax_scale)
                out["dq"] = dq
            outs.append(out)
        torch.cuda.synchronize()
        assert r.status() == 0
        grads = r.grads_by_token(w.context) if backward else (None, None)
    return outs, grads


def _random_block_selections(w, seed):
    rng = np.random.default_rng(seed)
    nq = (w.chunk_len + TILE - 1) // TILE
    sels = []
    for c in range(w.num_chunks):
        n_past = c * w.pages_per_chunk
        sels.append([[sorted(rng.choice(n_past, size=int(rng.integers(0, n_past + 1)),
                                        replace=False).tolist()) if n_past else []
                      for _ in range(w.num_kv_heads)] for _ in range(nq)])
    return sels


def _check(w, ref, outs, grads):
    C = w.chunk_len
    for c, out in enumerate(outs):
        o, lse = to64(out["o"]), to64(out["lse"])
        o_ref, lse_ref = ref["o"][c * C:(c + 1) * C], ref["lse"][:, c * C:(c + 1) * C]
        assert rel_l2(o, o_ref) <= FWD_REL and np.max(np.abs(o - o_ref)) <= FWD_ABS, c
        assert rel_l2(lse, lse_ref) <= FWD_REL and np.max(np.abs(lse - lse_ref)) <= FWD_ABS, c
    dq = np.concatenate([to64(o["dq"]) for o in outs], axis=0)
    dk, dv = grads
    assert rel_l2(dq, ref["dq"]) <= BWD_REL, rel_l2(dq, ref["dq"])
    assert rel_l2(dk, ref["dk"]) <= BWD_REL, rel_l2(dk, ref["dk"])
    assert rel_l2(dv, ref["dv"]) <= BWD_REL, rel_l2(dv, ref["dv"])


@pytest.mark.parametrize("w", [
    # 2.5 query tiles per chunk (ragged last tile), GQA 7:1, shuffled pages
    synth.Workload("qt7", 14, 2, 128, 64, 320, 4, seed=61, shuffle_pages=True),
    synth.Workload("qt2", 4, 2, 64, 32, 256, 4, seed=62),
], ids=["g7_d128_p64_ragged", "g2_d64_p32"])
def test_per_qtile_lists_match_oracle(w):
    inp = synth.sequence_inputs(w)
    sels = _random_block_selections(w, 63)
    ref = run_sequence_blocks(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                              w.softmax_scale, TILE, selections=sels)
    outs, grads = _run(w, sels)
    _check(w, ref, outs, grads)


def test_identical_qtile_lists_equal_chunk_lists():
    w = synth.Workload("qteq", 8, 2, 128, 64, 384, 3, seed=64, shuffle_pages=True)
    nq = w.chunk_len // TILE
    chunk_sels = [s[0] for s in _random_block_selections(w, 65)]
    outs, (dk, dv) = _run(w, [[s] * nq for s in chunk_sels])
    with PagedRun(w) as r:
        ref = [r.chunk(c, synth.chunk_inputs(w, c), selected=chunk_sels[c] if c else None)
               for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        dk_r, dv_r = r.grads_by_token(w.context)
    for a, b in zip(outs, ref):
        assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
        assert torch.equal(a["dq"], b["dq"])
    assert rel_l2(dk, dk_r) <= 1e-6 and rel_l2(dv, dv_r) <= 1e-6


def test_per_qtile_topk_then_attention():
    """Batched Top-K with one problem per query tile feeds the per-tile lists."""
    w = synth.Workload("qtk", 14, 2, 128, 64, 384, 4, seed=66, shuffle_pages=True,
                       page_direction=0.5, top_k=3, n_recent=2)
    K, R = w.top_k, w.n_recent
    Hkv, C, P = w.num_kv_heads, w.chunk_len, w.page_size
    nq = C // TILE
    inp = synth.sequence_inputs(w)
    sels, outs = [], []
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            n_past = c * w.pages_per_chunk
            q = ch["q"].to(DEV).contiguous()
            if n_past:
                out_l = torch.full((nq, Hkv, K + R), -1, dtype=torch.int32, device=DEV)
                out_p = torch.full_like(out_l, 0)
                cnt = torch.zeros((nq, Hkv), dtype=torch.int32, device=DEV)
                sc = torch.zeros((nq, Hkv, n_past), dtype=torch.float32, device=DEV)
                ws = torch.empty(pk.page_topk_batched_workspace_size(nq, Hkv, w.head_dim, n_past),
                                 dtype=torch.uint8, device=DEV)
                rs = torch.tensor([t * TILE for t in range(nq + 1)], dtype=torch.int32, device=DEV)
                npast = torch.full((nq,), n_past, dtype=torch.int32, device=DEV)
                pt = torch.tensor(r.page_table[:n_past], dtype=torch.int32, device=DEV)
                pk.page_topk_batched(r.pool, q, rs, TILE, npast, n_past, pt, K, R, out_l, out_p,
                                     cnt, ws, out_scores=sc)
                torch.cuda.synchronize()
                n = cnt.cpu().numpy()
                sel_c = [[out_l[t, g, :n[t, g]].cpu().tolist() for g in range(Hkv)]
                         for t in range(nq)]
                kbar = page_key_means(inp["k"][:c * C], P)
                for t in range(nq):
                    ref_s = page_scores(group_query_means(ch["q"][t * TILE:(t + 1) * TILE], Hkv),
                                        kbar)
                    want = select_pages(ref_s, n_past, K, R)
                    for g in range(Hkv):
                        kth = kth_score(ref_s[g], n_past, K, R)
                        for pg in set(sel_c[t][g]) ^ set(want[g]):
                            assert kth is not None and abs(ref_s[g, pg] - kth) <= 1e-5
                past, counts = out_p, cnt
            else:
                sel_c = [[[] for _ in range(Hkv)] for _ in range(nq)]
                past, counts = None, None
            sels.append(sel_c)
            cur = r.append(ch["k"], ch["v"])
            o = torch.empty_like(q)
            lse = torch.empty((w.num_q_heads, C), dtype=torch.float32, device=DEV)
            pk.chunk_attn_fwd(r.pool, q, o, lse, past, counts, cur, w.softmax_scale,
                              fwd_ws=r.fwd_ws)
            dq = torch.empty_like(q)
            pk.chunk_attn_bwd(r.pool, q, o, lse, ch["do"].to(DEV).contiguous(), dq,
                              torch.empty_like(lse), past, counts, cur, w.softmax_scale)
            outs.append({"o": o, "lse": lse, "dq": dq})
        torch.cuda.synchronize()
        assert r.status() == 0
        grads = r.grads_by_token(w.context)
    ref = run_sequence_blocks(inp["q"], inp["k"], inp["v"], inp["do"], C, P, w.softmax_scale,
                              TILE, selections=sels)
    _check(w, ref, outs, grads)
