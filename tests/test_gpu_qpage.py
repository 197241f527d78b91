"""GPU parity: one past-page list per QUERY PAGE (page_size consecutive rows
of the chunk; [pt] §2C "Sparse Attention em Nível de Página": the key pages
most relevant to each query page) vs the oracle's per-row-block attention
with block_rows = page_size.

The attention kernels work on 128-row query tiles, so a tile with two (or
more) query pages gets the union of their lists plus a membership mask per
entry (oomb_qpage_lists); each row attends only to the entries of its own
query page.  Checked here:

* the union lists and masks against their construction on the host, bit for
  bit (page sizes 64, 32 and 16; a ragged last tile);
* attention on random per-query-page selections against
  ``oracle.recurrent.run_sequence_blocks(block_rows = page_size)``: forward
  O / LSE relative L2 <= 5e-3 and max abs <= 1e-2, dQ / dK / dV relative L2
  <= 1e-2 (the forward and backward tolerances used throughout);
* identical lists for every query page of a tile reproduce the per-tile lists
  (all mask bits set: no masking, so the same arithmetic): forward and dQ bit
  for bit, gradient pool up to fp32 summation order;
* the batched Top-K with one problem per query page, then these lists, end
  to end against the oracle (selections outside the 1e-5 tie band).
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


def _sel_tensors(r, sel_c, max_sel):
    """Per-query-page selections (logical, ascending) -> device logical,
    physical [n_qpages][Hkv][max_sel] and counts [n_qpages][Hkv]."""
    nb, Hkv = len(sel_c), r.w.num_kv_heads
    lg = torch.full((nb, Hkv, max_sel), -1, dtype=torch.int32)
    ph = torch.full((nb, Hkv, max_sel), -1, dtype=torch.int32)
    cnt = torch.zeros((nb, Hkv), dtype=torch.int32)
    for b in range(nb):
        for g in range(Hkv):
            s = sel_c[b][g]
            if s:
                lg[b, g, :len(s)] = torch.tensor(s, dtype=torch.int32)
                ph[b, g, :len(s)] = torch.tensor([r.page_table[p] for p in s], dtype=torch.int32)
            cnt[b, g] = len(s)
    return lg.to(DEV), ph.to(DEV), cnt.to(DEV)


def _union_lists(r, sel_c, C):
    """oomb_qpage_lists on the device: (pages, masks, counts) per query tile."""
    P, Hkv = r.w.page_size, r.w.num_kv_heads
    max_sel = max(1, max(len(s) for blk in sel_c for s in blk))
    per = TILE // P
    nt = (C + TILE - 1) // TILE
    max_union = min(per, C // P) * max_sel
    lg, ph, cnt = _sel_tensors(r, sel_c, max_sel)
    pages = torch.full((nt, Hkv, max_union), -7, dtype=torch.int32, device=DEV)
    masks = torch.zeros((nt, Hkv, max_union), dtype=torch.uint8, device=DEV)
    counts = torch.full((nt, Hkv), -7, dtype=torch.int32, device=DEV)
    pk.qpage_lists(r.pool, lg, ph, cnt, C, pages, masks, counts)
    return pages, masks, counts


def _host_union(sel_c, P, C, t, g):
    per = TILE // P
    blocks = range(t * per, min((t + 1) * per, C // P))
    union = sorted(set().union(*[set(sel_c[b][g]) for b in blocks]))
    masks = [sum(1 << (b - t * per) for b in blocks if p in sel_c[b][g]) for p in union]
    return union, masks


def _random_page_selections(w, seed):
    """Per chunk, per query page (block of page_size rows), per group: a random
    ascending subset of the past pages (empty lists included)."""
    rng = np.random.default_rng(seed)
    nb = w.chunk_len // w.page_size
    sels = []
    for c in range(w.num_chunks):
        n_past = c * w.pages_per_chunk
        sels.append([[sorted(rng.choice(n_past, size=int(rng.integers(0, n_past + 1)),
                                        replace=False).tolist()) if n_past else []
                      for _ in range(w.num_kv_heads)] for _ in range(nb)])
    return sels


def _run(w, sels, union=True):
    """Every chunk through the C ABI; union=False passes the first query
    page's list as a per-tile list instead (for the equivalence check)."""
    outs = []
    C = w.chunk_len
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            inp = synth.chunk_inputs(w, c)
            cur = r.append(inp["k"], inp["v"])
            past = cnt = masks = None
            if c:
                if union:
                    past, masks, cnt = _union_lists(r, sels[c], C)
                else:
                    per = TILE // w.page_size
                    nt = (C + TILE - 1) // TILE
                    tile_sel = [sels[c][t * per] for t in range(nt)]
                    m = max(1, max(len(s) for blk in tile_sel for s in blk))
                    past = torch.zeros((nt, w.num_kv_heads, m), dtype=torch.int32)
                    cnt = torch.zeros((nt, w.num_kv_heads), dtype=torch.int32)
                    for t in range(nt):
                        for g in range(w.num_kv_heads):
                            s = tile_sel[t][g]
                            past[t, g, :len(s)] = torch.tensor([r.page_table[p] for p in s],
                                                               dtype=torch.int32)
                            cnt[t, g] = len(s)
                    past, cnt = past.to(DEV), cnt.to(DEV)
            q = inp["q"].to(DEV).contiguous()
            o = torch.empty_like(q)
            lse = torch.empty((w.num_q_heads, C), dtype=torch.float32, device=DEV)
            pk.chunk_attn_fwd(r.pool, q, o, lse, past, cnt, cur, w.softmax_scale, fwd_ws=r.fwd_ws,
                              past_masks=masks)
            dq = torch.empty_like(q)
            pk.chunk_attn_bwd(r.pool, q, o, lse, inp["do"].to(DEV).contiguous(), dq,
                              torch.empty_like(lse), past, cnt, cur, w.softmax_scale,
                              past_masks=masks)
            outs.append({"o": o, "lse": lse, "dq": dq})
        torch.cuda.synchronize()
        assert r.status() == 0
        grads = r.grads_by_token(w.context)
    return outs, grads


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


@pytest.mark.parametrize("P,C", [(64, 320), (32, 256), (16, 192)])
def test_union_lists_and_masks_bit_exact(P, C):
    w = synth.Workload("ql", 4, 2, 64, P, C, 3, seed=70 + P, shuffle_pages=True)
    sels = _random_page_selections(w, 71 + P)
    c = w.num_chunks - 1
    with PagedRun(w) as r:
        for cc in range(w.num_chunks):
            r.append(**{k: v for k, v in synth.chunk_inputs(w, cc).items() if k in ("k", "v")})
        pages, masks, counts = _union_lists(r, sels[c], C)
        torch.cuda.synchronize()
        assert r.status() == 0
        pages, masks, counts = pages.cpu(), masks.cpu(), counts.cpu()
        for t in range((C + TILE - 1) // TILE):
            for g in range(w.num_kv_heads):
                union, want_m = _host_union(sels[c], P, C, t, g)
                n = int(counts[t, g])
                assert n == len(union), (t, g)
                assert pages[t, g, :n].tolist() == [r.page_table[p] for p in union], (t, g)
                assert masks[t, g, :n].tolist() == want_m, (t, g)


@pytest.mark.parametrize("w", [
    # 64-token query pages, 2.5 query tiles per chunk (ragged last tile), GQA 7:1
    synth.Workload("qp7", 14, 2, 128, 64, 320, 4, seed=72, shuffle_pages=True),
    # 32-token query pages (four per tile), d 64
    synth.Workload("qp2", 4, 2, 64, 32, 256, 4, seed=73),
    # 16-token query pages (eight per tile), a ragged 1.5-tile chunk
    synth.Workload("qp16", 8, 2, 64, 16, 192, 3, seed=74, shuffle_pages=True),
], ids=["g7_d128_p64_ragged", "g2_d64_p32", "g4_d64_p16_ragged"])
def test_per_query_page_lists_match_oracle(w):
    inp = synth.sequence_inputs(w)
    sels = _random_page_selections(w, 75)
    ref = run_sequence_blocks(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                              w.softmax_scale, w.page_size, selections=sels)
    outs, grads = _run(w, sels)
    _check(w, ref, outs, grads)


def test_same_list_for_every_query_page_equals_per_tile_lists():
    w = synth.Workload("qpeq", 8, 2, 128, 64, 384, 3, seed=76, shuffle_pages=True)
    per = TILE // w.page_size
    base = _random_page_selections(w, 77)
    # every query page of a tile takes the list of the tile's first query page
    sels = [[blk[(b // per) * per] for b, _ in enumerate(blk)] for blk in base]
    outs_u, (dk_u, dv_u) = _run(w, sels, union=True)
    outs_t, (dk_t, dv_t) = _run(w, sels, union=False)
    for a, b in zip(outs_u, outs_t):
        assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
        assert torch.equal(a["dq"], b["dq"])
    assert rel_l2(dk_u, dk_t) <= 1e-6 and rel_l2(dv_u, dv_t) <= 1e-6


def test_per_query_page_topk_then_attention():
    """Batched Top-K with one problem per 64-token query page, the union lists
    on the device, then attention, against the oracle on the same selections
    (which must match the oracle's own per-page Top-K outside the tie band)."""
    w = synth.Workload("qpk", 14, 2, 128, 64, 384, 4, seed=78, shuffle_pages=True,
                       page_direction=0.5, top_k=3, n_recent=2)
    K, R = w.top_k, w.n_recent
    Hkv, C, P = w.num_kv_heads, w.chunk_len, w.page_size
    nb = C // P
    inp = synth.sequence_inputs(w)
    sels, outs = [], []
    with PagedRun(w) as r:
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            n_past = c * w.pages_per_chunk
            q = ch["q"].to(DEV).contiguous()
            past = counts = masks = None
            sel_c = [[[] for _ in range(Hkv)] for _ in range(nb)]
            if n_past:
                out_l = torch.full((nb, Hkv, K + R), -1, dtype=torch.int32, device=DEV)
                out_p = torch.full_like(out_l, 0)
                cnt = torch.zeros((nb, Hkv), dtype=torch.int32, device=DEV)
                ws = torch.empty(pk.page_topk_batched_workspace_size(nb, Hkv, w.head_dim, n_past),
                                 dtype=torch.uint8, device=DEV)
                rs = torch.tensor([b * P for b in range(nb + 1)], dtype=torch.int32, device=DEV)
                npast = torch.full((nb,), n_past, dtype=torch.int32, device=DEV)
                pt = torch.tensor(r.page_table[:n_past], dtype=torch.int32, device=DEV)
                pk.page_topk_batched(r.pool, q, rs, P, npast, n_past, pt, K, R, out_l, out_p,
                                     cnt, ws)
                nt = (C + TILE - 1) // TILE
                mu = (TILE // P) * (K + R)
                past = torch.zeros((nt, Hkv, mu), dtype=torch.int32, device=DEV)
                masks = torch.zeros((nt, Hkv, mu), dtype=torch.uint8, device=DEV)
                counts = torch.zeros((nt, Hkv), dtype=torch.int32, device=DEV)
                pk.qpage_lists(r.pool, out_l, out_p, cnt, C, past, masks, counts)
                torch.cuda.synchronize()
                n = cnt.cpu().numpy()
                sel_c = [[out_l[b, g, :n[b, g]].cpu().tolist() for g in range(Hkv)]
                         for b in range(nb)]
                kbar = page_key_means(inp["k"][:c * C], P)
                for b in range(nb):
                    ref_s = page_scores(group_query_means(ch["q"][b * P:(b + 1) * P], Hkv), kbar)
                    want = select_pages(ref_s, n_past, K, R)
                    for g in range(Hkv):
                        kth = kth_score(ref_s[g], n_past, K, R)
                        for pg in set(sel_c[b][g]) ^ set(want[g]):
                            assert kth is not None and abs(ref_s[g, pg] - kth) <= 1e-5
            sels.append(sel_c)
            cur = r.append(ch["k"], ch["v"])
            o = torch.empty_like(q)
            lse = torch.empty((w.num_q_heads, C), dtype=torch.float32, device=DEV)
            pk.chunk_attn_fwd(r.pool, q, o, lse, past, counts, cur, w.softmax_scale,
                              fwd_ws=r.fwd_ws,
                              past_masks=masks)
            dq = torch.empty_like(q)
            pk.chunk_attn_bwd(r.pool, q, o, lse, ch["do"].to(DEV).contiguous(), dq,
                              torch.empty_like(lse), past, counts, cur, w.softmax_scale,
                              past_masks=masks)
            outs.append({"o": o, "lse": lse, "dq": dq})
        torch.cuda.synchronize()
        assert r.status() == 0
        grads = r.grads_by_token(w.context)
    ref = run_sequence_blocks(inp["q"], inp["k"], inp["v"], inp["do"], C, P, w.softmax_scale,
                              P, selections=sels)
    _check(w, ref, outs, grads)
