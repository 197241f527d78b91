"""GPU parity: segmented attention (the past taken in pieces, merged in fp32).

A chunk's past pages are split into segments; the forward runs FIRST, NEXT...,
LAST (the last with the chunk itself), merging into an fp32 running output and
LSE; the backward runs the same segments, adding dK/dV into the pool and
accumulating dQ in fp32.  Results must match the oracle's dense run with the
usual tolerances (forward O/LSE relative L2 <= 5e-3, max abs <= 1e-2;
dQ/dK/dV relative L2 <= 1e-2) and the whole-key-set GPU run within 5e-3:
each path rounds P to bf16 against its own running maximum (per segment
here, per pass there), so each lies up to a few 1e-3 from the exact result
and their difference can reach the sum.
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.recurrent import run_sequence
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS, BWD_REL = 5e-3, 1e-2, 1e-2
DEV = torch.device("cuda", 0)


def _segments(n_past, seg_pages, empty_last):
    """[(mode, [first_page, last_page)) ...] covering the past; the last carries the chunk."""
    if n_past == 0:
        return [(pk.SEG_WHOLE, (0, 0))]
    bounds = [(a, min(a + seg_pages, n_past)) for a in range(0, n_past, seg_pages)]
    if empty_last:
        bounds.append((n_past, n_past))
    if len(bounds) == 1:
        return [(pk.SEG_WHOLE, bounds[0])]
    modes = [pk.SEG_FIRST] + [pk.SEG_NEXT] * (len(bounds) - 2) + [pk.SEG_LAST]
    return list(zip(modes, bounds))


def _run_segmented(w, seg_pages, empty_last=False, split_fwd=True):
    Hkv, C, Hq, d = w.num_kv_heads, w.chunk_len, w.num_q_heads, w.head_dim
    outs = []
    with PagedRun(w, split_fwd=split_fwd) as r:
        o_acc = torch.empty((C, Hq, d), dtype=torch.float32, device=DEV)
        dq_acc = torch.empty_like(o_acc)
        for c in range(w.num_chunks):
            inp = synth.chunk_inputs(w, c)
            n_past = c * w.pages_per_chunk
            cur = r.append(inp["k"], inp["v"])
            q = inp["q"].to(DEV).contiguous()
            do = inp["do"].to(DEV).contiguous()
            o = torch.empty_like(q)
            lse = torch.empty((Hq, C), dtype=torch.float32, device=DEV)
            dq = torch.empty_like(q)
            delta = torch.empty_like(lse)
            segs = _segments(n_past, seg_pages, empty_last)
            lists = []
            for mode, (a, b) in segs:
                if b > a:
                    ids = torch.tensor([r.page_table[a:b]] * Hkv, dtype=torch.int32, device=DEV)
                    cnt = torch.full((Hkv,), b - a, dtype=torch.int32, device=DEV)
                else:
                    ids, cnt = None, None
                lists.append((mode, ids, cnt))
            for mode, ids, cnt in lists:
                pk.chunk_attn_fwd(r.pool, q, o, lse, ids, cnt, cur, w.softmax_scale,
                                  fwd_ws=r.fwd_ws, segment=mode, o_acc=o_acc)
            for mode, ids, cnt in lists:
                pk.chunk_attn_bwd(r.pool, q, o, lse, do, dq, delta, ids, cnt, cur,
                                  w.softmax_scale, segment=mode, o_acc=o_acc, dq_acc=dq_acc)
            outs.append({"o": o, "lse": lse, "dq": dq})
        torch.cuda.synchronize()
        assert r.status() == 0
        dk, dv = r.grads_by_token(w.context)
    return outs, dk, dv


def _whole(w):
    with PagedRun(w) as r:
        outs = [r.chunk(c, synth.chunk_inputs(w, c)) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        dk, dv = r.grads_by_token(w.context)
    return outs, dk, dv


@pytest.mark.parametrize("split_fwd", [True, False], ids=["split_last_wave", "whole_units"])
@pytest.mark.parametrize("w,seg_pages,empty_last", [
    (synth.Workload("sg7", 14, 2, 128, 64, 320, 4, seed=71, shuffle_pages=True), 3, False),
    (synth.Workload("sg7e", 14, 2, 128, 64, 320, 4, seed=72, shuffle_pages=True), 4, True),
    (synth.Workload("sg2", 4, 2, 64, 32, 256, 4, seed=73), 5, False),
], ids=["g7_d128_seg3", "g7_d128_seg4_empty_last", "g2_d64_seg5"])
def test_segmented_matches_oracle_and_whole(w, seg_pages, empty_last, split_fwd):
    """With the forward workspace every segment call of these small shapes
    splits its units (a partial wave) and merges the parts into the running
    o_acc / LSE in the merge launch; without it the units run whole."""
    inp = synth.sequence_inputs(w)
    ref = run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                       w.softmax_scale)
    outs, dk, dv = _run_segmented(w, seg_pages, empty_last, split_fwd)
    whole, dk_w, dv_w = _whole(w)
    C = w.chunk_len
    for c, (out, wo) in enumerate(zip(outs, whole)):
        o, lse = to64(out["o"]), to64(out["lse"])
        o_ref, lse_ref = ref["o"][c * C:(c + 1) * C], ref["lse"][:, c * C:(c + 1) * C]
        assert rel_l2(o, o_ref) <= FWD_REL and np.max(np.abs(o - o_ref)) <= FWD_ABS, c
        assert rel_l2(lse, lse_ref) <= FWD_REL and np.max(np.abs(lse - lse_ref)) <= FWD_ABS, c
        assert rel_l2(o, to64(wo["o"])) <= 5e-3, c
        assert rel_l2(lse, to64(wo["lse"])) <= 5e-3, c
        assert rel_l2(to64(out["dq"]), to64(wo["dq"])) <= 5e-3, c
    dq = np.concatenate([to64(o["dq"]) for o in outs], axis=0)
    assert rel_l2(dq, ref["dq"]) <= BWD_REL
    assert rel_l2(dk, ref["dk"]) <= BWD_REL and rel_l2(dv, ref["dv"]) <= BWD_REL
    assert rel_l2(dk, dk_w) <= 5e-3 and rel_l2(dv, dv_w) <= 5e-3


def test_segment_arguments_are_checked():
    w = synth.Workload("sga", 4, 2, 64, 32, 128, 1, seed=74)
    with PagedRun(w) as r:
        inp = synth.chunk_inputs(w, 0)
        cur = r.append(inp["k"], inp["v"])
        q = inp["q"].to(DEV).contiguous()
        o, lse = torch.empty_like(q), torch.empty((4, 128), dtype=torch.float32, device=DEV)
        with pytest.raises(pk.OombError):     # a segment without the fp32 running output
            pk.chunk_attn_fwd(r.pool, q, o, lse, None, None, cur, w.softmax_scale, fwd_ws=r.fwd_ws,
                              segment=pk.SEG_FIRST)
        with pytest.raises(pk.OombError):     # mode out of range
            pk.chunk_attn_fwd(r.pool, q, o, lse, None, None, cur, w.softmax_scale,
                              fwd_ws=r.fwd_ws, segment=7,
                              o_acc=torch.empty((128, 4, 64), dtype=torch.float32, device=DEV))
