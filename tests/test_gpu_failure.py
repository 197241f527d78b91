"""Failure detection on the GPU without faulting it.

Kernels never trap: an invalid page id in a list is reported in the pool's
device status word and read as zeros (TMA out-of-bounds fill), a count above
the list stride is clamped and reported, and a wait whose arrival never
comes gives up after its limit and reports.  Each test checks the status the
host reads and that the context keeps working afterwards.
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
import paged_kv_chunk_query_b200._lib as L
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun

pytestmark = pytest.mark.gpu


def _small():
    return synth.Workload("fail", 8, 2, 128, 64, 256, 3, seed=71)


def _run_chunk(r, w, c, past, cnt):
    ch = synth.chunk_inputs(w, c)
    cur = r.append(ch["k"], ch["v"])
    q = ch["q"].cuda()
    o = torch.empty_like(q)
    lse = torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32, device="cuda")
    pk.chunk_attn_fwd(r.pool, q, o, lse, past, cnt, cur, w.softmax_scale, fwd_ws=r.fwd_ws)
    dq = torch.empty_like(q)
    delta = torch.empty_like(lse)
    pk.chunk_attn_bwd(r.pool, q, o, lse, ch["do"].cuda(), dq, delta, past, cnt, cur,
                      w.softmax_scale)
    torch.cuda.synchronize()
    return o, lse, dq


def test_invalid_page_id_is_reported_not_faulted():
    w = _small()
    with PagedRun(w) as r:
        _run_chunk(r, w, 0, None, None)
        good = r.page_table[: w.pages_per_chunk]
        bad = [good[0], w.num_pages + 5, good[2], -3]         # two invalid ids
        past = torch.tensor([bad, good], dtype=torch.int32, device="cuda")
        cnt = torch.tensor([4, 4], dtype=torch.int32, device="cuda")
        o, lse, dq = _run_chunk(r, w, 1, past, cnt)
        word = r.status()
        assert word & 1, word
        assert torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()
        assert r.status() == 0                                 # reading clears it
        # the context still works
        _run_chunk(r, w, 2, r.past_lists(2 * w.pages_per_chunk)[0],
                   r.past_lists(2 * w.pages_per_chunk)[1])
        assert r.status() == 0


def test_count_above_list_stride_is_clamped_and_reported():
    w = _small()
    with PagedRun(w) as r:
        _run_chunk(r, w, 0, None, None)
        past, cnt = r.past_lists(w.pages_per_chunk)
        cnt = torch.tensor([w.pages_per_chunk + 9, w.pages_per_chunk], dtype=torch.int32,
                           device="cuda")
        o, _, _ = _run_chunk(r, w, 1, past, cnt)
        assert r.status() & 4
        assert torch.isfinite(o.float()).all()


def test_wait_limit_reports_and_context_survives():
    w = _small()
    with PagedRun(w) as r:
        ev = torch.cuda.Event()
        L.selftest_wait_limit(r.pool)
        ev.record()
        with pytest.raises(L.OombError) as e:                  # still running (~1 s)
            pk.wait(ev, 1000)
        assert e.value.status == L.ERR_TIMEOUT
        pk.wait(ev, 30_000_000)
        assert r.status() & 2
        assert r.status() == 0
        _run_chunk(r, w, 0, None, None)
        assert r.status() == 0
