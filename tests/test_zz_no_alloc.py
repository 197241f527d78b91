"""The allocation-free Top-K entry point (oomb_page_topk_static).

It serves callers that cannot allocate device memory (a host framework that
owns all device allocations, or a loop where a cudaMalloc is not acceptable):
the scratch comes from a static device array inside the library instead of a
caller workspace.  This checks, through the C ABI, that two calls in a row
(different chunks, so the second finds the first one's leftovers in the
shared array) give exactly what oomb_page_topk gives with a fresh workspace.
Collected last on purpose: it must pass alone in a fresh process and after
the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
import paged_kv_chunk_query_b200._lib as L
from paged_kv_chunk_query_b200 import synth

pytestmark = pytest.mark.gpu


def _outs(Hkv, ms, n_past, dev):
    return (torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev),
            torch.full((Hkv, ms), -1, dtype=torch.int32, device=dev),
            torch.zeros(Hkv, dtype=torch.int32, device=dev),
            torch.zeros((Hkv, max(n_past, 1)), dtype=torch.float32, device=dev))


def test_static_scratch_topk_matches_workspace_topk_on_two_calls():
    dev = torch.device("cuda", 0)
    w = synth.Workload("noalloc", 14, 2, 128, 64, 256, 5, seed=91, shuffle_pages=True,
                       page_direction=0.5)
    K, R = 3, 2
    pool = pk.pool_create(w.num_pages, w.page_size, w.num_kv_heads, w.head_dim, pk.LOC_DEVICE,
                          True, w.alloc_seed, 0)
    try:
        table = []
        for c in range(w.num_chunks):
            ch = synth.chunk_inputs(w, c)
            ids = [pk.pool_alloc_page(pool) for _ in range(w.pages_per_chunk)]
            table += ids
            pk.kv_append(pool, torch.tensor(ids, dtype=torch.int32, device=dev),
                         ch["k"].to(dev), ch["v"].to(dev))
        pt = torch.tensor(table, dtype=torch.int32, device=dev)
        for c in (4, 2):  # two calls in a row, different sizes and queries
            q = synth.chunk_inputs(w, c)["q"].to(dev)
            n_past = c * w.pages_per_chunk
            ms = K + R
            ref = _outs(w.num_kv_heads, ms, n_past, dev)
            ws = torch.empty(pk.page_topk_workspace_size(w.chunk_len, w.num_q_heads,
                                                         w.num_kv_heads, w.head_dim, n_past),
                             dtype=torch.uint8, device=dev)
            pk.page_topk(pool, q, pt[:n_past], n_past, K, R, ref[0], ref[1], ref[2], ws,
                         out_scores=ref[3])
            got = _outs(w.num_kv_heads, ms, n_past, dev)
            L.page_topk_static(pool, q, pt[:n_past], n_past, K, R, got[0], got[1], got[2],
                               out_scores=got[3])
            torch.cuda.synchronize()
            assert torch.equal(got[2], ref[2])
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
            np.testing.assert_allclose(got[3][:, :n_past].cpu().numpy(),
                                       ref[3][:, :n_past].cpu().numpy(), rtol=1e-6, atol=1e-7)
        assert pk.get_device_status(pool) == 0
    finally:
        pk.pool_destroy(pool)


def test_static_scratch_rejects_oversized_problems():
    dev = torch.device("cuda", 0)
    pool = pk.pool_create(64, 64, 4, 128, pk.LOC_DEVICE, False, 0, 0)
    try:
        q = torch.zeros((256, 28, 128), dtype=torch.bfloat16, device=dev)
        n_past = 30000  # needs more than the static scratch holds
        assert pk.page_topk_workspace_size(256, 28, 4, 128, n_past) > L.TOPK_STATIC_SCRATCH_BYTES
        pt = torch.zeros(n_past, dtype=torch.int32, device=dev)
        o = _outs(4, 66, n_past, dev)
        with pytest.raises(L.OombError) as e:
            L.page_topk_static(pool, q, pt, n_past, 64, 2, o[0], o[1], o[2])
        assert e.value.status == L.ERR_UNSUPPORTED
    finally:
        pk.pool_destroy(pool)
