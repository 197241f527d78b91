"""GPU parity: the Q/K/V projection GEMM with its paged epilogue.

Q, K, V are bf16 roundings of fp32 sums; the oracle rounds its fp64 products
to bf16, so the two may differ by one bf16 step (the rounding of nearly tied
values), and where the dot product nearly cancels the fp32 sum itself is off
by up to ~K eps_32 max|x w| in absolute terms: each element must lie within
one bf16 ulp of the oracle's rounded value or within 1e-4 of it.  The page
means and the per-group Q sums are checked against their definition on the
GPU's own bf16 outputs (fp32 atomics: relative 1e-5).
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.projection import qkv_projection

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _bf16_ulp(x):
    a = np.maximum(np.abs(x), 1e-30)
    return np.exp2(np.floor(np.log2(a)) - 7)


def _within_one_ulp(got, ref):
    ref_b = torch.tensor(ref, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    err = np.abs(got - ref_b)
    ok = (err <= _bf16_ulp(ref) * 1.0001) | (err <= 1e-4)
    assert ok.all(), (float(err.max()), int((~ok).sum()), float(np.abs(got - ref).max()))
    return True


@pytest.mark.parametrize("C,hidden,Hq,Hkv,d,P", [(256, 512, 14, 2, 128, 64),
                                                 (192, 128, 4, 2, 64, 16)],
                         ids=["g7_d128_p64", "g2_d64_p16_ragged"])
def test_projection_matches_oracle(C, hidden, Hq, Hkv, d, P):
    gen = torch.Generator().manual_seed(C + hidden)
    x = torch.randn(C, hidden, generator=gen).to(torch.bfloat16)
    n_out = (Hq + 2 * Hkv) * d
    w = (torch.randn(n_out, hidden, generator=gen) / hidden ** 0.5).to(torch.bfloat16)
    q_ref, k_ref, v_ref = qkv_projection(x.float().numpy(), w.float().numpy(), Hq, Hkv, d)
    n_pages = C // P
    pool = pk.pool_create(2 * n_pages + 3, P, Hkv, d, pk.LOC_DEVICE, True, 9, 0)
    try:
        pages = [pk.pool_alloc_page(pool) for _ in range(n_pages)]
        pid = torch.tensor(pages, dtype=torch.int32, device=DEV)
        kv, grad, summ = pk.pool_views(pool)
        grad.fill_(7.0)
        xd, wd = x.to(DEV), w.to(DEV)
        q = torch.zeros((C, Hq, d), dtype=torch.bfloat16, device=DEV)
        qsum = torch.full((Hkv, d), 3.0, dtype=torch.float32, device=DEV)
        pk.qkv_project(pool, xd, wd, Hq, pk.PROJ_Q, q=q, qsum=qsum)
        pk.qkv_project(pool, xd, wd, Hq, pk.PROJ_KV, page_ids=pid)
        torch.cuda.synchronize()
        assert pk.get_device_status(pool) == 0
        qg = q.double().cpu().numpy()
        assert _within_one_ulp(qg, q_ref)
        ids = torch.tensor(pages, dtype=torch.long, device=DEV)
        blk = kv[ids].double().cpu().numpy()          # [pages][Hkv][2][P][d]
        kg = blk[:, :, 0].transpose(0, 2, 1, 3).reshape(C, Hkv, d)
        vg = blk[:, :, 1].transpose(0, 2, 1, 3).reshape(C, Hkv, d)
        assert _within_one_ulp(kg, k_ref) and _within_one_ulp(vg, v_ref)
        # page means of the stored K, and the per-group sums of the stored Q
        want_s = kg.reshape(n_pages, P, Hkv, d).mean(axis=1)
        got_s = summ[ids].double().cpu().numpy()
        assert np.max(np.abs(got_s - want_s)) <= 1e-5 * max(1.0, np.max(np.abs(want_s)))
        want_q = qg.reshape(C, Hkv, Hq // Hkv, d).sum(axis=(0, 2))
        assert np.max(np.abs(qsum.double().cpu().numpy() - want_q)) <= \
            1e-5 * max(1.0, np.max(np.abs(want_q)))
        assert float(grad[ids].abs().max()) == 0.0       # gradient blocks zeroed
        # the one-launch form writes the same Q, K and V
        q2 = torch.zeros_like(q)
        kv.zero_()
        pk.qkv_project(pool, xd, wd, Hq, pk.PROJ_QKV, q=q2, page_ids=pid)
        torch.cuda.synchronize()
        assert torch.equal(q2, q)
        blk2 = kv[ids].double().cpu().numpy()
        assert np.array_equal(blk2, blk)
    finally:
        pk.pool_destroy(pool)


def test_projection_arguments_are_checked():
    pool = pk.pool_create(8, 64, 2, 128, pk.LOC_DEVICE, True, 0, 0)
    try:
        x = torch.zeros((128, 100), dtype=torch.bfloat16, device=DEV)   # hidden % 64 != 0
        w = torch.zeros((6 * 128, 100), dtype=torch.bfloat16, device=DEV)
        with pytest.raises(pk.OombError):
            pk.qkv_project(pool, x, w, 4, pk.PROJ_Q, q=torch.zeros((128, 4, 128),
                                                                dtype=torch.bfloat16, device=DEV))
        x = torch.zeros((128, 128), dtype=torch.bfloat16, device=DEV)
        w = torch.zeros((6 * 128, 128), dtype=torch.bfloat16, device=DEV)
        with pytest.raises(pk.OombError):                              # K/V part needs pages
            pk.qkv_project(pool, x, w, 4, pk.PROJ_KV)
    finally:
        pk.pool_destroy(pool)
