"""GPU tests of the offload path: pinned-host pools, block prefetch / store,
gradient write-back, and a whole offloaded Top-K run against the same run
with every page resident on the device.

The offloaded run computes on a small staging pool; its forward outputs must
equal the device-resident run's bit for bit (same kernels, same key order),
and the host gradient pool must match the device one up to fp32 summation
order (relative L2 <= 1e-5), and the oracle within the backward tolerance.
"""
import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200 as pk
from oracle.recurrent import run_sequence
from paged_kv_chunk_query_b200 import synth
from paged_kv_chunk_query_b200.offload import OffloadRun
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu


def test_store_and_prefetch_round_trip_bit_exact():
    dev = torch.device("cuda", 0)
    P, Hkv, d = 64, 2, 128
    a = pk.pool_create(8, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    h = pk.pool_create(16, P, Hkv, d, pk.LOC_PINNED_HOST, True, 3, 0)
    b = pk.pool_create(8, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    try:
        gen = torch.Generator().manual_seed(1)
        k = torch.randn(4 * P, Hkv, d, generator=gen).to(torch.bfloat16).to(dev)
        v = torch.randn(4 * P, Hkv, d, generator=gen).to(torch.bfloat16).to(dev)
        pages_a = [pk.pool_alloc_page(a) for _ in range(4)]
        pk.kv_append(a, torch.tensor(pages_a, dtype=torch.int32, device=dev), k, v)
        pages_h = [pk.pool_alloc_page(h) for _ in range(4)]
        src = [p * Hkv + g for p in pages_a for g in range(Hkv)]
        dst = [p * Hkv + g for p in pages_h for g in range(Hkv)]
        pk.page_prefetch(a, h, src, dst)                  # device -> pinned host (store)
        torch.cuda.synchronize()
        kv_a, _, s_a = pk.pool_views(a)
        kv_h, _, s_h = pk.pool_views(h)
        assert s_h.is_cuda and not kv_h.is_cuda
        for pa, ph in zip(pages_a, pages_h):
            assert torch.equal(kv_h[ph], kv_a[pa].cpu())
            assert torch.equal(s_h[ph], s_a[pa])
        # pinned host -> another device pool, one head only, reversed order
        pages_b = [pk.pool_alloc_page(b) for _ in range(4)]
        src = [p * Hkv + 1 for p in reversed(pages_h)]
        dst = [p * Hkv + 1 for p in pages_b]
        ev = torch.cuda.Event()
        pk.page_prefetch(h, b, src, dst, done_event=ev)
        pk.wait(ev, 10_000_000)
        kv_b, _, _ = pk.pool_views(b)
        for ph, pb in zip(reversed(pages_h), pages_b):
            assert torch.equal(kv_b[pb, 1].cpu(), kv_h[ph, 1])
        with pytest.raises(pk.OombError) as e:           # out-of-range block id
            pk.page_prefetch(h, b, [16 * Hkv], [0])
        assert e.value.status == pk._lib.ERR_BAD_PAGE
    finally:
        for pool in (a, h, b):
            pk.pool_destroy(pool)


def test_grad_writeback_adds_and_zeroes():
    dev = torch.device("cuda", 0)
    P, Hkv, d = 32, 2, 64
    a = pk.pool_create(6, P, Hkv, d, pk.LOC_DEVICE, True, 0, 0)
    h = pk.pool_create(10, P, Hkv, d, pk.LOC_PINNED_HOST, True, 0, 0)
    try:
        _, ga, _ = pk.pool_views(a)
        _, gh, _ = pk.pool_views(h)
        gen = torch.Generator().manual_seed(2)
        ga.copy_(torch.randn(ga.shape, generator=gen).to(dev))
        gh.copy_(torch.randn(gh.shape, generator=gen))
        before_h = gh.clone()
        before_a = ga.cpu()
        src = [0, 1, 2, 3, 7, 9, 10]          # block ids (page * Hkv + head)
        dst = [19, 18, 4, 5, 6, 0, 11]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            pk.grad_writeback(a, h, src, dst, stream=stream)
        stream.synchronize()
        pk.grad_writeback_sync(a)
        bh = before_h.view(-1, 2 * P * d)
        ba = before_a.view(-1, 2 * P * d)
        want = bh.clone()
        for s_, d_ in zip(src, dst):
            want[d_] = bh[d_] + ba[s_]  # one IEEE fp32 add per element, as on the host
        assert torch.equal(gh.view(-1, 2 * P * d), want)
        ga_now = ga.cpu().view(-1, 2 * P * d)
        for blk in range(ga_now.shape[0]):
            if blk in src:
                assert float(ga_now[blk].abs().max()) == 0.0
            else:
                assert torch.equal(ga_now[blk], ba[blk])
    finally:
        pk.pool_destroy(a)
        pk.pool_destroy(h)


def test_offloaded_topk_run_matches_device_resident_run():
    dev = torch.device("cuda", 0)
    w = synth.Workload("off", 14, 2, 128, 64, 256, 8, seed=61, shuffle_pages=True,
                       page_direction=0.5, top_k=3, n_recent=2, host_resident=True)
    ins = [{k: v.to(dev) for k, v in synth.chunk_inputs(w, c).items()} for c in range(w.num_chunks)]
    C, Hq = w.chunk_len, w.num_q_heads
    outs = [(torch.empty_like(x["q"]), torch.empty((Hq, C), dtype=torch.float32, device=dev),
             torch.empty_like(x["q"])) for x in ins]
    run = OffloadRun(w, dev)
    try:
        run.run(lambda c: ins[c], lambda c: outs[c])
        run.sync()
        assert pk.get_device_status(run.stage) == 0
        sels = run.selections
        _, gh, _ = pk.pool_views(run.host)
        P = w.page_size
        ids = torch.tensor(run.table, dtype=torch.long)
        g = gh[ids].permute(0, 3, 1, 2, 4).reshape(w.context, w.num_kv_heads, 2, w.head_dim)
        dk_off, dv_off = g[:, :, 0].double().numpy(), g[:, :, 1].double().numpy()
    finally:
        run.close()
    with PagedRun(w) as r:
        ref = [r.chunk(c, synth.chunk_inputs(w, c), selected=sels[c] if c else None)
               for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        dk_dev, dv_dev = r.grads_by_token(w.context)
    for c in range(w.num_chunks):
        assert torch.equal(outs[c][0], ref[c]["o"]), c
        assert torch.equal(outs[c][1], ref[c]["lse"]), c
        assert torch.equal(outs[c][2], ref[c]["dq"]), c
    assert rel_l2(dk_off, dk_dev) <= 1e-5 and rel_l2(dv_off, dv_dev) <= 1e-5
    inp = synth.sequence_inputs(w)
    orc = run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], C, P, w.softmax_scale,
                       selections=sels)
    assert rel_l2(dk_off, orc["dk"]) <= 1e-2 and rel_l2(dv_off, orc["dv"]) <= 1e-2
    _check_outputs_against_oracle(outs, orc)


def _check_outputs_against_oracle(outs, orc):
    """Forward O and LSE (rel L2 <= 5e-3, max abs <= 1e-2) and dQ (rel L2 <=
    1e-2) of every chunk, concatenated, against the oracle's sequence run."""
    o = np.concatenate([to64(x[0]) for x in outs])
    lse = np.concatenate([to64(x[1]) for x in outs], axis=1)
    dq = np.concatenate([to64(x[2]) for x in outs])
    assert rel_l2(o, orc["o"]) <= 5e-3 and np.max(np.abs(o - orc["o"])) <= 1e-2
    assert rel_l2(lse, orc["lse"]) <= 5e-3 and np.max(np.abs(lse - orc["lse"])) <= 1e-2
    assert rel_l2(dq, orc["dq"]) <= 1e-2


@pytest.mark.parametrize("window,grad_path,slots", [(3, "gpu", 3), (20, "gpu", 3),
                                                    (3, "host", 3), (3, "gpu", 2),
                                                    (2, "host", 2), (3, "host", 4)])
def test_dense_offload_matches_device_resident_run(window, grad_path, slots):
    """Dense attention with KV and gradients in pinned host memory and
    `slots` slots of `window` past pages on the device (segments merged in
    fp32; fetches slots - 1 calls ahead) against the device-resident dense
    run and the oracle."""
    from paged_kv_chunk_query_b200.offload import DenseOffloadRun
    dev = torch.device("cuda", 0)
    w = synth.Workload("doff", 14, 2, 128, 64, 256, 5, seed=67, shuffle_pages=True)
    ins = [{k: v.to(dev) for k, v in synth.chunk_inputs(w, c).items()} for c in range(w.num_chunks)]
    C, Hq = w.chunk_len, w.num_q_heads
    outs = [(torch.empty_like(x["q"]), torch.empty((Hq, C), dtype=torch.float32, device=dev),
             torch.empty_like(x["q"])) for x in ins]
    run = DenseOffloadRun(w, dev, window, grad_path, slots)
    try:
        run.run(lambda c: ins[c], lambda c: outs[c])
        run.sync()
        assert pk.get_device_status(run.stage) == 0 and pk.get_device_status(run.host) == 0
        _, gh, _ = pk.pool_views(run.host)
        ids = torch.tensor(run.table, dtype=torch.long)
        g = gh[ids].permute(0, 3, 1, 2, 4).reshape(w.context, w.num_kv_heads, 2, w.head_dim)
        dk_off, dv_off = g[:, :, 0].double().numpy(), g[:, :, 1].double().numpy()
    finally:
        run.close()
    with PagedRun(w) as r:
        ref = [r.chunk(c, synth.chunk_inputs(w, c)) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        dk_dev, dv_dev = r.grads_by_token(w.context)
    for c in range(w.num_chunks):
        for i, key in enumerate(("o", "lse", "dq")):
            assert rel_l2(to64(outs[c][i]), to64(ref[c][key])) <= 5e-3, (c, key)
    assert rel_l2(dk_off, dk_dev) <= 5e-3 and rel_l2(dv_off, dv_dev) <= 5e-3
    inp = synth.sequence_inputs(w)
    orc = run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], C, w.page_size, w.softmax_scale)
    assert rel_l2(dk_off, orc["dk"]) <= 1e-2 and rel_l2(dv_off, orc["dv"]) <= 1e-2
    _check_outputs_against_oracle(outs, orc)
