"""C-ABI checks that need no GPU: the library loads, exports every function
include/oomb.h declares, and its host logic (page allocator, argument
validation, status strings) behaves as specified.  Pools here use
OOMB_LOC_HOST, which makes no CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import paged_kv_chunk_query_b200._lib as L
from oracle.pool import PoolModel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "oomb.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(oomb_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = L.load()
    declared = _declared()
    assert len(declared) >= 19
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(L.EXPORTS) == declared


def test_version_and_status_strings():
    assert L.version() == 100
    assert L.status_string(0) == "ok"
    assert L.status_string(2) == "out of pages"
    assert L.status_string(99) == "unknown status"


@pytest.mark.parametrize("seed", [0, 1, 1003, 2**63 + 5])
def test_allocator_matches_free_list_model_bit_exact(seed):
    n = 257
    pool = L.pool_create(n, 16, 2, 64, L.LOC_HOST, True, seed)
    model = PoolModel(n, seed)
    try:
        ops = [("a",)] * 100 + [("f", 5), ("f", 77), ("a",), ("a",), ("f", 3)] + [("a",)] * 200
        for op in ops:
            if op[0] == "a":
                want = model.alloc()
                if want is None:
                    with pytest.raises(L.OombError) as e:
                        L.pool_alloc_page(pool)
                    assert e.value.status == L.ERR_OUT_OF_PAGES
                else:
                    assert L.pool_alloc_page(pool) == want
            else:
                ok = model.free(op[1])
                if ok:
                    L.pool_free_page(pool, op[1])
                else:
                    with pytest.raises(L.OombError) as e:
                        L.pool_free_page(pool, op[1])
                    assert e.value.status == L.ERR_BAD_PAGE
        assert L.pool_num_free(pool) == len(model.stack)
    finally:
        L.pool_destroy(pool)


def test_allocator_errors():
    pool = L.pool_create(4, 16, 1, 64, L.LOC_HOST, False, 0)
    try:
        for bad in (-1, 4, 100):
            with pytest.raises(L.OombError) as e:
                L.pool_free_page(pool, bad)
            assert e.value.status == L.ERR_BAD_PAGE
        p = L.pool_alloc_page(pool)
        L.pool_free_page(pool, p)
        with pytest.raises(L.OombError) as e:  # double free
            L.pool_free_page(pool, p)
        assert e.value.status == L.ERR_BAD_PAGE
    finally:
        L.pool_destroy(pool)


@pytest.mark.parametrize("kw,status", [
    (dict(num_pages=0), L.ERR_INVALID_ARG),
    (dict(num_kv_heads=0), L.ERR_INVALID_ARG),
    (dict(head_dim=96), L.ERR_UNSUPPORTED),
    (dict(page_size=48), L.ERR_UNSUPPORTED),
    (dict(location=7), L.ERR_INVALID_ARG),
])
def test_pool_create_rejects_bad_descriptors(kw, status):
    args = dict(num_pages=8, page_size=16, num_kv_heads=1, head_dim=64, location=L.LOC_HOST,
                with_grad=True, alloc_seed=0)
    args.update(kw)
    with pytest.raises(L.OombError) as e:
        L.pool_create(**args)
    assert e.value.status == status


def test_host_pool_layout_and_views():
    pool = L.pool_create(3, 16, 2, 64, L.LOC_HOST, True, 0)
    try:
        d = L.pool_get_desc(pool)
        assert (d.num_pages, d.page_size, d.num_kv_heads, d.head_dim) == (3, 16, 2, 64)
        kv, grad, summ = L.pool_views(pool)
        assert tuple(kv.shape) == (3, 2, 2, 16, 64) and tuple(grad.shape) == (3, 2, 2, 16, 64)
        assert tuple(summ.shape) == (3, 2, 64)
        assert float(kv.float().abs().sum()) == 0.0 and float(grad.abs().sum()) == 0.0
    finally:
        L.pool_destroy(pool)


def test_compute_calls_reject_host_pools_without_touching_cuda():
    """Argument errors are caught on the host before any launch."""
    lib = L.load()
    pool = L.pool_create(8, 16, 1, 64, L.LOC_HOST, True, 0)
    try:
        assert lib.oomb_kv_append(pool, None, 1, None, None, None) == L.ERR_INVALID_ARG
        args = L.AttnArgs()
        assert lib.oomb_chunk_attn_fwd(pool, ctypes.byref(args), None) == L.ERR_INVALID_ARG
        assert lib.oomb_chunk_attn_bwd(pool, ctypes.byref(args), None) == L.ERR_INVALID_ARG
        assert lib.oomb_chunk_attn_bwd_step(pool, ctypes.byref(args), 7, None) == L.ERR_INVALID_ARG
        assert lib.oomb_page_topk(pool, None, 64, 4, None, 0, 4, 2, None, None, None, None,
                                  None, 0, None) == L.ERR_INVALID_ARG
        assert lib.oomb_page_prefetch(pool, pool, None, None, 0, None, None) == L.ERR_INVALID_ARG
        assert lib.oomb_grad_writeback(pool, pool, None, None, 1, None) == L.ERR_INVALID_ARG
        assert lib.oomb_chunk_attn_fwd(None, ctypes.byref(args), None) == L.ERR_INVALID_ARG
        assert lib.oomb_wait(None, 10) == L.ERR_INVALID_ARG
    finally:
        L.pool_destroy(pool)


def test_topk_workspace_size_formula():
    ws = L.page_topk_workspace_size(4096, 28, 4, 128, 4094)
    # 128 slices x 4 groups x 128 d fp32 partials + 4 x 4094 64-bit keys, 256-byte aligned
    # query-mean partials (128 slices), q_bar, then the 64-bit page keys
    assert ws == 128 * 4 * 128 * 4 + 4 * 128 * 4 + ((4 * 4094 * 8 + 255) // 256) * 256
    assert L.page_topk_workspace_size(0, 28, 4, 128, 10) == 0
    # key rows have an even stride (16-byte aligned rows): 4095 pages take 4096 slots
    assert L.page_topk_workspace_size(4096, 28, 4, 128, 4095) == \
        128 * 4 * 128 * 4 + 4 * 128 * 4 + 4 * 4096 * 8


def test_qsum_topk_workspace_size_formula():
    """The one-launch selection needs only the counters and the keys."""
    def a256(x):
        return (x + 255) // 256 * 256
    assert L.page_topk_qsum_workspace_size(4, 4032) == a256(4 * 4) + a256(4 * 4032 * 8)
    assert L.page_topk_qsum_workspace_size(4, 4031) == a256(4 * 4) + a256(4 * 4032 * 8)
    assert L.page_topk_qsum_workspace_size(2, 0) == a256(2 * 4) + a256(2 * 2 * 8)
    assert L.page_topk_qsum_workspace_size(0, 10) == 0
    assert L.page_topk_qsum_workspace_size(4, -1) == 0


def test_host_block_lists_checked_before_the_call():
    """Block lists are copied to the host and must pair up one to one; a
    mismatch is refused before the library is called."""
    with pytest.raises(ValueError):
        L.page_prefetch(None, None, [1, 2, 3], [4, 5])
    with pytest.raises(ValueError):
        L.grad_writeback(None, None, np.arange(4, dtype=np.int64), [0])
    t, ptr = L._host_i32(torch.arange(5, dtype=torch.int64))
    assert t.dtype == torch.int32 and not t.is_cuda and ptr == t.data_ptr()
    assert t.tolist() == [0, 1, 2, 3, 4]


def test_fwd_workspace_size_formula():
    # 256 parts x 128 rows: normalised fp32 O (d values) and the LSE per row
    assert L.chunk_attn_fwd_workspace_size(128) == 256 * 128 * (128 + 1) * 4
    assert L.chunk_attn_fwd_workspace_size(64) == 256 * 128 * (64 + 1) * 4
    assert L.chunk_attn_fwd_workspace_size(96) == 0


def test_newer_entry_points_reject_host_pools_without_touching_cuda():
    """Block moves, list builders, batched / static Top-K and the projection
    check their pools' locations on the host first."""
    lib = L.load()
    pool = L.pool_create(8, 16, 1, 64, L.LOC_HOST, True, 0)
    try:
        assert lib.oomb_block_copy(pool, pool, None, None, 1, None) == L.ERR_INVALID_ARG
        assert lib.oomb_grad_block_add(pool, pool, None, None, 1, 1, None) == L.ERR_INVALID_ARG
        assert lib.oomb_prefetch_lists(pool, pool, None, None, 4, None, 0, None, None, None,
                                       None, None) == L.ERR_INVALID_ARG
        assert lib.oomb_local_pages(pool, None, 0, 4, None, None, None) == L.ERR_INVALID_ARG
        assert lib.oomb_page_topk_batched(pool, None, 64, 4, 1, None, 64, None, 0, None, 4, 2,
                                          None, None, None, None, None, 0,
                                          None) == L.ERR_INVALID_ARG
        assert lib.oomb_page_topk_static(pool, None, 64, 4, None, 0, 4, 2, None, None, None,
                                         None, None) == L.ERR_INVALID_ARG
        assert lib.oomb_qkv_project(pool, None, None, 128, 64, 4, L.PROJ_QKV, None, None, None,
                                    None) == L.ERR_INVALID_ARG
        assert lib.oomb_block_copy(None, pool, None, None, 0, None) == L.ERR_INVALID_ARG
        assert lib.oomb_selftest_wait_limit(pool, None) == L.ERR_INVALID_ARG
        assert lib.oomb_qpage_lists(pool, None, None, None, 64, 4, None, None, None, 8,
                                    None) == L.ERR_INVALID_ARG
        assert lib.oomb_page_topk_qsum(pool, None, 64, 4, None, 0, 4, 2, None, None, None,
                                       None, None, 0, None) == L.ERR_INVALID_ARG
    finally:
        L.pool_destroy(pool)


def test_batched_topk_workspace_size_formula():
    def a256(x):
        return (x + 255) // 256 * 256
    B, Hkv, d, mp = 64, 4, 128, 4032
    want = a256(B * 128 * Hkv * d * 4) + a256(B * Hkv * d * 4) + a256(B * Hkv * mp * 8)
    assert L.page_topk_batched_workspace_size(B, Hkv, d, mp) == want
    # one problem is the per-chunk workspace
    assert L.page_topk_batched_workspace_size(1, Hkv, d, mp) == \
        L.page_topk_workspace_size(4096, 28, Hkv, d, mp)
    assert L.page_topk_batched_workspace_size(0, Hkv, d, mp) == 0


def test_grad_writeback_rejects_repeated_destinations_before_cuda():
    """The worker's CPU threads add blocks in parallel, so a destination listed
    twice would lose an addition: the list is checked in one pass, in order,
    before the pools' locations (so host pools reach the check here)."""
    lib = L.load()
    pool = L.pool_create(8, 16, 1, 64, L.LOC_HOST, True, 0)
    try:
        src = (ctypes.c_int32 * 3)(0, 1, 2)
        dup = (ctypes.c_int32 * 3)(4, 4, 99)     # repeat first, out of range after
        out = (ctypes.c_int32 * 3)(4, 5, 99)     # out of range, no repeat
        ok = (ctypes.c_int32 * 3)(4, 5, 6)
        assert lib.oomb_grad_writeback(pool, pool, src, dup, 3, None) == L.ERR_INVALID_ARG
        assert lib.oomb_grad_writeback(pool, pool, src, out, 3, None) == L.ERR_BAD_PAGE
        # a valid distinct list passes the list checks and stops at the location check
        assert lib.oomb_grad_writeback(pool, pool, src, ok, 3, None) == L.ERR_INVALID_ARG
        bad_src = (ctypes.c_int32 * 3)(0, 1, 8)
        assert lib.oomb_grad_writeback(pool, pool, bad_src, ok, 3, None) == L.ERR_BAD_PAGE
    finally:
        L.pool_destroy(pool)


def test_grad_writeback_worker_skips_a_failed_copy_and_reports_it():
    """A staging slot whose device->host copy failed is not added into the host
    gradients, and the sync reports OOMB_ERR_CUDA; a completed copy is added."""
    import numpy as np
    lib = L.load()
    n, bf = 5, 96
    host = np.full(n * bf + 7, 2.5, dtype=np.float32)
    ptr = host.ctypes.data_as(ctypes.c_void_p)
    assert lib.oomb_selftest_writeback_copy(ptr, n, bf, 1) == L.ERR_CUDA
    assert np.all(host == 2.5)
    assert lib.oomb_selftest_writeback_copy(ptr, n, bf, 0) == L.OK
    assert np.all(host[:n * bf] == 3.5) and np.all(host[n * bf:] == 2.5)
    assert lib.oomb_selftest_writeback_copy(None, n, bf, 0) == L.ERR_INVALID_ARG
