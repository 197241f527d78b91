"""ctypes binding of liboomb.so: argument marshalling only.

Every function here forwards to the C ABI declared in include/oomb.h, taking
torch tensors for device buffers (their data pointers are passed) and raising
:class:`OombError` on a non-OK status.  No step of the computation runs here;
if the shared library is missing or fails to load, importing the package fails
loudly — there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboomb.so")

STATUS = {
    0: "OOMB_OK", 1: "OOMB_ERR_INVALID_ARG", 2: "OOMB_ERR_OUT_OF_PAGES", 3: "OOMB_ERR_BAD_PAGE",
    4: "OOMB_ERR_CUDA", 5: "OOMB_ERR_TIMEOUT", 6: "OOMB_ERR_UNSUPPORTED",
    7: "OOMB_ERR_DEVICE_CHECK",
}
OK, ERR_INVALID_ARG, ERR_OUT_OF_PAGES, ERR_BAD_PAGE, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED, \
    ERR_DEVICE_CHECK = range(8)
LOC_DEVICE, LOC_PINNED_HOST, LOC_HOST = 0, 1, 2
BWD_PREPROCESS, BWD_DKDV, BWD_DQ = 0, 1, 2
SEG_WHOLE, SEG_FIRST, SEG_NEXT, SEG_LAST = 0, 1, 2, 3
PROJ_Q, PROJ_KV, PROJ_QKV = 0, 1, 2

# Every exported symbol of include/oomb.h.
EXPORTS = (
    "oomb_pool_create", "oomb_pool_destroy", "oomb_pool_alloc_page", "oomb_pool_free_page",
    "oomb_pool_num_free", "oomb_pool_buffers", "oomb_pool_get_desc", "oomb_kv_append",
    "oomb_chunk_attn_fwd", "oomb_chunk_attn_bwd", "oomb_chunk_attn_bwd_step",
    "oomb_page_topk_workspace_size", "oomb_page_topk", "oomb_page_prefetch",
    "oomb_grad_writeback", "oomb_wait", "oomb_get_device_status", "oomb_status_string",
    "oomb_version", "oomb_page_topk_static", "oomb_grad_writeback_sync",
    "oomb_selftest_wait_limit", "oomb_page_topk_batched_workspace_size", "oomb_page_topk_batched",
    "oomb_block_copy", "oomb_grad_block_add", "oomb_prefetch_lists", "oomb_local_pages",
    "oomb_qkv_project", "oomb_selftest_writeback_copy", "oomb_qpage_lists",
    "oomb_page_topk_qsum_workspace_size", "oomb_page_topk_qsum",
    "oomb_chunk_attn_fwd_workspace_size",
)


class OombError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class PoolDesc(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("location", ctypes.c_int32), ("with_grad", ctypes.c_int32),
                ("alloc_seed", ctypes.c_uint64), ("device", ctypes.c_int32)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("d_o", ctypes.c_void_p), ("dq", ctypes.c_void_p),
                ("delta_ws", ctypes.c_void_p), ("chunk_len", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("past_pages", ctypes.c_void_p),
                ("past_counts", ctypes.c_void_p), ("max_past", ctypes.c_int32),
                ("cur_pages", ctypes.c_void_p), ("softmax_scale", ctypes.c_float),
                ("lists_per_qtile", ctypes.c_int32), ("segment", ctypes.c_int32),
                ("o_acc", ctypes.c_void_p), ("dq_acc", ctypes.c_void_p),
                ("past_masks", ctypes.c_void_p), ("fwd_ws", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m paged_kv_chunk_query_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    sig = {
        "oomb_pool_create": [ctypes.POINTER(PoolDesc), ctypes.POINTER(vp)],
        "oomb_pool_destroy": [vp],
        "oomb_pool_alloc_page": [vp, ctypes.POINTER(i32)],
        "oomb_pool_free_page": [vp, i32],
        "oomb_pool_num_free": [vp, ctypes.POINTER(i32)],
        "oomb_pool_buffers": [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp)],
        "oomb_pool_get_desc": [vp, ctypes.POINTER(PoolDesc)],
        "oomb_kv_append": [vp, vp, i32, vp, vp, vp],
        "oomb_chunk_attn_fwd": [vp, ctypes.POINTER(AttnArgs), vp],
        "oomb_chunk_attn_bwd": [vp, ctypes.POINTER(AttnArgs), vp],
        "oomb_chunk_attn_bwd_step": [vp, ctypes.POINTER(AttnArgs), i32, vp],
        "oomb_page_topk": [vp, vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp, vp,
                           ctypes.c_size_t, vp],
        "oomb_page_topk_static": [vp, vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp, vp],
        "oomb_page_topk_qsum": [vp, vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp, vp,
                                ctypes.c_size_t, vp],
        "oomb_page_prefetch": [vp, vp, vp, vp, i32, vp, vp],
        "oomb_grad_writeback": [vp, vp, vp, vp, i32, vp],
        "oomb_grad_writeback_sync": [vp, ctypes.c_int64],
        "oomb_wait": [vp, ctypes.c_int64],
        "oomb_get_device_status": [vp, ctypes.POINTER(ctypes.c_uint32)],
        "oomb_selftest_wait_limit": [vp, vp],
        "oomb_page_topk_batched": [vp, vp, i32, i32, i32, vp, i32, vp, i32, vp, i32, i32, vp, vp,
                                   vp, vp, vp, ctypes.c_size_t, vp],
        "oomb_block_copy": [vp, vp, vp, vp, i32, vp],
        "oomb_grad_block_add": [vp, vp, vp, vp, i32, i32, vp],
        "oomb_prefetch_lists": [vp, vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, vp],
        "oomb_local_pages": [vp, vp, i32, i32, vp, vp, vp],
        "oomb_qkv_project": [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp],
        "oomb_selftest_writeback_copy": [vp, i32, i32, i32],
        "oomb_qpage_lists": [vp, vp, vp, vp, i32, i32, vp, vp, vp, i32, vp],
    }
    for name, args in sig.items():
        if not hasattr(lib, name):  # completeness is checked by the export test
            continue
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    if hasattr(lib, "oomb_page_topk_workspace_size"):
        lib.oomb_page_topk_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        lib.oomb_page_topk_workspace_size.restype = ctypes.c_size_t
    if hasattr(lib, "oomb_page_topk_qsum_workspace_size"):
        lib.oomb_page_topk_qsum_workspace_size.argtypes = [i32, i32]
        lib.oomb_page_topk_qsum_workspace_size.restype = ctypes.c_size_t
    if hasattr(lib, "oomb_chunk_attn_fwd_workspace_size"):
        lib.oomb_chunk_attn_fwd_workspace_size.argtypes = [i32]
        lib.oomb_chunk_attn_fwd_workspace_size.restype = ctypes.c_size_t
    if hasattr(lib, "oomb_page_topk_batched_workspace_size"):
        lib.oomb_page_topk_batched_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.oomb_page_topk_batched_workspace_size.restype = ctypes.c_size_t
    lib.oomb_status_string.argtypes = [ctypes.c_int]
    lib.oomb_status_string.restype = ctypes.c_char_p
    lib.oomb_version.argtypes = []
    lib.oomb_version.restype = i32
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != OK:
        raise OombError(status, where)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dev_tensor(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# ------------------------------------------------------------------- pools
def pool_create(num_pages, page_size, num_kv_heads, head_dim, location=LOC_DEVICE,
                with_grad=True, alloc_seed=0, device=0) -> int:
    d = PoolDesc(num_pages, page_size, num_kv_heads, head_dim, location, int(bool(with_grad)),
                 alloc_seed, device)
    h = ctypes.c_void_p()
    _check(load().oomb_pool_create(ctypes.byref(d), ctypes.byref(h)), "oomb_pool_create")
    return h.value


def pool_destroy(pool: int):
    _check(load().oomb_pool_destroy(pool), "oomb_pool_destroy")


def pool_alloc_page(pool: int) -> int:
    out = ctypes.c_int32()
    _check(load().oomb_pool_alloc_page(pool, ctypes.byref(out)), "oomb_pool_alloc_page")
    return out.value


def pool_free_page(pool: int, page_id: int):
    _check(load().oomb_pool_free_page(pool, page_id), "oomb_pool_free_page")


def pool_num_free(pool: int) -> int:
    out = ctypes.c_int32()
    _check(load().oomb_pool_num_free(pool, ctypes.byref(out)), "oomb_pool_num_free")
    return out.value


def pool_get_desc(pool: int) -> PoolDesc:
    d = PoolDesc()
    _check(load().oomb_pool_get_desc(pool, ctypes.byref(d)), "oomb_pool_get_desc")
    return d


def pool_buffers(pool: int):
    """(kv, grad, summary) raw pointers (0 where absent)."""
    kv, grad, summ = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    _check(load().oomb_pool_buffers(pool, ctypes.byref(kv), ctypes.byref(grad),
                                    ctypes.byref(summ)), "oomb_pool_buffers")
    return kv.value or 0, grad.value or 0, summ.value or 0


class _CudaArray:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": tuple(shape),
                                         "typestr": typestr, "version": 3, "strides": None}


def pool_views(pool: int):
    """Torch views (kv, grad, summary) of a pool's buffers, borrowed: valid until
    pool_destroy.  Device pools give CUDA tensors; pinned-host pools give CPU
    tensors for kv and grad and a CUDA tensor for the summaries (which the
    library keeps on the device); host pools give CPU tensors."""
    d = pool_get_desc(pool)
    kv, grad, summ = pool_buffers(pool)
    shape = (d.num_pages, d.num_kv_heads, 2, d.page_size, d.head_dim)
    sshape = (d.num_pages, d.num_kv_heads, d.head_dim)
    dev = torch.device("cuda", d.device)

    def host(ptr, shp, ctype, dt):
        n = 1
        for x in shp:
            n *= x
        buf = (ctype * n).from_address(ptr)
        return torch.frombuffer(buf, dtype=dt).view(shp)

    if d.location == LOC_DEVICE:
        t_kv = torch.as_tensor(_CudaArray(kv, shape, "<i2"), device=dev).view(torch.bfloat16)
        t_g = torch.as_tensor(_CudaArray(grad, shape, "<f4"), device=dev) if grad else None
        t_s = torch.as_tensor(_CudaArray(summ, sshape, "<f4"), device=dev)
        return t_kv, t_g, t_s
    t_kv = host(kv, shape, ctypes.c_int16, torch.int16).view(torch.bfloat16)
    t_g = host(grad, shape, ctypes.c_float, torch.float32) if grad else None
    if d.location == LOC_PINNED_HOST:
        t_s = torch.as_tensor(_CudaArray(summ, sshape, "<f4"), device=dev)
    else:
        t_s = host(summ, sshape, ctypes.c_float, torch.float32)
    return t_kv, t_g, t_s


def _event_handle(event, stream):
    """Raw cudaEvent_t of a torch.cuda.Event.  torch creates the CUDA event on
    its first record, so an event never recorded is recorded once here to
    exist (the library records it again after its own work)."""
    if event is None:
        return None
    if not event.cuda_event:
        event.record(stream if isinstance(stream, torch.cuda.Stream)
                     else torch.cuda.current_stream())
    return event.cuda_event


# ------------------------------------------------------------------- compute
def kv_append(pool: int, page_ids: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None):
    n = page_ids.numel()
    _check(load().oomb_kv_append(pool, _dev_tensor(page_ids, torch.int32, "page_ids"), n,
                                 _dev_tensor(k, torch.bfloat16, "k"),
                                 _dev_tensor(v, torch.bfloat16, "v"), _stream(stream)),
           "oomb_kv_append")


def _attn_args(q, o, lse, past_pages, past_counts, cur_pages, softmax_scale, d_o=None, dq=None,
               delta_ws=None, segment=SEG_WHOLE, o_acc=None, dq_acc=None, past_masks=None,
               fwd_ws=None):
    """past_pages [Hkv][max_past] (one list per group) or [n_qtiles][Hkv][max_past]
    (one list per 128-row query tile and group; counts [n_qtiles][Hkv]); with
    past_masks (uint8, layout of past_pages) the per-tile lists are unions of
    per-query-page lists (oomb_qpage_lists)."""
    C, Hq, _ = q.shape
    per_qtile = past_pages is not None and past_pages.dim() == 3
    max_past = past_pages.shape[-1] if past_pages is not None and past_pages.numel() else 0
    if past_masks is not None and not per_qtile:
        raise ValueError("past_masks need per-query-tile past_pages [n_qtiles][Hkv][max_past]")
    if per_qtile and max_past:
        n_qt = (C + 127) // 128
        if past_pages.shape[0] != n_qt or past_counts is None or \
                tuple(past_counts.shape) != tuple(past_pages.shape[:2]):
            raise ValueError(f"per-query-tile lists need past_pages [{n_qt}][Hkv][max_past] and "
                             f"past_counts [{n_qt}][Hkv]")
        if past_masks is not None and tuple(past_masks.shape) != tuple(past_pages.shape):
            raise ValueError("past_masks must have the shape of past_pages")
    mode = (2 if past_masks is not None else 1) if per_qtile else 0
    return AttnArgs(
        _dev_tensor(q, torch.bfloat16, "q"), _dev_tensor(o, torch.bfloat16, "o"),
        _dev_tensor(lse, torch.float32, "lse"),
        _dev_tensor(d_o, torch.bfloat16, "d_o") if d_o is not None else None,
        _dev_tensor(dq, torch.bfloat16, "dq") if dq is not None else None,
        _dev_tensor(delta_ws, torch.float32, "delta_ws") if delta_ws is not None else None,
        C, Hq,
        _dev_tensor(past_pages, torch.int32, "past_pages") if max_past else None,
        _dev_tensor(past_counts, torch.int32, "past_counts") if max_past else None,
        max_past, _dev_tensor(cur_pages, torch.int32, "cur_pages"), softmax_scale,
        mode, segment,
        _dev_tensor(o_acc, torch.float32, "o_acc") if o_acc is not None else None,
        _dev_tensor(dq_acc, torch.float32, "dq_acc") if dq_acc is not None else None,
        _dev_tensor(past_masks, torch.uint8, "past_masks") if past_masks is not None and max_past
        else None,
        _dev_tensor(fwd_ws, torch.float32, "fwd_ws") if fwd_ws is not None else None)


def chunk_attn_fwd(pool, q, o, lse, past_pages, past_counts, cur_pages, softmax_scale,
                   stream=None, segment=SEG_WHOLE, o_acc=None, past_masks=None, fwd_ws=None):
    """fwd_ws: optional fp32 device workspace of chunk_attn_fwd_workspace_size(d) bytes
    (see fwd_workspace); with it the last partial wave of units is split along its key
    tiles and merged by a second launch."""
    a = _attn_args(q, o, lse, past_pages, past_counts, cur_pages, softmax_scale,
                   segment=segment, o_acc=o_acc, past_masks=past_masks, fwd_ws=fwd_ws)
    _check(load().oomb_chunk_attn_fwd(pool, ctypes.byref(a), _stream(stream)),
           "oomb_chunk_attn_fwd")


def chunk_attn_fwd_workspace_size(head_dim) -> int:
    return load().oomb_chunk_attn_fwd_workspace_size(head_dim)


def fwd_workspace(head_dim, device) -> torch.Tensor:
    """A forward workspace (fp32, zero-initialised) for chunk_attn_fwd's fwd_ws."""
    n = chunk_attn_fwd_workspace_size(head_dim)
    if n == 0:
        raise ValueError(f"no forward workspace for head_dim {head_dim}")
    return torch.zeros(n // 4, dtype=torch.float32, device=device)


def chunk_attn_bwd(pool, q, o, lse, d_o, dq, delta_ws, past_pages, past_counts, cur_pages,
                   softmax_scale, stream=None, step=None, segment=SEG_WHOLE, o_acc=None,
                   dq_acc=None, past_masks=None):
    a = _attn_args(q, o, lse, past_pages, past_counts, cur_pages, softmax_scale, d_o, dq,
                   delta_ws, segment=segment, o_acc=o_acc, dq_acc=dq_acc, past_masks=past_masks)
    if step is None:
        _check(load().oomb_chunk_attn_bwd(pool, ctypes.byref(a), _stream(stream)),
               "oomb_chunk_attn_bwd")
    else:
        _check(load().oomb_chunk_attn_bwd_step(pool, ctypes.byref(a), step, _stream(stream)),
               "oomb_chunk_attn_bwd_step")


def page_topk_workspace_size(chunk_len, num_q_heads, num_kv_heads, head_dim, n_past) -> int:
    return load().oomb_page_topk_workspace_size(chunk_len, num_q_heads, num_kv_heads, head_dim,
                                                n_past)


def page_topk(pool, q, page_table, n_past, top_k, n_recent, out_logical, out_physical,
              out_count, workspace, out_scores=None, stream=None):
    C, Hq, _ = q.shape
    _check(load().oomb_page_topk(
        pool, _dev_tensor(q, torch.bfloat16, "q"), C, Hq,
        _dev_tensor(page_table, torch.int32, "page_table") if n_past else None, n_past, top_k,
        n_recent, _dev_tensor(out_logical, torch.int32, "out_logical"),
        _dev_tensor(out_physical, torch.int32, "out_physical") if out_physical is not None
        else None, _dev_tensor(out_count, torch.int32, "out_count"),
        _dev_tensor(out_scores, torch.float32, "out_scores") if out_scores is not None else None,
        _dev_tensor(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "oomb_page_topk")


def page_topk_qsum_workspace_size(num_kv_heads, n_past) -> int:
    return load().oomb_page_topk_qsum_workspace_size(num_kv_heads, n_past)


def page_topk_qsum(pool, qsum, chunk_len, num_q_heads, page_table, n_past, top_k, n_recent,
                   out_logical, out_physical, out_count, workspace, out_scores=None, stream=None):
    """oomb_page_topk_qsum: the selection from per-group sums of Q ([Hkv][d]
    fp32, e.g. qkv_project's qsum).  The workspace's counters must be zero
    before its first use (torch.zeros); each call leaves them at zero."""
    _check(load().oomb_page_topk_qsum(
        pool, _dev_tensor(qsum, torch.float32, "qsum"), chunk_len, num_q_heads,
        _dev_tensor(page_table, torch.int32, "page_table") if n_past else None, n_past, top_k,
        n_recent, _dev_tensor(out_logical, torch.int32, "out_logical"),
        _dev_tensor(out_physical, torch.int32, "out_physical") if out_physical is not None
        else None, _dev_tensor(out_count, torch.int32, "out_count"),
        _dev_tensor(out_scores, torch.float32, "out_scores") if out_scores is not None else None,
        _dev_tensor(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "oomb_page_topk_qsum")


def page_topk_batched_workspace_size(n_problems, num_kv_heads, head_dim, max_past) -> int:
    return load().oomb_page_topk_batched_workspace_size(n_problems, num_kv_heads, head_dim,
                                                        max_past)


def page_topk_batched(pool, q, row_start, max_rows, n_past, max_past, page_table, top_k,
                      n_recent, out_logical, out_physical, out_count, workspace,
                      out_scores=None, stream=None):
    """oomb_page_topk_batched: one selection per problem b (query rows
    row_start[b]:row_start[b+1] of q, candidates among the first n_past[b]
    logical pages of page_table); outputs [B][Hkv][K+R] / [B][Hkv]."""
    T, Hq, _ = q.shape
    B = n_past.numel()
    _check(load().oomb_page_topk_batched(
        pool, _dev_tensor(q, torch.bfloat16, "q"), T, Hq, B,
        _dev_tensor(row_start, torch.int32, "row_start"), max_rows,
        _dev_tensor(n_past, torch.int32, "n_past"), max_past,
        _dev_tensor(page_table, torch.int32, "page_table") if max_past else None, top_k, n_recent,
        _dev_tensor(out_logical, torch.int32, "out_logical"),
        _dev_tensor(out_physical, torch.int32, "out_physical") if out_physical is not None
        else None, _dev_tensor(out_count, torch.int32, "out_count"),
        _dev_tensor(out_scores, torch.float32, "out_scores") if out_scores is not None else None,
        _dev_tensor(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "oomb_page_topk_batched")


def qpage_lists(pool, sel_logical, sel_physical, sel_count, chunk_len, out_pages, out_masks,
                out_count, stream=None):
    """oomb_qpage_lists: per-query-page selections [n_qpages][Hkv][max_sel] ->
    per-query-tile union lists [n_qtiles][Hkv][max_union] (physical ids), their
    membership masks (uint8) and counts [n_qtiles][Hkv]."""
    _check(load().oomb_qpage_lists(
        pool, _dev_tensor(sel_logical, torch.int32, "sel_logical"),
        _dev_tensor(sel_physical, torch.int32, "sel_physical"),
        _dev_tensor(sel_count, torch.int32, "sel_count"), chunk_len, sel_logical.shape[-1],
        _dev_tensor(out_pages, torch.int32, "out_pages"),
        _dev_tensor(out_masks, torch.uint8, "out_masks"),
        _dev_tensor(out_count, torch.int32, "out_count"), out_pages.shape[-1], _stream(stream)),
        "oomb_qpage_lists")


def local_pages(pool, page_table, n_past, out_pages, out_count, stream=None):
    """oomb_local_pages: the last window = out_pages.shape[1] past pages of every
    group (physical ids, ascending) and their counts."""
    window = out_pages.shape[1]
    _check(load().oomb_local_pages(
        pool, _dev_tensor(page_table, torch.int32, "page_table") if n_past else None, n_past,
        window, _dev_tensor(out_pages, torch.int32, "out_pages"),
        _dev_tensor(out_count, torch.int32, "out_count"), _stream(stream)), "oomb_local_pages")


def qkv_project(pool, x, w, num_q_heads, part, q=None, qsum=None, page_ids=None, stream=None):
    """oomb_qkv_project: x [C][hidden] bf16, w [(Hq + 2 Hkv) d][hidden] bf16;
    part PROJ_Q (q and/or qsum), PROJ_KV (K/V into the pages page_ids, page
    means, zeroed gradients) or PROJ_QKV."""
    C, hidden = x.shape
    _check(load().oomb_qkv_project(
        pool, _dev_tensor(x, torch.bfloat16, "x"), _dev_tensor(w, torch.bfloat16, "w"), C, hidden,
        num_q_heads, part, _dev_tensor(q, torch.bfloat16, "q") if q is not None else None,
        _dev_tensor(qsum, torch.float32, "qsum") if qsum is not None else None,
        _dev_tensor(page_ids, torch.int32, "page_ids") if page_ids is not None else None,
        _stream(stream)), "oomb_qkv_project")


TOPK_STATIC_SCRATCH_BYTES = 1 << 20


def page_topk_static(pool, q, page_table, n_past, top_k, n_recent, out_logical, out_physical,
                     out_count, out_scores=None, stream=None):
    """oomb_page_topk_static: Top-K with the library's static scratch (no
    workspace argument; allocates nothing)."""
    C, Hq, _ = q.shape
    _check(load().oomb_page_topk_static(
        pool, _dev_tensor(q, torch.bfloat16, "q"), C, Hq,
        _dev_tensor(page_table, torch.int32, "page_table") if n_past else None, n_past, top_k,
        n_recent, _dev_tensor(out_logical, torch.int32, "out_logical"),
        _dev_tensor(out_physical, torch.int32, "out_physical") if out_physical is not None
        else None, _dev_tensor(out_count, torch.int32, "out_count"),
        _dev_tensor(out_scores, torch.float32, "out_scores") if out_scores is not None else None,
        _stream(stream)), "oomb_page_topk_static")


def _host_i32(blocks):
    """A host int32 copy of a block list (list, array or tensor, on any device)
    and its pointer; the C side reads these lists on the host."""
    if isinstance(blocks, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(blocks, dtype=np.int32))
    else:
        t = torch.as_tensor(blocks, dtype=torch.int32).cpu().contiguous()
    return t, t.data_ptr()


def page_prefetch(host_pool, device_pool, src_blocks, dst_blocks, stream=None, done_event=None):
    s, sp = _host_i32(src_blocks)
    d, dp = _host_i32(dst_blocks)  # d keeps the array behind dp alive
    if d.numel() != s.numel():
        raise ValueError("src_blocks and dst_blocks must have the same length")
    ev = _event_handle(done_event, stream)
    _check(load().oomb_page_prefetch(host_pool, device_pool, sp, dp, s.numel(), _stream(stream),
                                     ev), "oomb_page_prefetch")


def grad_writeback(device_pool, host_pool, src_blocks, dst_blocks, stream=None):
    s, sp = _host_i32(src_blocks)
    d, dp = _host_i32(dst_blocks)  # d keeps the array behind dp alive
    if d.numel() != s.numel():
        raise ValueError("src_blocks and dst_blocks must have the same length")
    _check(load().oomb_grad_writeback(device_pool, host_pool, sp, dp, s.numel(),
                                      _stream(stream)), "oomb_grad_writeback")


def grad_writeback_sync(device_pool, timeout_us: int = 120_000_000):
    _check(load().oomb_grad_writeback_sync(device_pool, timeout_us), "oomb_grad_writeback_sync")


def block_copy(src_pool, dst_pool, src_blocks, dst_blocks, stream=None):
    """oomb_block_copy with block lists in device memory (int32 CUDA tensors)."""
    n = src_blocks.numel()
    if dst_blocks.numel() != n:
        raise ValueError("src_blocks and dst_blocks differ in length")
    _check(load().oomb_block_copy(src_pool, dst_pool,
                                  _dev_tensor(src_blocks, torch.int32, "src_blocks"),
                                  _dev_tensor(dst_blocks, torch.int32, "dst_blocks"), n,
                                  _stream(stream)), "oomb_block_copy")


def grad_block_add(src_pool, dst_pool, src_blocks, dst_blocks, zero_src=True, stream=None):
    """oomb_grad_block_add with block lists in device memory."""
    n = src_blocks.numel()
    if dst_blocks.numel() != n:
        raise ValueError("src_blocks and dst_blocks differ in length")
    _check(load().oomb_grad_block_add(src_pool, dst_pool,
                                      _dev_tensor(src_blocks, torch.int32, "src_blocks"),
                                      _dev_tensor(dst_blocks, torch.int32, "dst_blocks"), n,
                                      int(bool(zero_src)), _stream(stream)),
           "oomb_grad_block_add")


def prefetch_lists(src_pool, dst_pool, sel_logical, sel_count, page_table, slot_pages,
                   out_src_blocks, out_dst_blocks, out_past_pages, stream=None):
    """oomb_prefetch_lists: selection [Hkv][max_sel] -> slot-major block lists
    [max_sel * Hkv] and the staging past-page list [Hkv][max_sel]."""
    max_sel = sel_logical.shape[1]
    _check(load().oomb_prefetch_lists(
        src_pool, dst_pool, _dev_tensor(sel_logical, torch.int32, "sel_logical"),
        _dev_tensor(sel_count, torch.int32, "sel_count"), max_sel,
        _dev_tensor(page_table, torch.int32, "page_table") if page_table.numel() else None,
        page_table.numel(), _dev_tensor(slot_pages, torch.int32, "slot_pages"),
        _dev_tensor(out_src_blocks, torch.int32, "out_src_blocks"),
        _dev_tensor(out_dst_blocks, torch.int32, "out_dst_blocks"),
        _dev_tensor(out_past_pages, torch.int32, "out_past_pages"), _stream(stream)),
        "oomb_prefetch_lists")


def wait(event, timeout_us: int):
    _check(load().oomb_wait(event.cuda_event or None, timeout_us), "oomb_wait")


def get_device_status(pool) -> int:
    w = ctypes.c_uint32()
    st = load().oomb_get_device_status(pool, ctypes.byref(w))
    if st not in (OK, ERR_DEVICE_CHECK):
        raise OombError(st, "oomb_get_device_status")
    return w.value


def selftest_wait_limit(pool, stream=None):
    _check(load().oomb_selftest_wait_limit(pool, _stream(stream)), "oomb_selftest_wait_limit")


def status_string(status: int) -> str:
    return load().oomb_status_string(status).decode()


def version() -> int:
    return load().oomb_version()
