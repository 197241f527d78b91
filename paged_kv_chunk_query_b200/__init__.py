"""Paged chunk attention for NVIDIA B200 (sm_100a).

One chunk's queries attend to a paged KV cache holding every earlier chunk and
the chunk itself (causal); the backward adds dK/dV in place into a paged fp32
gradient pool; a page-level Top-K variant keeps the most relevant pages; pages
can live in pinned host memory and be prefetched on a side stream.  All
compute runs in hand-written CUDA kernels inside ``liboomb.so`` (C ABI in
``include/oomb.h``); this package only marshals arguments to it.
"""
from . import _lib
from ._lib import (BWD_DKDV, BWD_DQ, BWD_PREPROCESS, LOC_DEVICE, LOC_HOST, LOC_PINNED_HOST,
                   PROJ_KV, PROJ_Q, PROJ_QKV, SEG_FIRST, SEG_LAST, SEG_NEXT, SEG_WHOLE,
                   OombError, block_copy, chunk_attn_bwd, chunk_attn_fwd, chunk_attn_fwd_workspace_size,
                   fwd_workspace, get_device_status,
                   grad_block_add, grad_writeback, grad_writeback_sync, kv_append, local_pages, page_prefetch,
                   page_topk, page_topk_batched, page_topk_batched_workspace_size,
                   page_topk_qsum, page_topk_qsum_workspace_size, page_topk_workspace_size, pool_alloc_page, pool_buffers, pool_create,
                   pool_destroy, pool_free_page, pool_get_desc, pool_num_free, pool_views,
                   prefetch_lists, qkv_project, qpage_lists, status_string, version, wait)
from .synth import WORKLOADS, Workload

__all__ = [
    "OombError", "pool_create", "pool_destroy", "pool_alloc_page", "pool_free_page",
    "pool_num_free", "pool_buffers", "pool_get_desc", "pool_views", "kv_append",
    "chunk_attn_fwd", "chunk_attn_bwd", "page_topk", "page_topk_workspace_size",
    "page_topk_batched", "page_topk_batched_workspace_size", "page_prefetch", "grad_writeback",
    "grad_writeback_sync", "local_pages", "block_copy", "grad_block_add", "prefetch_lists", "wait",
    "get_device_status", "status_string", "version",
    "LOC_DEVICE", "LOC_PINNED_HOST", "LOC_HOST", "BWD_PREPROCESS", "BWD_DKDV", "BWD_DQ",
    "SEG_WHOLE", "SEG_FIRST", "SEG_NEXT", "SEG_LAST", "PROJ_Q", "PROJ_KV", "PROJ_QKV",
    "qkv_project", "qpage_lists", "page_topk_qsum", "page_topk_qsum_workspace_size",
    "chunk_attn_fwd_workspace_size", "fwd_workspace",
    "WORKLOADS", "Workload",
]
