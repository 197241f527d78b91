"""Seeded synthetic inputs for paged chunk attention.

This module only draws random numbers and rounds them to bf16; it holds none of
the attention, Top-K or paging arithmetic.  Both the CUDA path (through the
tests and ``bench.py``) and the CPU oracle receive the very bytes produced
here, so a parity test compares the two on identical inputs.

Workloads (one attention layer each):

* ``tiny``      Hq=4, Hkv=1, d=64, 16-token pages, 8 chunks of 64 (L=512), dense.
* ``qwen32k``   Hq=28, Hkv=4 (GQA 7:1), d=128, 64-token pages, 8 chunks of 4096,
                identity page table, dO ~ N(0, 1e-2^2), dense.
* ``qwen256k``  same shape, 64 chunks of 4096 (4096 pages), shuffled page table, dense.
* ``qwen256k_topk``  as ``qwen256k`` plus a per-(page, KV head) direction
                u ~ N(0, I_d) * 0.5 added to every key of the page; Top-64 pages
                plus the 2 most recent pages per chunk and KV-head group.
* ``qwen1m_topk_offload``  as ``qwen256k_topk`` with 256 chunks (16384 pages),
                past KV and gradients in pinned host memory.
* ``qwen256k_topk_qpage``  as ``qwen256k_topk`` with one selection per 64-token
                query page instead of per chunk.

Every draw is fp32 ``torch.randn`` from a CPU generator seeded per (workload
seed, chunk, tensor), then rounded to bf16 with round-to-nearest-even
(``Tensor.to(torch.bfloat16)``).  Drawing per chunk lets a test regenerate any
single chunk of a 256K or 1M workload without drawing the others.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_q_heads: int        # Hq
    num_kv_heads: int       # Hkv
    head_dim: int           # d
    page_size: int          # P, tokens per page
    chunk_len: int          # C, tokens per chunk
    num_chunks: int         # N
    seed: int
    do_std: float = 1.0
    shuffle_pages: bool = False
    page_direction: float = 0.0   # scale of the per-page key direction (0: none)
    top_k: int = 0                # 0: dense
    n_recent: int = 0
    host_resident: bool = False   # past KV and grads in pinned host memory
    window: int = 0               # > 0: recent-only lists of this many past pages
    qtile_topk: bool = False      # Top-K per 128-row query tile instead of per chunk
    qpage_topk: bool = False      # Top-K per query page (page_size rows) instead of per chunk

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def context(self) -> int:
        return self.chunk_len * self.num_chunks

    @property
    def num_pages(self) -> int:
        return self.context // self.page_size

    @property
    def pages_per_chunk(self) -> int:
        return self.chunk_len // self.page_size

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def alloc_seed(self) -> int:
        return self.seed if self.shuffle_pages else 0


WORKLOADS = {
    "tiny": Workload("tiny", 4, 1, 64, 16, 64, 8, seed=1000),
    "qwen32k": Workload("qwen32k", 28, 4, 128, 64, 4096, 8, seed=1001, do_std=1e-2),
    # profiling-sized sparse case (not a headline configuration)
    "qwen32k_topk": Workload("qwen32k_topk", 28, 4, 128, 64, 4096, 8, seed=1005,
                             shuffle_pages=True, page_direction=0.5, top_k=64, n_recent=2),
    "qwen256k": Workload("qwen256k", 28, 4, 128, 64, 4096, 64, seed=1002,
                         shuffle_pages=True),
    "qwen256k_topk": Workload("qwen256k_topk", 28, 4, 128, 64, 4096, 64, seed=1003,
                              shuffle_pages=True, page_direction=0.5, top_k=64,
                              n_recent=2),
    # one Top-K selection per 128-row query tile (two 64-token query pages share one list)
    "qwen256k_topk_qtile": Workload("qwen256k_topk_qtile", 28, 4, 128, 64, 4096, 64, seed=1007,
                                    shuffle_pages=True, page_direction=0.5, top_k=64,
                                    n_recent=2, qtile_topk=True),
    # one Top-K selection per 64-token query page (per-query-page sparsity)
    "qwen256k_topk_qpage": Workload("qwen256k_topk_qpage", 28, 4, 128, 64, 4096, 64, seed=1008,
                                    shuffle_pages=True, page_direction=0.5, top_k=64,
                                    n_recent=2, qpage_topk=True),
    # recent-only page lists: the last 64 past pages (4096 tokens) + the chunk
    "qwen256k_local": Workload("qwen256k_local", 28, 4, 128, 64, 4096, 64, seed=1006,
                               shuffle_pages=True, window=64),
    "qwen1m_topk_offload": Workload("qwen1m_topk_offload", 28, 4, 128, 64, 4096, 256,
                                    seed=1004, shuffle_pages=True, page_direction=0.5,
                                    top_k=64, n_recent=2, host_resident=True),
}


def _generator(seed: int, chunk: int, stream: int) -> torch.Generator:
    # A plain injective mix of three small non-negative integers into one seed.
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + chunk * 16 + stream) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _randn(shape, gen) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def chunk_inputs(w: Workload, c: int, which=("q", "k", "v", "do")) -> dict[str, torch.Tensor]:
    """Q, K, V, dO of chunk ``c`` as bf16 CPU tensors (only those named in
    ``which``; each tensor has its own generator, so skipping some does not
    change the others).

    Layouts: q, do ``[C][Hq][d]``; k, v ``[C][Hkv][d]`` (token-major, as a
    projection would write them).
    """
    C, Hq, Hkv, d, P = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size
    out = {}
    if "q" in which:
        out["q"] = _randn((C, Hq, d), _generator(w.seed, c, 0)).to(torch.bfloat16)
    if "k" in which:
        k = _randn((C, Hkv, d), _generator(w.seed, c, 1))
        if w.page_direction:
            u = _randn((C // P, Hkv, d), _generator(w.seed, c, 4)) * w.page_direction
            k = k + u.repeat_interleave(P, dim=0)
        out["k"] = k.to(torch.bfloat16)
    if "v" in which:
        out["v"] = _randn((C, Hkv, d), _generator(w.seed, c, 2)).to(torch.bfloat16)
    if "do" in which:
        out["do"] = (_randn((C, Hq, d), _generator(w.seed, c, 3)) * w.do_std).to(torch.bfloat16)
    return out


def sequence_inputs(w: Workload) -> dict[str, torch.Tensor]:
    """All chunks concatenated along the token axis (small workloads only)."""
    parts = [chunk_inputs(w, c) for c in range(w.num_chunks)]
    return {key: torch.cat([p[key] for p in parts], dim=0) for key in parts[0]}


def device_chunk_inputs(w: Workload, c: int, device) -> dict[str, torch.Tensor]:
    """Same shapes and distributions as :func:`chunk_inputs`, drawn directly on
    the device (for throughput runs, where the host draw would dominate).  The
    values differ from the CPU draw; parity runs use :func:`chunk_inputs`."""
    C, Hq, Hkv, d, P = w.chunk_len, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size
    g = torch.Generator(device=device)
    g.manual_seed((w.seed * 1_000_003 + c * 16 + 7) & 0x7FFF_FFFF_FFFF_FFFF)
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    q = torch.randn((C, Hq, d), **f32)
    k = torch.randn((C, Hkv, d), **f32)
    v = torch.randn((C, Hkv, d), **f32)
    do = torch.randn((C, Hq, d), **f32) * w.do_std
    if w.page_direction:
        u = torch.randn((C // P, Hkv, d), **f32) * w.page_direction
        k = k + u.repeat_interleave(P, dim=0)
    return {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16),
            "v": v.to(torch.bfloat16), "do": do.to(torch.bfloat16)}
