"""Drives the CUDA path chunk by chunk for the parity tests and smoke().

Only test infrastructure: builds the page table through the library's
allocator, appends each chunk, runs forward / backward through the C ABI and
hands back host copies of what the oracle is compared against.
"""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_chunk_query_b200 as pk


class PagedRun:
    def __init__(self, w, device="cuda", num_pages=None, alloc_seed=None, split_fwd=True):
        self.w = w
        self.dev = torch.device(device)
        # forward workspace: the last partial wave of (query tile, head) units is
        # split along its key tiles (every small test shape takes that path)
        self.fwd_ws = pk.fwd_workspace(w.head_dim, self.dev) if split_fwd else None
        self.num_pages = num_pages or w.num_pages
        seed = w.alloc_seed if alloc_seed is None else alloc_seed
        self.pool = pk.pool_create(self.num_pages, w.page_size, w.num_kv_heads, w.head_dim,
                                   pk.LOC_DEVICE, True, seed, self.dev.index or 0)
        self.page_table = []          # logical page -> physical id

    def close(self):
        if self.pool:
            pk.pool_destroy(self.pool)
            self.pool = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def append(self, k, v):
        n = k.shape[0] // self.w.page_size
        ids = [pk.pool_alloc_page(self.pool) for _ in range(n)]
        self.page_table += ids
        d_ids = torch.tensor(ids, dtype=torch.int32, device=self.dev)
        pk.kv_append(self.pool, d_ids, k.to(self.dev).contiguous(), v.to(self.dev).contiguous())
        return d_ids

    def past_lists(self, n_past, selected=None):
        """Device [Hkv][max_past] physical ids and counts; dense when selected is None."""
        Hkv = self.w.num_kv_heads
        if selected is None:
            if n_past == 0:
                return None, None
            ids = torch.tensor([self.page_table[:n_past]] * Hkv, dtype=torch.int32)
            cnt = torch.full((Hkv,), n_past, dtype=torch.int32)
        else:
            m = max(1, max(len(s) for s in selected))
            ids = torch.zeros((Hkv, m), dtype=torch.int32)
            cnt = torch.zeros((Hkv,), dtype=torch.int32)
            for g, sel in enumerate(selected):
                ids[g, :len(sel)] = torch.tensor([self.page_table[p] for p in sel], dtype=torch.int32)
                cnt[g] = len(sel)
        return ids.to(self.dev), cnt.to(self.dev)

    def chunk(self, c, inp, selected=None, backward=True):
        """Append chunk c, run fwd (and bwd) on it; returns device tensors."""
        w = self.w
        n_past = c * w.pages_per_chunk
        cur = self.append(inp["k"], inp["v"])
        past, counts = self.past_lists(n_past, selected)
        q = inp["q"].to(self.dev).contiguous()
        o = torch.empty_like(q)
        lse = torch.empty((w.num_q_heads, w.chunk_len), dtype=torch.float32, device=self.dev)
        pk.chunk_attn_fwd(self.pool, q, o, lse, past, counts, cur, w.softmax_scale,
                          fwd_ws=self.fwd_ws)
        out = {"o": o, "lse": lse, "cur": cur, "past": past, "counts": counts}
        if backward:
            do = inp["do"].to(self.dev).contiguous()
            dq = torch.empty_like(q)
            delta = torch.empty_like(lse)
            pk.chunk_attn_bwd(self.pool, q, o, lse, do, dq, delta, past, counts, cur,
                              w.softmax_scale)
            out["dq"] = dq
            out["delta"] = delta
        return out

    def grads_by_token(self, n_tokens):
        """Gradient pool gathered into [tokens][Hkv][d] (dK, dV) float64 numpy."""
        _, grad, _ = pk.pool_views(self.pool)
        P = self.w.page_size
        ids = torch.tensor(self.page_table[: n_tokens // P], dtype=torch.long, device=self.dev)
        g = grad[ids]                        # [pages][Hkv][2][P][d]
        g = g.permute(0, 3, 1, 2, 4).reshape(n_tokens, self.w.num_kv_heads, 2, self.w.head_dim)
        g = g.double().cpu().numpy()
        return g[:, :, 0, :], g[:, :, 1, :]

    def status(self):
        return pk.get_device_status(self.pool)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def to64(t):
    return t.detach().double().cpu().numpy()
