"""The Q/K/V projection of a chunk, fp64 (test infrastructure only).

The pages: for sparse attention the ids of the pages a chunk needs are known
as soon as its queries exist, so their transfer can overlap the rest of the
chunk's work ([pt] §2D; [es] §2B, KV offloaded).  The work they overlap with
in a transformer layer is the projection that produces K and V:

  Q = X W_q^T,  K = X W_k^T,  V = X W_v^T

with X ``[C][hidden]`` and the weight rows stacked as [W_q; W_k; W_v]
(``num_q_heads * d`` rows, then ``num_kv_heads * d``, then ``num_kv_heads * d``).
A matrix product is used as the library primitive; nothing else is done.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64


def qkv_projection(x, w, num_q_heads, num_kv_heads, head_dim):
    """Returns Q ``[C][Hq][d]``, K and V ``[C][Hkv][d]`` in fp64."""
    x, w = _f64(x), _f64(w)
    y = x @ w.T
    nq, nk = num_q_heads * head_dim, num_kv_heads * head_dim
    C = x.shape[0]
    q = y[:, :nq].reshape(C, num_q_heads, head_dim)
    k = y[:, nq:nq + nk].reshape(C, num_kv_heads, head_dim)
    v = y[:, nq + nk:nq + 2 * nk].reshape(C, num_kv_heads, head_dim)
    return q, k, v
