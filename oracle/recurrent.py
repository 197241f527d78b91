"""The chunk-recurrent loop over a whole sequence, fp64, contiguous KV.

The pages split the sequence into chunks processed one after another, with
activations dropped after the forward and recomputed for the backward ([pt]
§2A; [es] §2A; [it] §2A).  Chunk c's rows attend to every earlier token (or,
page-sparse, to the tokens of the pages kept for the chunk and group) and
causally to the chunk itself.  Gradients of the keys and values of every chunk
are summed over all later chunks, in place ([pt] §2B; [it] §2B), so the order
in which chunk backwards run does not change the sums.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, chunk_backward, chunk_forward
from .sparse import topk_for_chunk


def run_sequence(q, k, v, do, chunk_len, page_size, scale, top_k=0, n_recent=0,
                 with_backward=True, selections=None):
    """Forward (and backward) of every chunk of a sequence.

    q, do ``[L][Hq][d]``; k, v ``[L][Hkv][d]``.  ``top_k == 0`` means dense.
    ``selections`` may give, per chunk, the kept logical page lists per group
    (to evaluate attention on a selection made elsewhere); otherwise the
    oracle's own Top-K is used.

    Returns a dict with o, lse ``[Hq][L]``, dq, dk, dv (dk/dv summed over all
    chunks) and ``selected`` (per chunk, per group, ascending page ids; None
    for dense).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    L, Hq, d = q.shape
    Hkv = k.shape[1]
    N = L // chunk_len
    o = np.zeros((L, Hq, v.shape[2]))
    lse = np.zeros((Hq, L))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    selected = []
    for c in range(N):
        a, b = c * chunk_len, (c + 1) * chunk_len
        if top_k == 0 and selections is None:
            tok = [np.arange(a) for _ in range(Hkv)]
            selected.append(None)
        else:
            if selections is not None:
                sel = selections[c]
            else:
                sel, _ = topk_for_chunk(q[a:b], k[:a], page_size, top_k, n_recent)
            selected.append(sel)
            tok = [np.concatenate([np.arange(p * page_size, (p + 1) * page_size)
                                   for p in sel[g]]).astype(np.int64)
                   if len(sel[g]) else np.zeros(0, dtype=np.int64)
                   for g in range(Hkv)]
        kp = [k[tok[g], g, :] for g in range(Hkv)]
        vp = [v[tok[g], g, :] for g in range(Hkv)]
        o_c, lse_c = chunk_forward(q[a:b], kp, vp, k[a:b], v[a:b], scale)
        o[a:b], lse[:, a:b] = o_c, lse_c
        if with_backward:
            dq_c, dkp, dvp, dkc, dvc = chunk_backward(q[a:b], kp, vp, k[a:b], v[a:b],
                                                      do[a:b], scale)
            dq[a:b] = dq_c
            for g in range(Hkv):
                np.add.at(dk[:, g, :], tok[g], dkp[g])
                np.add.at(dv[:, g, :], tok[g], dvp[g])
            dk[a:b] += dkc
            dv[a:b] += dvc
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "selected": selected}
