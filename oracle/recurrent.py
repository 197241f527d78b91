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

from .attention import (_f64, chunk_backward, chunk_backward_blocks, chunk_forward,
                        chunk_forward_blocks)
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


def _page_tokens(pages, page_size):
    if not len(pages):
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(p * page_size, (p + 1) * page_size)
                           for p in pages]).astype(np.int64)


def run_sequence_blocks(q, k, v, do, chunk_len, page_size, scale, block_rows, top_k=0,
                        n_recent=0, with_backward=True, selections=None):
    """As :func:`run_sequence`, with one page selection per block of
    ``block_rows`` query rows of a chunk instead of one per chunk ([pt] §2C:
    the pages relevant to each query page).

    ``selections[c][b][g]`` gives block b's kept logical pages for group g
    (chunk 0 may be None: it has no past); otherwise each block runs the
    oracle's Top-K on its own rows.  Returns the dict of :func:`run_sequence`
    with ``selected[c][b][g]``."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    L, Hq, d = q.shape
    Hkv = k.shape[1]
    N = L // chunk_len
    nb = (chunk_len + block_rows - 1) // block_rows
    o = np.zeros((L, Hq, v.shape[2]))
    lse = np.zeros((Hq, L))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    selected = []
    for c in range(N):
        a, e = c * chunk_len, (c + 1) * chunk_len
        sel = []
        for b in range(nb):
            if c == 0:
                sel.append([[] for _ in range(Hkv)])
            elif selections is not None:
                sel.append(selections[c][b])
            else:
                r0, r1 = a + b * block_rows, min(e, a + (b + 1) * block_rows)
                sb, _ = topk_for_chunk(q[r0:r1], k[:a], page_size, top_k, n_recent)
                sel.append(sb)
        selected.append(sel)
        tok = [[_page_tokens(sel[b][g], page_size) for g in range(Hkv)] for b in range(nb)]
        kp = [[k[tok[b][g], g, :] for g in range(Hkv)] for b in range(nb)]
        vp = [[v[tok[b][g], g, :] for g in range(Hkv)] for b in range(nb)]
        o_c, lse_c = chunk_forward_blocks(q[a:e], block_rows, kp, vp, k[a:e], v[a:e], scale)
        o[a:e], lse[:, a:e] = o_c, lse_c
        if with_backward:
            dq_c, dkp, dvp, dkc, dvc = chunk_backward_blocks(q[a:e], block_rows, kp, vp, k[a:e],
                                                             v[a:e], do[a:e], scale)
            dq[a:e] = dq_c
            for b in range(nb):
                for g in range(Hkv):
                    np.add.at(dk[:, g, :], tok[b][g], dkp[b][g])
                    np.add.at(dv[:, g, :], tok[b][g], dvp[b][g])
            dk[a:e] += dkc
            dv[a:e] += dvc
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "selected": selected}

