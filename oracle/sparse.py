"""Page-level Top-K selection, fp64.

The pages: attention restricted to the key pages most relevant to the queries,
found by Top-K retrieval ([pt] §2C "Sparse Attention em Nível de Página";
[it] §2D); for dense models an average representative vector is computed per
key page and the pages most relevant to the current queries are kept ([es] §2B
"Atención Escasa a Nivel de Página"); natively sparse models keep the most
recent or selected pages ([it] §2D).

Readings where the pages are silent:
  * representative of a key page = mean of its P keys (per KV head);
  * query side = mean of the chunk's C rows over the G query heads of the
    group (one representative per chunk and KV-head group);
  * score = q_bar . k_bar (the softmax scale does not change the ranking and
    is left out);
  * candidates are the past pages except the R most recent; the R most recent
    pages are always kept; Top-K ranks candidates by (score descending,
    logical page id ascending) and keeps min(K, #candidates);
  * the kept list is returned in ascending logical page id; the current chunk
    is always attended (causally) and is not part of the list.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64


def page_key_means(k, page_size):
    """k ``[T][Hkv][d]`` (T a multiple of P) -> ``[T/P][Hkv][d]`` page means."""
    k = _f64(k)
    T, Hkv, d = k.shape
    return k.reshape(T // page_size, page_size, Hkv, d).mean(axis=1)


def group_query_means(q_chunk, num_kv_heads):
    """q ``[C][Hq][d]`` -> ``[Hkv][d]``: mean over the chunk's rows and the G heads
    of each group (heads g*G .. g*G+G-1)."""
    q = _f64(q_chunk)
    C, Hq, d = q.shape
    G = Hq // num_kv_heads
    return q.reshape(C, num_kv_heads, G, d).mean(axis=(0, 2))


def page_scores(q_bar, k_bar):
    """``[Hkv][d]`` x ``[n][Hkv][d]`` -> ``[Hkv][n]`` dot products."""
    return np.einsum("gd,pgd->gp", _f64(q_bar), _f64(k_bar))


def select_pages(scores, n_past, top_k, n_recent):
    """Kept logical page ids per group from the scores of the past pages.

    scores ``[Hkv][>= n_past]``.  Returns a list (one per group) of ascending
    logical ids: the Top-K candidates among pages [0, n_past - R) plus pages
    [max(0, n_past - R), n_past)."""
    scores = np.asarray(scores, dtype=np.float64)
    n_cand = max(0, n_past - n_recent)
    out = []
    for g in range(scores.shape[0]):
        cand = list(range(n_cand))
        cand.sort(key=lambda p: (-scores[g, p], p))
        kept = set(cand[:min(top_k, n_cand)])
        kept.update(range(n_cand, n_past))
        out.append(sorted(kept))
    return out


def kth_score(scores_g, n_past, top_k, n_recent):
    """Score of the K-th ranked candidate of one group (None if every candidate
    is kept).  Pages whose score lies within a tolerance of it are ties."""
    n_cand = max(0, n_past - n_recent)
    if top_k >= n_cand or top_k == 0:
        return None
    s = np.sort(np.asarray(scores_g[:n_cand], dtype=np.float64))[::-1]
    return float(s[top_k - 1])


def topk_for_chunk(q_chunk, k_past_tokens, page_size, top_k, n_recent):
    """Full selection for one chunk: returns (per-group kept lists, scores)."""
    k_past_tokens = _f64(k_past_tokens)
    num_kv_heads = k_past_tokens.shape[1]
    n_past = k_past_tokens.shape[0] // page_size
    if n_past == 0:
        return [[] for _ in range(num_kv_heads)], np.zeros((num_kv_heads, 0))
    k_bar = page_key_means(k_past_tokens, page_size)
    q_bar = group_query_means(q_chunk, k_bar.shape[1])
    s = page_scores(q_bar, k_bar)
    return select_pages(s, n_past, top_k, n_recent), s


def local_pages(n_past, window, num_kv_heads):
    """Recent-only page lists: layers that are sparse by construction attend
    to the most recent pages ([it] §2D) — here the last ``window`` of the
    ``n_past`` past pages, ascending, the same list for every group (plus,
    as always, the chunk itself causally)."""
    lo = max(0, n_past - window)
    return [list(range(lo, n_past)) for _ in range(num_kv_heads)]

