"""Pins for the oracle's Top-K selection and page-allocator model (CPU only)."""
import itertools
import os

import numpy as np
import pytest

from oracle.pool import PoolModel, SplitMix64, initial_order
from oracle.recurrent import run_sequence
from oracle.sparse import (group_query_means, kth_score, local_pages, page_key_means,
                           page_scores, select_pages, topk_for_chunk)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def test_splitmix64_published_outputs():
    r = SplitMix64(0)
    assert [r.next() for _ in range(3)] == [int(x, 16) for x in _golden_lines("splitmix64_state0.txt")]
    r = SplitMix64(1234567)
    assert [r.next() for _ in range(5)] == [int(x) for x in _golden_lines("splitmix64_state1234567.txt")]


def test_fisher_yates_is_uniform_permutation():
    # every one of the 6 permutations of 3 ids appears about 1/6 of the time
    counts = {}
    for seed in range(1, 6001):
        counts[tuple(initial_order(3, seed))] = counts.get(tuple(initial_order(3, seed)), 0) + 1
    assert sorted(counts) == sorted(itertools.permutations(range(3)))
    assert all(800 < c < 1200 for c in counts.values())
    # seed 0 keeps ascending order; any seed gives a permutation
    assert initial_order(10, 0) == list(range(10))
    assert sorted(initial_order(1000, 99)) == list(range(1000))


def test_fisher_yates_two_ids_swaps_on_even_draw():
    # i = 1: j = r mod 2; j == 0 swaps a[1] with a[0], j == 1 leaves it in place
    for seed in range(1, 50):
        first = SplitMix64(seed).next()
        assert initial_order(2, seed) == ([1, 0] if first % 2 == 0 else [0, 1])


def test_pool_model_lifo_and_errors():
    m = PoolModel(4)
    assert [m.alloc() for _ in range(4)] == [0, 1, 2, 3]
    assert m.alloc() is None
    assert m.free(2) and m.free(0)
    assert not m.free(0) and not m.free(7) and not m.free(-1)
    assert m.alloc() == 0 and m.alloc() == 2


def test_page_key_means_closed_form():
    P, Hkv, d = 4, 2, 3
    k = np.zeros((3 * P, Hkv, d))
    for p in range(3):
        k[p * P:(p + 1) * P] = p + 1.0         # constant page -> its value
    k[P + 1, 1, 0] += 8.0                      # one key off by 8 -> mean off by 8/P
    m = page_key_means(k, P)
    assert m.shape == (3, Hkv, d)
    assert m[0, 0, 0] == 1.0 and m[2, 1, 2] == 3.0
    assert m[1, 1, 0] == 2.0 + 8.0 / P and m[1, 0, 0] == 2.0


def test_group_query_means_uses_contiguous_head_groups():
    C, Hq, Hkv, d = 5, 6, 2, 4
    q = np.zeros((C, Hq, d))
    q[:, 0:3, :] = 1.5          # heads 0,1,2 -> group 0
    q[:, 3:6, :] = -100.0       # heads 3,4,5 -> group 1
    m = group_query_means(q, Hkv)
    np.testing.assert_array_equal(m[0], np.full(d, 1.5))
    np.testing.assert_array_equal(m[1], np.full(d, -100.0))


def _brute_force_kept(scores, n_past, K, R):
    n_cand = max(0, n_past - R)
    order = np.lexsort((np.arange(n_cand), -np.asarray(scores[:n_cand])))  # score desc, id asc
    kept = set(order[:min(K, n_cand)].tolist()) | set(range(n_cand, n_past))
    return sorted(kept)


@pytest.mark.parametrize("n_past,K,R", [(0, 4, 2), (1, 4, 2), (3, 4, 2), (10, 4, 2), (50, 7, 0),
                                        (50, 0, 3), (66, 64, 2), (67, 64, 2), (200, 64, 2)])
def test_select_pages_matches_brute_force_and_counts(n_past, K, R):
    rng = np.random.default_rng(n_past * 31 + K)
    s = rng.standard_normal((3, max(n_past, 1)))
    s[1, : n_past // 2] = np.round(s[1, : n_past // 2], 1)     # plenty of exact ties
    kept = select_pages(s, n_past, K, R)
    for g in range(3):
        assert kept[g] == _brute_force_kept(s[g], n_past, K, R)
        assert len(kept[g]) == min(K, max(0, n_past - R)) + min(R, n_past)
        assert set(range(max(0, n_past - R), n_past)) <= set(kept[g])
        assert kept[g] == sorted(kept[g])


def test_planted_page_is_selected():
    rng = np.random.default_rng(5)
    C, Hq, Hkv, d, P, n_pages = 32, 4, 2, 16, 8, 40
    q = rng.standard_normal((C, Hq, d))
    q[:, 2:4, :] += 3.0 * np.eye(d)[7]          # group 1's mean query points along axis 7
    k = rng.standard_normal((n_pages * P, Hkv, d))
    k[13 * P:14 * P, 1, 7] += 10.0              # page 13 of KV head 1 is aligned with it
    sel, s = topk_for_chunk(q, k, P, 1, 2)
    assert sel[1] == [13, n_pages - 2, n_pages - 1]
    assert s.shape == (Hkv, n_pages)
    np.testing.assert_allclose(s, page_scores(group_query_means(q, Hkv), page_key_means(k, P)))


def test_kth_score():
    s = np.array([0.5, 0.1, 0.9, 0.3, 0.7, 0.2])
    assert kth_score(s, 6, 2, 2) == 0.5      # candidates 0..3 sorted: .9 .5 .3 .1
    assert kth_score(s, 6, 4, 2) is None


@pytest.mark.parametrize("n_past,W", [(0, 4), (3, 4), (4, 4), (10, 4), (10, 1), (200, 64)])
def test_local_pages_are_the_last_window_pages(n_past, W):
    got = local_pages(n_past, W, 3)
    brute = [p for p in range(n_past) if n_past - p <= W]
    assert got == [brute] * 3
    assert len(got[0]) == min(W, n_past)
    # the same rule as Top-K's forced recent pages with no Top-K candidates kept
    s = np.zeros((3, max(n_past, 1)))
    assert got == select_pages(s, n_past, 0, W)


def test_local_window_covering_the_past_is_dense():
    rng = np.random.default_rng(9)
    L, C, P, Hq, Hkv, d = 64, 16, 4, 4, 2, 8
    q, do = rng.standard_normal((L, Hq, d)), rng.standard_normal((L, Hq, d))
    k, v = rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d))
    dense = run_sequence(q, k, v, do, C, P, 0.35)
    sels = [local_pages(c * C // P, L // P, Hkv) for c in range(L // C)]
    local = run_sequence(q, k, v, do, C, P, 0.35, selections=sels)
    for key in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(local[key], dense[key], rtol=1e-12, atol=1e-12)
    # a window of one page: rows see only the last past page and the chunk
    sels1 = [local_pages(c * C // P, 1, Hkv) for c in range(L // C)]
    one = run_sequence(q, k, v, do, C, P, 0.35, selections=sels1, with_backward=False)
    from oracle.attention import chunk_forward
    c = 2
    a = c * C
    kp = [k[a - P:a, g] for g in range(Hkv)]
    vp = [v[a - P:a, g] for g in range(Hkv)]
    o_c, _ = chunk_forward(q[a:a + C], kp, vp, k[a:a + C], v[a:a + C], 0.35)
    np.testing.assert_allclose(one["o"][a:a + C], o_c, rtol=1e-12, atol=1e-12)

