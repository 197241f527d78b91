"""GPU parity: paged chunk attention (fwd, bwd, page-sparse lists) vs the oracle.

Inputs come from the seeded generator; the oracle runs on the same bf16 values
in fp64 over contiguous KV.  Tolerances: forward O and LSE relative L2 <= 5e-3
and max abs <= 1e-2 (bf16 inputs, fp32 accumulation, bf16 P and O); dQ, dK,
dV relative L2 <= 1e-2.
"""
import numpy as np
import pytest
import torch

from oracle.recurrent import run_sequence
from paged_kv_chunk_query_b200 import synth
from tests.paged_harness import PagedRun, rel_l2, to64

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS, BWD_REL = 5e-3, 1e-2, 1e-2

CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    # several Q/KV tiles, ragged last tile (320 = 2.5 tiles), GQA 7:1, shuffled pages
    "g7_d128_p64_ragged": synth.Workload("g7", 14, 2, 128, 64, 320, 3, seed=7, shuffle_pages=True),
    "g4_d128_p32": synth.Workload("g4", 8, 2, 128, 32, 256, 3, seed=8, shuffle_pages=True),
    "g2_d64_p128": synth.Workload("g2", 4, 2, 64, 128, 384, 2, seed=9),
    "g1_d128_p16": synth.Workload("g1", 2, 2, 128, 16, 192, 3, seed=10, shuffle_pages=True),
}


def _oracle(w, inp, selections=None, backward=True):
    return run_sequence(inp["q"], inp["k"], inp["v"], inp["do"], w.chunk_len, w.page_size,
                        w.softmax_scale, with_backward=backward, selections=selections)


def _check_fwd(w, ref, outs):
    C = w.chunk_len
    for c, out in enumerate(outs):
        o_ref = ref["o"][c * C:(c + 1) * C]
        lse_ref = ref["lse"][:, c * C:(c + 1) * C]
        o, lse = to64(out["o"]), to64(out["lse"])
        assert rel_l2(o, o_ref) <= FWD_REL, (c, rel_l2(o, o_ref))
        assert np.max(np.abs(o - o_ref)) <= FWD_ABS, (c, np.max(np.abs(o - o_ref)))
        assert rel_l2(lse, lse_ref) <= FWD_REL, (c, rel_l2(lse, lse_ref))
        assert np.max(np.abs(lse - lse_ref)) <= FWD_ABS, (c, np.max(np.abs(lse - lse_ref)))


@pytest.mark.parametrize("name", list(CASES))
def test_forward_dense_matches_oracle(name):
    w = CASES[name]
    inp = synth.sequence_inputs(w)
    ref = _oracle(w, inp, backward=False)
    with PagedRun(w) as r:
        outs = [r.chunk(c, synth.chunk_inputs(w, c), backward=False) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        assert r.status() == 0
        _check_fwd(w, ref, outs)


@pytest.mark.parametrize("name", list(CASES))
def test_backward_dense_matches_oracle(name):
    w = CASES[name]
    inp = synth.sequence_inputs(w)
    ref = _oracle(w, inp)
    with PagedRun(w) as r:
        outs = [r.chunk(c, synth.chunk_inputs(w, c)) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        assert r.status() == 0
        _check_fwd(w, ref, outs)
        dq = np.concatenate([to64(o["dq"]) for o in outs], axis=0)
        dk, dv = r.grads_by_token(w.context)
    assert rel_l2(dq, ref["dq"]) <= BWD_REL, rel_l2(dq, ref["dq"])
    assert rel_l2(dk, ref["dk"]) <= BWD_REL, rel_l2(dk, ref["dk"])
    assert rel_l2(dv, ref["dv"]) <= BWD_REL, rel_l2(dv, ref["dv"])


def _random_selections(w, seed, frac=0.5):
    rng = np.random.default_rng(seed)
    sels = []
    for c in range(w.num_chunks):
        n_past = c * w.pages_per_chunk
        per_group = []
        for g in range(w.num_kv_heads):
            k = int(rng.integers(0, n_past + 1)) if n_past else 0
            per_group.append(sorted(rng.choice(n_past, size=k, replace=False).tolist()) if k else [])
        sels.append(per_group)
    return sels


@pytest.mark.parametrize("name", ["g7_d128_p64_ragged", "g1_d128_p16", "tiny"])
def test_page_lists_per_group_match_oracle(name):
    """Per-group page lists of different lengths (ragged past tiles)."""
    w = CASES[name]
    inp = synth.sequence_inputs(w)
    sels = _random_selections(w, 123)
    ref = _oracle(w, inp, selections=sels)
    with PagedRun(w) as r:
        outs = [r.chunk(c, synth.chunk_inputs(w, c), selected=sels[c] if c else None)
                for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        assert r.status() == 0
        _check_fwd(w, ref, outs)
        dq = np.concatenate([to64(o["dq"]) for o in outs], axis=0)
        dk, dv = r.grads_by_token(w.context)
    assert rel_l2(dq, ref["dq"]) <= BWD_REL
    assert rel_l2(dk, ref["dk"]) <= BWD_REL
    assert rel_l2(dv, ref["dv"]) <= BWD_REL


# Units are (128-row query tile, query head); the forward runs one per SM.
# 160 units on 148 SMs: 148 whole, the last 12 split 12 ways (n_full > 0);
# 148 units fill the SMs exactly (no split even with a workspace).
SPLIT_CASES = {
    "units160_tail12": synth.Workload("u160", 80, 4, 64, 32, 256, 2, seed=21, shuffle_pages=True),
    "units148_no_tail": synth.Workload("u148", 74, 2, 64, 32, 256, 2, seed=22),
    "g7_d128_p64_ragged": CASES["g7_d128_p64_ragged"],
}


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("name", list(SPLIT_CASES))
def test_forward_split_last_wave_matches_oracle(name, split):
    """With and without the forward workspace, the forward gives the oracle's O
    and LSE: the split last wave (parts of a unit's key tiles, merged by
    log-sum-exp) within the same tolerance as the whole units."""
    w = SPLIT_CASES[name]
    inp = synth.sequence_inputs(w)
    ref = _oracle(w, inp, backward=False)
    with PagedRun(w, split_fwd=split) as r:
        outs = [r.chunk(c, synth.chunk_inputs(w, c), backward=False) for c in range(w.num_chunks)]
        torch.cuda.synchronize()
        assert r.status() == 0
        _check_fwd(w, ref, outs)
