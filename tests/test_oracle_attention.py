"""Pins for the oracle's attention (CPU only).

Each test ties ``oracle.attention`` / ``oracle.recurrent`` to something other
than the oracle itself: torch's fp64 scaled-dot-product attention and autograd,
central finite differences, closed forms, and invariants of softmax attention.
"""
import numpy as np
import pytest
import torch

from oracle.attention import (causal_attention, causal_attention_backward,
                              chunk_backward, chunk_forward, chunk_keys_backward,
                              chunk_rows_backward, chunk_rows_forward)
from oracle.recurrent import run_sequence, run_sequence_blocks
from oracle.sparse import topk_for_chunk


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _torch_sdpa(q, k, v, scale):
    """fp64 torch SDPA with K/V heads repeated for GQA; returns O [L][Hq][d]."""
    Hq, Hkv = q.shape[1], k.shape[1]
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(k).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)[None]
    vt = torch.tensor(v).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)[None]
    return qt, kt, vt


@pytest.mark.parametrize("L,Hq,Hkv,d", [(24, 4, 2, 8), (40, 6, 3, 16), (17, 2, 1, 4)])
def test_full_causal_matches_torch_sdpa_fwd_and_autograd(L, Hq, Hkv, d):
    q, k, v, do = (_rand((L, Hq, d), 1), _rand((L, Hkv, d), 2), _rand((L, Hkv, d), 3),
                   _rand((L, Hq, d), 4))
    scale = 0.37
    o, lse = causal_attention(q, k, v, scale)
    qt, kt, vt = _torch_sdpa(q, k, v, scale)
    kt0 = torch.tensor(k, requires_grad=True)
    vt0 = torch.tensor(v, requires_grad=True)
    qt0 = torch.tensor(q, requires_grad=True)
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt0.permute(1, 0, 2)[None],
        kt0.repeat_interleave(G, dim=1).permute(1, 0, 2)[None],
        vt0.repeat_interleave(G, dim=1).permute(1, 0, 2)[None],
        is_causal=True, scale=scale)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    (ref * torch.tensor(do)).sum().backward()
    dq, dk, dv = causal_attention_backward(q, k, v, do, scale)
    np.testing.assert_allclose(dq, qt0.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt0.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vt0.grad.numpy(), rtol=1e-10, atol=1e-12)
    # LSE pinned through torch's logsumexp of the masked logits
    for h in range(Hq):
        s = torch.tensor(q[:, h]) @ torch.tensor(k[:, h // G]).T * scale
        s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
        np.testing.assert_allclose(lse[h], torch.logsumexp(s, dim=1).numpy(), rtol=1e-12)


@pytest.mark.parametrize("C,P", [(8, 4), (16, 4), (32, 8)])
def test_chunk_recurrent_equals_full_causal(C, P):
    L, Hq, Hkv, d = 64, 4, 2, 8
    q, k, v, do = (_rand((L, Hq, d), 11), _rand((L, Hkv, d), 12), _rand((L, Hkv, d), 13),
                   _rand((L, Hq, d), 14))
    r = run_sequence(q, k, v, do, C, P, 0.3)
    o, lse = causal_attention(q, k, v, 0.3)
    dq, dk, dv = causal_attention_backward(q, k, v, do, 0.3)
    for a, b in [(r["o"], o), (r["lse"], lse), (r["dq"], dq), (r["dk"], dk), (r["dv"], dv)]:
        assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(b)))


def test_softmax_rows_sum_to_one_dense_and_sparse():
    L, Hq, Hkv, d, C, P = 64, 4, 2, 8, 16, 4
    q, k = _rand((L, Hq, d), 21, 3.0), _rand((L, Hkv, d), 22, 3.0)
    ones = np.ones((L, Hkv, 1))
    for top_k in (0, 2):
        r = run_sequence(q, k, ones, np.zeros((L, Hq, 1)), C, P, 0.5, top_k=top_k,
                         n_recent=1, with_backward=False)
        assert np.max(np.abs(r["o"] - 1.0)) <= 1e-12


def _loss(q, k, v, do, C, P, scale, **kw):
    return float(np.sum(run_sequence(q, k, v, do, C, P, scale, with_backward=False, **kw)["o"] * do))


@pytest.mark.parametrize("sparse", [False, True])
def test_gradients_match_central_finite_differences(sparse):
    L, C, P, Hq, Hkv, d = 32, 8, 4, 2, 1, 8
    q, k, v, do = (_rand((L, Hq, d), 31), _rand((L, Hkv, d), 32), _rand((L, Hkv, d), 33),
                   _rand((L, Hq, d), 34))
    scale = 1 / np.sqrt(d)
    kw = dict(top_k=2, n_recent=1) if sparse else {}
    r = run_sequence(q, k, v, do, C, P, scale, **kw)
    if sparse:  # freeze the selection: gradients do not flow through it
        kw = dict(selections=r["selected"])
    h = 1e-6
    for name, x, g in (("q", q, r["dq"]), ("k", k, r["dk"]), ("v", v, r["dv"])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, C, P, scale, **kw)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, C, P, scale, **kw)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert err <= 1e-6, (name, err)


def test_sparse_with_all_pages_equals_dense():
    L, Hq, Hkv, d, C, P = 96, 6, 2, 8, 16, 4
    q, k, v, do = (_rand((L, Hq, d), 41), _rand((L, Hkv, d), 42), _rand((L, Hkv, d), 43),
                   _rand((L, Hq, d), 44))
    dense = run_sequence(q, k, v, do, C, P, 0.35)
    sparse = run_sequence(q, k, v, do, C, P, 0.35, top_k=L // P, n_recent=2)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert np.max(np.abs(dense[key] - sparse[key])) <= 1e-12 * max(1, np.max(np.abs(dense[key])))


def test_closed_form_single_key():
    q, k, v = _rand((1, 3, 5), 51), _rand((1, 1, 5), 52), _rand((1, 1, 5), 53)
    o, lse = chunk_forward(q, [np.zeros((0, 5))], [np.zeros((0, 5))], k, v, 0.7)
    for h in range(3):
        np.testing.assert_allclose(o[0, h], v[0, 0], rtol=1e-14)
        assert abs(lse[h, 0] - 0.7 * float(q[0, h] @ k[0, 0])) <= 1e-14


def test_closed_form_zero_queries_give_prefix_means():
    L, Hq, Hkv, d = 48, 2, 1, 6
    q = np.zeros((L, Hq, d))
    k, v = _rand((L, Hkv, d), 61), _rand((L, Hkv, d), 62)
    r = run_sequence(q, k, v, np.zeros_like(q), 16, 4, 1.0, with_backward=False)
    prefix = np.cumsum(v[:, 0, :], axis=0) / np.arange(1, L + 1)[:, None]
    for h in range(Hq):
        np.testing.assert_allclose(r["o"][:, h, :], prefix, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["lse"][h], np.log(np.arange(1, L + 1)), rtol=1e-14)


def test_closed_form_constant_values():
    L, Hq, Hkv, d = 32, 4, 2, 8
    q, k, do = _rand((L, Hq, d), 71), _rand((L, Hkv, d), 72), _rand((L, Hq, d), 73)
    v = np.tile(_rand((1, Hkv, d), 74), (L, 1, 1))
    r = run_sequence(q, k, v, do, 8, 4, 0.4)
    for h in range(Hq):
        np.testing.assert_allclose(r["o"][:, h, :], v[:, h // 2, :], rtol=1e-12)
    assert np.max(np.abs(r["dq"])) <= 1e-12 and np.max(np.abs(r["dk"])) <= 1e-12


def test_key_shift_invariance():
    L, Hq, Hkv, d = 32, 2, 1, 8
    q, k, v = _rand((L, Hq, d), 81), _rand((L, Hkv, d), 82), _rand((L, Hkv, d), 83)
    c = _rand((d,), 84)
    o1, lse1 = causal_attention(q, k, v, 0.5)
    o2, lse2 = causal_attention(q, k + c, v, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
    for h in range(Hq):
        np.testing.assert_allclose(lse2[h] - lse1[h], 0.5 * q[:, h, :] @ c, rtol=1e-10, atol=1e-12)


def test_gqa_group_map_matches_repeated_heads():
    L, Hq, Hkv, d = 32, 6, 2, 8
    q, k, v, do = (_rand((L, Hq, d), 91), _rand((L, Hkv, d), 92), _rand((L, Hkv, d), 93),
                   _rand((L, Hq, d), 94))
    r = run_sequence(q, k, v, do, 8, 4, 0.3)
    kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)
    m = run_sequence(q, kr, vr, do, 8, 4, 0.3)
    np.testing.assert_allclose(r["o"], m["o"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["dq"], m["dq"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["dk"], m["dk"].reshape(L, Hkv, 3, d).sum(2), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("top_k", [0, 3])
def test_gradient_sum_invariants(top_k):
    L, Hq, Hkv, d, C, P = 64, 4, 2, 8, 16, 4
    q, k, v, do = (_rand((L, Hq, d), 101), _rand((L, Hkv, d), 102), _rand((L, Hkv, d), 103),
                   _rand((L, Hq, d), 104))
    r = run_sequence(q, k, v, do, C, P, 0.3, top_k=top_k, n_recent=1)
    # sum_j dS_ij = 0  =>  dk sums to zero per group; sum_j P_ij = 1 => dv sums to dO
    assert np.max(np.abs(r["dk"].sum(axis=0))) <= 1e-11
    for g in range(Hkv):
        np.testing.assert_allclose(r["dv"][:, g, :].sum(0), do[:, 2 * g:2 * g + 2, :].sum((0, 1)),
                                   rtol=1e-11, atol=1e-11)


def test_chunk_backward_matches_torch_autograd_on_key_set():
    C, Hq, Hkv, d, n = 12, 4, 2, 8, 20
    q, kc, vc, do = (_rand((C, Hq, d), 111), _rand((C, Hkv, d), 112), _rand((C, Hkv, d), 113),
                     _rand((C, Hq, d), 114))
    kp = [_rand((n, d), 115 + g) for g in range(Hkv)]
    vp = [_rand((n, d), 117 + g) for g in range(Hkv)]
    dq, dkp, dvp, dkc, dvc = chunk_backward(q, kp, vp, kc, vc, do, 0.4)
    # torch: explicit boolean mask over [past | current] keys, SDPA + autograd
    G = Hq // Hkv
    tq = torch.tensor(q, requires_grad=True)
    tkp = [torch.tensor(x, requires_grad=True) for x in kp]
    tvp = [torch.tensor(x, requires_grad=True) for x in vp]
    tkc, tvc = torch.tensor(kc, requires_grad=True), torch.tensor(vc, requires_grad=True)
    mask = torch.cat([torch.ones(C, n, dtype=torch.bool), torch.ones(C, C, dtype=torch.bool).tril()], 1)
    outs = []
    for h in range(Hq):
        g = h // G
        kk = torch.cat([tkp[g], tkc[:, g]], 0)
        vv = torch.cat([tvp[g], tvc[:, g]], 0)
        outs.append(torch.nn.functional.scaled_dot_product_attention(
            tq[:, h][None], kk[None], vv[None], attn_mask=mask[None], scale=0.4)[0])
    o_ref = torch.stack(outs, 1)
    o, _ = chunk_forward(q, kp, vp, kc, vc, 0.4)
    np.testing.assert_allclose(o, o_ref.detach().numpy(), rtol=1e-12, atol=1e-13)
    (o_ref * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dkc, tkc.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dvc, tvc.grad.numpy(), rtol=1e-10, atol=1e-12)
    for g in range(Hkv):
        np.testing.assert_allclose(dkp[g], tkp[g].grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dvp[g], tvp[g].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_sampled_rows_match_full_chunk():
    L, Hq, Hkv, d, C = 64, 2, 1, 8, 16
    q, k, v = _rand((L, Hq, d), 121), _rand((L, Hkv, d), 122), _rand((L, Hkv, d), 123)
    o, lse = causal_attention(q, k, v, 0.3)
    rows = np.array([0, 5, 17, 40, 63])
    o_s, lse_s = chunk_rows_forward(q[rows, 1], rows, k[:, 0], v[:, 0], np.arange(L), 0.3)
    np.testing.assert_allclose(o_s, o[rows, 1], rtol=1e-13)
    np.testing.assert_allclose(lse_s, lse[1, rows], rtol=1e-13)


def _block_selections(L, C, P, Hkv, T, seed):
    rng = np.random.default_rng(seed)
    sels = []
    for c in range(L // C):
        n_past = c * C // P
        sels.append([[sorted(rng.choice(n_past, size=int(rng.integers(0, n_past + 1)),
                                        replace=False).tolist()) if n_past else []
                      for _ in range(Hkv)] for _ in range((C + T - 1) // T)])
    return sels


@pytest.mark.parametrize("T", [8, 6])
def test_row_block_selections_match_torch_masked_attention_and_autograd(T):
    """Per-row-block key sets against a whole-sequence masked softmax in torch
    (fp64) and its autograd gradients; T = 6 leaves a ragged last block."""
    L, C, P, Hq, Hkv, d, scale = 48, 16, 4, 4, 2, 8, 0.3
    q, k, v, do = (_rand((L, Hq, d), 131), _rand((L, Hkv, d), 132), _rand((L, Hkv, d), 133),
                   _rand((L, Hq, d), 134))
    sels = _block_selections(L, C, P, Hkv, T, 135)
    ref = run_sequence_blocks(q, k, v, do, C, P, scale, T, selections=sels)
    G = Hq // Hkv
    mask = np.zeros((Hkv, L, L), dtype=bool)
    for i in range(L):
        c, b = i // C, (i % C) // T
        for g in range(Hkv):
            for pg in sels[c][b][g]:
                mask[g, i, pg * P:(pg + 1) * P] = True
            mask[g, i, c * C:i + 1] = True
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    outs, lses = [], []
    for h in range(Hq):
        g = h // G
        s = scale * (tq[:, h] @ tk[:, g].T)
        s = torch.where(torch.tensor(mask[g]), s, torch.tensor(float("-inf"), dtype=s.dtype))
        lses.append(torch.logsumexp(s, 1))
        outs.append(torch.softmax(s, 1) @ tv[:, g])
    o_t = torch.stack(outs, 1)
    np.testing.assert_allclose(ref["o"], o_t.detach().numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(ref["lse"], torch.stack(lses).detach().numpy(), rtol=1e-12,
                               atol=1e-12)
    (o_t * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(ref["dq"], tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(ref["dk"], tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(ref["dv"], tv.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_row_blocks_with_one_shared_selection_equal_the_chunk_form():
    L, C, P, Hq, Hkv, d = 48, 16, 4, 4, 2, 8
    q, k, v, do = (_rand((L, Hq, d), 141), _rand((L, Hkv, d), 142), _rand((L, Hkv, d), 143),
                   _rand((L, Hq, d), 144))
    chunk_sels = [s[0] for s in _block_selections(L, C, P, Hkv, C, 145)]
    blocks = [[s] * 2 for s in chunk_sels]                  # two 8-row blocks, same lists
    a = run_sequence(q, k, v, do, C, P, 0.3, selections=chunk_sels)
    b = run_sequence_blocks(q, k, v, do, C, P, 0.3, 8, selections=blocks)
    for key in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(b[key], a[key], rtol=1e-12, atol=1e-13)


def test_row_block_topk_is_the_selection_of_the_block_rows():
    L, C, P, Hq, Hkv, d, T = 48, 16, 4, 4, 2, 8, 8
    q, k, v, do = (_rand((L, Hq, d), 151), _rand((L, Hkv, d), 152), _rand((L, Hkv, d), 153),
                   _rand((L, Hq, d), 154))
    r = run_sequence_blocks(q, k, v, do, C, P, 0.3, T, top_k=2, n_recent=1, with_backward=False)
    for c in range(1, L // C):
        for b in range(C // T):
            rows = slice(c * C + b * T, c * C + (b + 1) * T)
            want, _ = topk_for_chunk(q[rows], k[:c * C], P, 2, 1)
            assert r["selected"][c][b] == want



def _torch_positions_attention(q, k, v, row_pos, key_pos, scale):
    """fp64 torch SDPA of rows [R][Hh][d] against keys [n][d] (one KV head)
    with the mask key_pos <= row_pos; tensors require grad."""
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    mask = torch.tensor(np.asarray(key_pos)[None, :] <= np.asarray(row_pos)[:, None])
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.permute(1, 0, 2), tk[None], tv[None], attn_mask=mask[None], scale=scale)
    return tq, tk, tv, o.permute(1, 0, 2)


def test_sampled_rows_backward_matches_torch_autograd():
    """O, LSE and dQ of sampled rows against torch SDPA + autograd on the same
    position mask: rows at the chunk start (only past keys + itself), inside,
    and at the end; keys out of order in memory."""
    n, d, scale = 70, 16, 0.29
    rng = np.random.default_rng(131)
    key_pos = rng.permutation(n)                       # absolute positions, shuffled
    row_pos = np.array([40, 41, 55, 69])
    q, do = _rand((4, d), 132), _rand((4, d), 133)
    k, v = _rand((n, d), 134), _rand((n, d), 135)
    o, lse, dq = chunk_rows_backward(q, do, row_pos, k, v, key_pos, scale)
    tq, tk, tv, ref = _torch_positions_attention(q[:, None], k, v, row_pos, key_pos, scale)
    np.testing.assert_allclose(o, ref[:, 0].detach().numpy(), rtol=1e-12, atol=1e-13)
    (ref[:, 0] * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad[:, 0].numpy(), rtol=1e-10, atol=1e-12)
    s = (torch.tensor(q) @ torch.tensor(k).T) * scale
    s = s.masked_fill(~torch.tensor(key_pos[None, :] <= row_pos[:, None]), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=1).numpy(), rtol=1e-12)


def test_sampled_keys_backward_matches_torch_autograd_and_finite_differences():
    """dK/dV of sampled keys of one group (three heads, causal chunk over a
    past) against torch autograd of the whole set, and against central
    finite differences of sum(O * dO) on two of the sampled keys."""
    past, C, G, d, scale = 24, 12, 3, 8, 0.41
    n = past + C
    key_pos = np.arange(n)
    row_pos = past + np.arange(C)
    q, do = _rand((C, G, d), 141), _rand((C, G, d), 142)
    k, v = _rand((n, d), 143), _rand((n, d), 144)
    idx = np.array([0, 7, 23, 24, 30, 35])            # past and current-chunk keys
    dk, dv = chunk_keys_backward(q, do, row_pos, k, v, key_pos, idx, scale)
    tq, tk, tv, ref = _torch_positions_attention(q, k, v, row_pos, key_pos, scale)
    (ref * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(dk, tk.grad.numpy()[idx], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy()[idx], rtol=1e-10, atol=1e-12)

    def loss(kk, vv):
        o = np.stack([chunk_rows_forward(q[:, h], row_pos, kk, vv, key_pos, scale)[0]
                      for h in range(G)], 1)
        return float(np.sum(o * do))
    h = 1e-6
    for j, which in ((1, "k"), (4, "v")):
        for e in range(d):
            kp, km, vp, vm = k.copy(), k.copy(), v.copy(), v.copy()
            if which == "k":
                kp[idx[j], e] += h
                km[idx[j], e] -= h
                fd = (loss(kp, v) - loss(km, v)) / (2 * h)
                assert abs(fd - dk[j, e]) <= 1e-6 * max(1.0, abs(dk[j, e]))
            else:
                vp[idx[j], e] += h
                vm[idx[j], e] -= h
                fd = (loss(k, vp) - loss(k, vm)) / (2 * h)
                assert abs(fd - dv[j, e]) <= 1e-6 * max(1.0, abs(dv[j, e]))
