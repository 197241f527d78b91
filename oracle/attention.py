"""fp64 attention: full causal reference and one chunk against a key set.

The pages describe custom operators that run attention directly on the paged
KV cache, forward and backward, with gradients added in place ([pt] §2B
"Kernels Personalizados"; [es] §2B "Gestión de Memoria Paginada" and "Kernels
Personalizados"; [it] §2B).  They print no formula, so the forward and backward
here are the textbook softmax attention definitions written out:

  S_ij = scale * q_i . k_j          over the row's key set
  LSE_i = ln sum_j exp(S_ij)        (natural log, computed with max subtraction)
  P_ij = exp(S_ij - LSE_i)
  O_i  = sum_j P_ij v_j
and for the loss  L = sum_i O_i . dO_i :
  D_i   = dO_i . O_i
  dP_ij = dO_i . v_j
  dS_ij = P_ij (dP_ij - D_i)
  dq_i  = scale * sum_j dS_ij k_j
  dk_j  = scale * sum_i dS_ij q_i      (summed over every query head of the group)
  dv_j  = sum_i P_ij dO_i              (likewise)

Head h reads KV head g = h // G with G = Hq / Hkv (contiguous groups).
Matrix products use numpy's fp64 matmul as a library primitive.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().float().numpy()
    return np.asarray(x, dtype=np.float64)


def _softmax_rows(s: np.ndarray):
    """Rows of logits (with -inf for masked entries) -> (P, LSE)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    lse = m + np.log(l)
    return e / l, lse[:, 0]


def causal_attention(q, k, v, scale):
    """Causal attention over a whole concatenated sequence.

    q ``[L][Hq][d]``, k and v ``[L][Hkv][d]``.  Row i sees keys j <= i.
    Returns O ``[L][Hq][d]`` and LSE ``[Hq][L]``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    keep = np.tril(np.ones((L, L), dtype=bool))
    o = np.zeros((L, Hq, v.shape[2]))
    lse = np.zeros((Hq, L))
    for h in range(Hq):
        g = h // G
        s = np.where(keep, scale * (q[:, h, :] @ k[:, g, :].T), -np.inf)
        p, lse[h] = _softmax_rows(s)
        o[:, h, :] = p @ v[:, g, :]
    return o, lse


def causal_attention_backward(q, k, v, do, scale):
    """Gradients of sum(O * dO) for :func:`causal_attention` (whole sequence)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    keep = np.tril(np.ones((L, L), dtype=bool))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(Hq):
        g = h // G
        s = np.where(keep, scale * (q[:, h, :] @ k[:, g, :].T), -np.inf)
        p, _ = _softmax_rows(s)
        o = p @ v[:, g, :]
        D = np.sum(do[:, h, :] * o, axis=1)
        dp = do[:, h, :] @ v[:, g, :].T
        ds = p * (dp - D[:, None])
        dq[:, h, :] = scale * (ds @ k[:, g, :])
        dk[:, g, :] += scale * (ds.T @ q[:, h, :])
        dv[:, g, :] += p.T @ do[:, h, :]
    return dq, dk, dv


def _chunk_logits(qh, kp, kc, scale):
    """Logits of one head's chunk rows against [selected past keys | current chunk].

    Past keys are seen by every row; the current chunk is causal (local key t'
    is seen by local row t iff t' <= t), which is the absolute-position causal
    rule because every past key precedes the chunk."""
    C = qh.shape[0]
    s_past = scale * (qh @ kp.T)
    s_cur = scale * (qh @ kc.T)
    s_cur = np.where(np.tril(np.ones((C, C), dtype=bool)), s_cur, -np.inf)
    return np.concatenate([s_past, s_cur], axis=1)


def chunk_forward(q, k_past, v_past, k_cur, v_cur, scale):
    """Forward of one chunk.

    q ``[C][Hq][d]``; ``k_past[g]``, ``v_past[g]`` ``[n_g][d]`` are the past keys
    group g attends to (every earlier token for dense, the tokens of the
    selected pages for page-sparse); ``k_cur``, ``v_cur`` ``[C][Hkv][d]`` are the
    chunk's own keys.  Returns O ``[C][Hq][d]`` and LSE ``[Hq][C]``.
    """
    q, k_cur, v_cur = _f64(q), _f64(k_cur), _f64(v_cur)
    C, Hq, d = q.shape
    Hkv = k_cur.shape[1]
    G = Hq // Hkv
    o = np.zeros((C, Hq, v_cur.shape[2]))
    lse = np.zeros((Hq, C))
    for h in range(Hq):
        g = h // G
        kp, vp = _f64(k_past[g]).reshape(-1, d), _f64(v_past[g]).reshape(-1, v_cur.shape[2])
        s = _chunk_logits(q[:, h, :], kp, k_cur[:, g, :], scale)
        p, lse[h] = _softmax_rows(s)
        o[:, h, :] = p @ np.concatenate([vp, v_cur[:, g, :]], axis=0)
    return o, lse


def chunk_backward(q, k_past, v_past, k_cur, v_cur, do, scale):
    """Backward of one chunk for the loss sum(O * dO).

    Returns dq ``[C][Hq][d]``, dk_past / dv_past (lists over groups of
    ``[n_g][d]``: this chunk's contribution to the selected past keys), and
    dk_cur / dv_cur ``[C][Hkv][d]``.  The selection is a constant: nothing
    flows through it.
    """
    q, k_cur, v_cur, do = _f64(q), _f64(k_cur), _f64(v_cur), _f64(do)
    C, Hq, d = q.shape
    Hkv = k_cur.shape[1]
    G = Hq // Hkv
    dv_dim = v_cur.shape[2]
    dq = np.zeros_like(q)
    dk_cur, dv_cur = np.zeros_like(k_cur), np.zeros_like(v_cur)
    dk_past = [np.zeros((np.asarray(k_past[g]).shape[0], d)) for g in range(Hkv)]
    dv_past = [np.zeros((np.asarray(v_past[g]).shape[0], dv_dim)) for g in range(Hkv)]
    for h in range(Hq):
        g = h // G
        kp, vp = _f64(k_past[g]).reshape(-1, d), _f64(v_past[g]).reshape(-1, dv_dim)
        n = kp.shape[0]
        kk = np.concatenate([kp, k_cur[:, g, :]], axis=0)
        vv = np.concatenate([vp, v_cur[:, g, :]], axis=0)
        s = _chunk_logits(q[:, h, :], kp, k_cur[:, g, :], scale)
        p, _ = _softmax_rows(s)
        o = p @ vv
        D = np.sum(do[:, h, :] * o, axis=1)
        dp = do[:, h, :] @ vv.T
        ds = p * (dp - D[:, None])
        dq[:, h, :] = scale * (ds @ kk)
        dkk = scale * (ds.T @ q[:, h, :])
        dvv = p.T @ do[:, h, :]
        dk_past[g] += dkk[:n]
        dv_past[g] += dvv[:n]
        dk_cur[:, g, :] += dkk[n:]
        dv_cur[:, g, :] += dvv[n:]
    return dq, dk_past, dv_past, dk_cur, dv_cur


def _block_logits(qh, row0, kp, kc, scale):
    """Logits of one head's row block (chunk rows row0 .. row0 + T - 1) against
    [its past keys | the chunk's keys 0 .. row0 + T - 1], causal on the latter."""
    T = qh.shape[0]
    kc = kc[: row0 + T]
    s_past = scale * (qh @ kp.T)
    s_cur = scale * (qh @ kc.T)
    keep = np.arange(row0 + T)[None, :] <= (row0 + np.arange(T))[:, None]
    s_cur = np.where(keep, s_cur, -np.inf)
    return np.concatenate([s_past, s_cur], axis=1)


def chunk_forward_blocks(q, block_rows, k_past, v_past, k_cur, v_cur, scale):
    """Forward of one chunk whose rows come in blocks of ``block_rows`` with a
    key set each: the pages relevant to each query page ([pt] §2C).

    ``k_past[b][g]``, ``v_past[b][g]`` ``[n_bg][d]`` are the past keys group g
    attends to from rows of block b; the chunk's own keys are causal as in
    :func:`chunk_forward`.  Returns O ``[C][Hq][d]`` and LSE ``[Hq][C]``."""
    q, k_cur, v_cur = _f64(q), _f64(k_cur), _f64(v_cur)
    C, Hq, d = q.shape
    Hkv = k_cur.shape[1]
    G = Hq // Hkv
    dv_dim = v_cur.shape[2]
    o = np.zeros((C, Hq, dv_dim))
    lse = np.zeros((Hq, C))
    for b in range((C + block_rows - 1) // block_rows):
        r0, r1 = b * block_rows, min(C, (b + 1) * block_rows)
        for h in range(Hq):
            g = h // G
            kp = _f64(k_past[b][g]).reshape(-1, d)
            vp = _f64(v_past[b][g]).reshape(-1, dv_dim)
            s = _block_logits(q[r0:r1, h, :], r0, kp, k_cur[:, g, :], scale)
            pm, lse[h, r0:r1] = _softmax_rows(s)
            o[r0:r1, h, :] = pm @ np.concatenate([vp, v_cur[:r1, g, :]], axis=0)
    return o, lse


def chunk_backward_blocks(q, block_rows, k_past, v_past, k_cur, v_cur, do, scale):
    """Backward of :func:`chunk_forward_blocks` for the loss sum(O * dO).

    Returns dq, dk_past / dv_past (``[b][g]`` lists: block b's contribution to
    its own past key set) and dk_cur / dv_cur ``[C][Hkv][d]``."""
    q, k_cur, v_cur, do = _f64(q), _f64(k_cur), _f64(v_cur), _f64(do)
    C, Hq, d = q.shape
    Hkv = k_cur.shape[1]
    G = Hq // Hkv
    dv_dim = v_cur.shape[2]
    nb = (C + block_rows - 1) // block_rows
    dq = np.zeros_like(q)
    dk_cur, dv_cur = np.zeros_like(k_cur), np.zeros_like(v_cur)
    dk_past = [[np.zeros((np.asarray(k_past[b][g]).reshape(-1, d).shape[0], d))
                for g in range(Hkv)] for b in range(nb)]
    dv_past = [[np.zeros((np.asarray(v_past[b][g]).reshape(-1, dv_dim).shape[0], dv_dim))
                for g in range(Hkv)] for b in range(nb)]
    for b in range(nb):
        r0, r1 = b * block_rows, min(C, (b + 1) * block_rows)
        for h in range(Hq):
            g = h // G
            kp = _f64(k_past[b][g]).reshape(-1, d)
            vp = _f64(v_past[b][g]).reshape(-1, dv_dim)
            n = kp.shape[0]
            kk = np.concatenate([kp, k_cur[:r1, g, :]], axis=0)
            vv = np.concatenate([vp, v_cur[:r1, g, :]], axis=0)
            s = _block_logits(q[r0:r1, h, :], r0, kp, k_cur[:, g, :], scale)
            pm, _ = _softmax_rows(s)
            o = pm @ vv
            D = np.sum(do[r0:r1, h, :] * o, axis=1)
            dp = do[r0:r1, h, :] @ vv.T
            ds = pm * (dp - D[:, None])
            dq[r0:r1, h, :] = scale * (ds @ kk)
            dkk = scale * (ds.T @ q[r0:r1, h, :])
            dvv = pm.T @ do[r0:r1, h, :]
            dk_past[b][g] += dkk[:n]
            dv_past[b][g] += dvv[:n]
            dk_cur[:r1, g, :] += dkk[n:]
            dv_cur[:r1, g, :] += dvv[n:]
    return dq, dk_past, dv_past, dk_cur, dv_cur


def chunk_rows_forward(q_rows, row_pos, k_keys, v_keys, key_pos, scale):
    """Forward for a few sampled rows of ONE head, used at sizes where a whole
    chunk is too slow in fp64.

    q_rows ``[R][d]`` with absolute positions ``row_pos`` ``[R]``; k_keys,
    v_keys ``[n][d]`` with absolute positions ``key_pos`` ``[n]`` (every key the
    row's chunk may see).  Row i sees key j iff key_pos[j] <= row_pos[i].
    Returns O ``[R][d]`` and LSE ``[R]``."""
    q_rows, k_keys, v_keys = _f64(q_rows), _f64(k_keys), _f64(v_keys)
    keep = np.asarray(key_pos)[None, :] <= np.asarray(row_pos)[:, None]
    s = np.where(keep, scale * (q_rows @ k_keys.T), -np.inf)
    p, lse = _softmax_rows(s)
    return p @ v_keys, lse


def chunk_rows_backward(q_rows, do_rows, row_pos, k_keys, v_keys, key_pos, scale):
    """Forward and dQ for a few sampled rows of ONE head (the sizes where a
    whole chunk is too slow in fp64).

    Same arguments as :func:`chunk_rows_forward` plus dO of those rows
    ``[R][d]``.  dq_i needs only row i's own softmax: D_i = dO_i . O_i,
    dP_ij = dO_i . v_j, dS_ij = P_ij (dP_ij - D_i), dq_i = scale sum_j dS_ij k_j.
    Returns O ``[R][d]``, LSE ``[R]`` and dQ ``[R][d]``."""
    q_rows, do_rows = _f64(q_rows), _f64(do_rows)
    k_keys, v_keys = _f64(k_keys), _f64(v_keys)
    keep = np.asarray(key_pos)[None, :] <= np.asarray(row_pos)[:, None]
    s = np.where(keep, scale * (q_rows @ k_keys.T), -np.inf)
    p, lse = _softmax_rows(s)
    o = p @ v_keys
    D = np.sum(do_rows * o, axis=1)
    dp = do_rows @ v_keys.T
    ds = p * (dp - D[:, None])
    return o, lse, scale * (ds @ k_keys)


def chunk_keys_backward(q, do, row_pos, k_keys, v_keys, key_pos, key_idx, scale):
    """One chunk's contribution to dK and dV of a few sampled keys of ONE
    KV-head group, summed over the group's query heads.

    q, do ``[R][G][d]``: every query row of the chunk for the G heads of the
    group (absolute positions ``row_pos`` ``[R]``); k_keys, v_keys ``[n][d]``:
    every key the chunk's rows may see (positions ``key_pos``; row i sees key
    j iff key_pos[j] <= row_pos[i]); ``key_idx``: indices into those keys.
    Each head's softmax needs every key (LSE_i and D_i = dO_i . O_i);
    then, for the sampled keys j only, dK_j = scale sum_i dS_ij q_i and
    dV_j = sum_i P_ij dO_i.  Returns dK, dV ``[len(key_idx)][d]``."""
    q, do = _f64(q), _f64(do)
    k_keys, v_keys = _f64(k_keys), _f64(v_keys)
    key_idx = np.asarray(key_idx, dtype=np.int64)
    keep = np.asarray(key_pos)[None, :] <= np.asarray(row_pos)[:, None]
    dk = np.zeros((len(key_idx), k_keys.shape[1]))
    dv = np.zeros((len(key_idx), v_keys.shape[1]))
    for h in range(q.shape[1]):
        s = np.where(keep, scale * (q[:, h, :] @ k_keys.T), -np.inf)
        p, _ = _softmax_rows(s)
        o = p @ v_keys
        D = np.sum(do[:, h, :] * o, axis=1)
        p_j = p[:, key_idx]
        dp_j = do[:, h, :] @ v_keys[key_idx].T
        ds_j = p_j * (dp_j - D[:, None])
        dk += scale * (ds_j.T @ q[:, h, :])
        dv += p_j.T @ do[:, h, :]
    return dk, dv
