"""Plain fp64 attention: the definition written out, score matrix materialised.

Test infrastructure only (see the package docstring).  Sources, cited by page
title and passage:

* "Fast and memory-efficient exact attention 分析", section 数学表达形式:
  Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V.
* "当注意力成为瓶颈从on困境到线性复杂度的技术突围", section 平方级的诅咒:
  S = Q K^T, P = softmax(S), O = P V, an n x n score matrix per head.
* "Self-attention Does Not Need O(n^2) Memory" (English summary), method
  bullets: the chunked method yields the same output as the standard method
  (it is exact), tracks the running maximum to avoid overflow, and is
  differentiated by recomputation.
* same page, method bullet on hardware-aware chunking: key/value blocks are
  processed independently and their results summarised and merged; and
  "当注意力成为瓶颈...", section IO感知, the two-block formulas
  m = max(max S1, max S2), l = sum e^(S1-m) + sum e^(S2-m),
  O = (e^(S1-m) V1 + e^(S2-m) V2) / l.

Readings where the pages are silent (each listed in the design notes):
* ``scale`` multiplies the dot product q.k (1/sqrt(d) in every workload).
* ``lse`` is the natural log of sum_j exp(scale * q.k_j) for each query row.
* The backward pass is ordinary softmax calculus, which the pages do not print:
  dV = P^T dO, dP = dO V^T, D_i = sum_d dO_id O_id, dS = P o (dP - D),
  dQ = scale dS K, dK = scale dS^T Q.

All arithmetic is fp64 on exact upcasts of the inputs.  ``numpy`` matmul is the
only library primitive used as a step.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    return a


# ---------------------------------------------------------------- one (b, h)

def scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """S[i, j] = scale * sum_d q[i, d] k[j, d]  (Nq x Nk, materialised)."""
    return float(scale) * (_f64(q) @ _f64(k).T)


def softmax_rows(s: np.ndarray):
    """Row softmax with the row maximum subtracted before exp.

    Returns (P, lse) with P[i, j] = exp(s[i, j] - m_i) / l_i,
    m_i = max_j s[i, j], l_i = sum_j exp(s[i, j] - m_i), lse_i = m_i + ln l_i.
    Subtracting the maximum is what keeps exp finite for logits of ~1e3; the
    method tracks the largest score for exactly this reason.
    """
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def attention_forward_2d(q, k, v, scale):
    """O = softmax(scale Q K^T) V and lse for one (batch, head): [Nq, D], [Nq]."""
    p, lse = softmax_rows(scores(q, k, scale))
    return p @ _f64(v), lse


def attention_backward_2d(q, k, v, do, scale):
    """Gradients of sum(dO o O) with respect to Q, K, V for one (batch, head).

    P is recomputed from the inputs (nothing of the forward is reused), which is
    also what the method does: its gradient recomputes intermediate states
    instead of storing them.
    Returns (dq, dk, dv, o, lse).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    p, lse = softmax_rows(scores(q, k, scale))
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    d_row = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - d_row)
    dq = float(scale) * (ds @ k)
    dk = float(scale) * (ds.T @ q)
    return dq, dk, dv, o, lse


# ------------------------------------------------------------- [B, H, N, D]

def _heads(x):
    x = _f64(x)
    assert x.ndim == 4, "expected [B, H, N, D]"
    return x


def attention_forward(q, k, v, scale):
    """Batched forward over [B, H, N, D]; returns (O [B,H,Nq,D], lse [B,H,Nq])."""
    q, k, v = _heads(q), _heads(k), _heads(v)
    B, H, Nq, D = q.shape
    o = np.empty((B, H, Nq, v.shape[3]))
    lse = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_2d(q[b, h], k[b, h], v[b, h], scale)
    return o, lse


def attention_backward(q, k, v, do, scale):
    """Batched backward over [B, H, N, D]; returns (dq, dk, dv, o, lse)."""
    q, k, v, do = _heads(q), _heads(k), _heads(v), _heads(do)
    B, H = q.shape[:2]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    o = np.empty(q.shape[:3] + (v.shape[3],))
    lse = np.empty(q.shape[:3])
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h], o[b, h], lse[b, h] = attention_backward_2d(
                q[b, h], k[b, h], v[b, h], do[b, h], scale)
    return dq, dk, dv, o, lse


# ------------------------------------------ shared key/value heads (GQA)
#
# "当注意力成为瓶颈从on困境到线性复杂度的技术突围", section 推理优化：减少KV Cache:
# multi-query and grouped-query attention let several query heads share one
# key/value head.  With H query heads and H_kv key/value heads (H a multiple of
# H_kv), query head h reads key/value head h // (H / H_kv): the page splits the
# query heads into consecutive groups without fixing the order, and consecutive
# groups are the plainest reading.  A shared K/V head is a parameter used by
# several heads, so its gradient is the sum over the heads that read it.

def attention_forward_gqa(q, k, v, scale):
    """q [B,H,Nq,D], k/v [B,H_kv,Nk,D] -> (O [B,H,Nq,D], lse [B,H,Nq])."""
    q, k, v = _heads(q), _heads(k), _heads(v)
    B, H, Nq, _ = q.shape
    Hkv = k.shape[1]
    assert H % Hkv == 0, "H must be a multiple of H_kv"
    G = H // Hkv
    o = np.empty((B, H, Nq, v.shape[3]))
    lse = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_2d(q[b, h], k[b, h // G], v[b, h // G], scale)
    return o, lse


def attention_backward_gqa(q, k, v, do, scale):
    """Gradients for shared key/value heads: dq [B,H,..], dk/dv [B,H_kv,..] summed over each group."""
    q, k, v, do = _heads(q), _heads(k), _heads(v), _heads(do)
    B, H = q.shape[:2]
    Hkv = k.shape[1]
    assert H % Hkv == 0, "H must be a multiple of H_kv"
    G = H // Hkv
    dq = np.empty_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    o = np.empty(q.shape[:3] + (v.shape[3],))
    lse = np.empty(q.shape[:3])
    for b in range(B):
        for h in range(H):
            dq[b, h], dk_h, dv_h, o[b, h], lse[b, h] = attention_backward_2d(
                q[b, h], k[b, h // G], v[b, h // G], do[b, h], scale)
            dk[b, h // G] += dk_h
            dv[b, h // G] += dv_h
    return dq, dk, dv, o, lse


# ------------------------------------------- sampled outputs at full size
#
# Query rows are independent problems, so the forward of a subset of rows is the
# definition applied to those rows.  Gradient entries are single entries of the
# same closed forms, evaluated one row (or one key column) at a time.

def attention_forward_rows(q2, k2, v2, scale, rows):
    """(O[rows], lse[rows]) for one (batch, head), each row over all keys."""
    rows = np.asarray(rows)
    return attention_forward_2d(_f64(q2)[rows], k2, v2, scale)


def attention_backward_rows(q2, k2, v2, do2, scale, rows):
    """dQ[rows] for one (batch, head): dQ_i = scale sum_j P_ij (dP_ij - D_i) k_j."""
    rows = np.asarray(rows)
    q, k, v, do = _f64(q2)[rows], _f64(k2), _f64(v2), _f64(do2)[rows]
    p, _ = softmax_rows(scores(q, k, scale))
    o = p @ v
    dp = do @ v.T
    d_row = (do * o).sum(axis=1, keepdims=True)
    return float(scale) * ((p * (dp - d_row)) @ k)


def attention_backward_keys(q2, k2, v2, do2, scale, keys, lse_all, o_all):
    """(dK[keys], dV[keys]) for one (batch, head).

    Needs, for every query row i, lse_i and O_i (from ``attention_forward_rows``
    over all rows); then P_ij = exp(scale q_i.k_j - lse_i) for the chosen
    columns j, dV_j = sum_i P_ij dO_i, dK_j = scale sum_i P_ij (dP_ij - D_i) q_i.
    """
    keys = np.asarray(keys)
    q, kk, vv, do = _f64(q2), _f64(k2)[keys], _f64(v2)[keys], _f64(do2)
    p = np.exp(scores(q, kk, scale) - _f64(lse_all)[:, None])
    dp = do @ vv.T
    d_row = (do * _f64(o_all)).sum(axis=1, keepdims=True)
    ds = p * (dp - d_row)
    return float(scale) * (ds.T @ q), p.T @ do


# ------------------------------------ the pages' chunked algorithm (checker)

def combine_two_blocks(m1, l1, acc1, m2, l2, acc2):
    """Merge two block summaries (m, l, acc) with the two-block formulas.

    m = max(m1, m2); l = l1 e^(m1-m) + l2 e^(m2-m); acc = acc1 e^(m1-m) + acc2 e^(m2-m).
    Here acc is the unnormalised sum of e^(s-m_block) v over the block.
    """
    m = np.maximum(m1, m2)
    a1 = np.exp(m1 - m)
    a2 = np.exp(m2 - m)
    return m, l1 * a1 + l2 * a2, acc1 * a1[..., None] + acc2 * a2[..., None]


def combine_partials(o_parts, lse_parts):
    """Merge R results computed over disjoint key ranges into the result over all of them.

    Each part r is exact attention over its own keys: O_r = sum_j p_rj v_j / l_r
    with lse_r = ln l_r (in the scaled-score units of lse).  The chunk summary
    of "Self-attention Does Not Need O(n^2) Memory" (English summary, the bullet
    on summarising chunk results) is (m_r, l_r, acc_r) with acc_r = l_r O_r e^{m_r};
    merged with the two-block formulas of "当注意力成为瓶颈" (section IO感知)
    it gives   lse = ln sum_r e^{lse_r},   O = sum_r e^{lse_r - lse} O_r.
    o_parts [R, ..., D], lse_parts [R, ...] -> (O [..., D], lse [...]).
    """
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m)
    total = w.sum(axis=0)
    lse = m + np.log(total)
    o = (w[..., None] * o_parts).sum(axis=0) / total[..., None]
    return o, lse


def chunked_forward_2d(q, k, v, scale, block):
    """The method's own order: keys/values in blocks, each block summarised as
    (running max m, total weight l, weighted value sum acc), summaries merged,
    normalisation postponed to the very end.

    Used only as a checker that the chunked method reaches the plain definition
    (it must agree with ``attention_forward_2d`` for any block size).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nk = k.shape[0]
    block = max(1, int(block))
    m = None
    for j0 in range(0, Nk, block):
        s = float(scale) * (q @ k[j0:j0 + block].T)
        mb = s.max(axis=1)
        e = np.exp(s - mb[:, None])
        lb = e.sum(axis=1)
        accb = e @ v[j0:j0 + block]
        if m is None:
            m, l, acc = mb, lb, accb
        else:
            m, l, acc = combine_two_blocks(m, l, acc, mb, lb, accb)
    return acc / l[:, None], m + np.log(l)
