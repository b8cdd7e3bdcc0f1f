"""Gradients of grouped-query attention: the plain definition, in fp64 NumPy.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

The pages describe the training side of FlashAttention as keeping a few statistics from the
forward pass and recomputing the local scores in the backward pass, so the probability matrix is
never stored [序列计算与存储 §两块算例, the paragraph after the listing; 第三章 §3.5]. What that
backward pass computes is fixed by the forward definition alone: the gradient of

    O_a = P_a V_{g(a)},   P_a = softmax(S_a),   S_a = Q_a K_{g(a)}^T * scale + M

with respect to Q, K and V for an upstream gradient dO. Written out per query head a (rows i,
visible keys j), with g = g(a):

    dV_g  += P_a^T dO_a                       (every head of the group adds into its K/V head)
    dP_a   = dO_a V_g^T
    D_i    = sum_j P_ij dP_ij                 (= sum_c dO_ic O_ic)
    dS_a   = P_a * (dP_a - D)                  (the softmax Jacobian applied row by row)
    dQ_a   = scale * dS_a K_g
    dK_g  += scale * dS_a^T Q_a

Invisible pairs have P = 0 and so contribute nothing; keys at or past kv_len get zero gradient.
Everything is materialised; nothing is recomputed or blocked here.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import group_of


def _visible(q_pos, kv_len, causal, window):
    j = np.arange(kv_len)
    vis = (j[None, :] <= q_pos[:, None]) if causal else np.ones((len(q_pos), kv_len), bool)
    if window is not None:
        vis &= j[None, :] > q_pos[:, None] - window
    return vis


def attention_backward_ref(q, k_cache, v_cache, d_o, q_start=None, kv_len=None, scale=None,
                           causal=True, window=None):
    """(dQ, dK, dV) of O = attention_ref(q, k_cache, v_cache, ...) for upstream gradient ``d_o``.

    q, d_o: (B, h_q, S_q, d_h); k_cache, v_cache: (B, h_kv, T_max, d_h).
    Returns dQ (B, h_q, S_q, d_h), dK and dV (B, h_kv, T_max, d_h), float64; rows j >= kv_len[b]
    of dK and dV are zero.
    """
    q = np.asarray(q, np.float64)
    d_o = np.asarray(d_o, np.float64)
    k_cache = np.asarray(k_cache, np.float64)
    v_cache = np.asarray(v_cache, np.float64)
    B, h_q, S_q, d_h = q.shape
    _, h_kv, T_max, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    q_start = np.zeros(B, np.int64) if q_start is None else np.asarray(q_start, np.int64)
    kv_len = np.full(B, T_max, np.int64) if kv_len is None else np.asarray(kv_len, np.int64)

    dQ = np.zeros_like(q)
    dK = np.zeros_like(k_cache)
    dV = np.zeros_like(v_cache)
    for b in range(B):
        n = int(kv_len[b])
        pos = q_start[b] + np.arange(S_q)
        vis = _visible(pos, n, causal, window)
        if not vis.any(axis=1).all():
            raise ValueError("query has no visible key")
        for a in range(h_q):
            g = group_of(a, h_q, h_kv)
            K = k_cache[b, g, :n]
            V = v_cache[b, g, :n]
            S = np.where(vis, (q[b, a] @ K.T) * scale, -np.inf)
            E = np.exp(S - S.max(axis=1, keepdims=True))
            P = E / E.sum(axis=1, keepdims=True)
            dO = d_o[b, a]
            dV[b, g, :n] += P.T @ dO
            dP = dO @ V.T
            D = (P * dP).sum(axis=1)
            dS = P * (dP - D[:, None])
            dQ[b, a] = scale * (dS @ K)
            dK[b, g, :n] += scale * (dS.T @ q[b, a])
    return dQ, dK, dV


def softmax_backward_rowterm(o, d_o):
    """D_i = sum_c dO_ic O_ic per row: the term the backward subtracts from dP (it equals
    sum_j P_ij dP_ij because O = P V)."""
    return (np.asarray(o, np.float64) * np.asarray(d_o, np.float64)).sum(axis=-1)
