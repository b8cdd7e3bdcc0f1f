"""Multi-head latent attention (MLA) decode over a latent cache, in fp64 NumPy.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

The pages [第 09 章 GQA、MLA 与跨层 KV 共享 §09.3; 第三章 §3.4]:

* The cache holds one low-dimensional latent per token, C = X W_D with C : [B, T, c], and the
  keys and values are its up-projections K = C W_UK, V = C W_UV (W_UK, W_UV : [c, H d]).
* For one head, by associativity and with no approximation,
      Q (C U_K)^T = (Q U_K^T) C^T        and        P (C U_V) = (P C) U_V,
  so a decode step can score the latent cache directly with the absorbed query Q U_K^T and
  up-project the latent output P C afterwards, never rebuilding K or V.
* Position: a rotation applied to the expanded key does not commute with the up-projection, so
  the full MLA keeps a separate position-dependent key part beside the latent (decoupled RoPE);
  the cache formula must count it. Here that part is kr : [B, T, d_r], shared by every head, and
  each head's query has a matching part q_r; both arrive already rotated (position encoding is
  outside the attention core, as for the GQA path).

Score of head h against token j:   s_hj = scale * (q_lat_h . C_j + q_r_h . kr_j),
output:                             o_lat_h = sum_j softmax_j(s_hj) C_j        (width c).

This is attention with one shared "KV head" whose key row is [C_j, kr_j] and whose value row is
C_j, the first c entries of the same row. The functions below state it both ways: the absorbed
form the kernel computes, and the explicit form (rebuild K_h, V_h per head, ordinary attention),
which the pins compare.
"""

from __future__ import annotations

import numpy as np


def mla_decode_ref(q, cache, d_v, kv_len=None, q_pos=None, scale=None):
    """Absorbed MLA decode: attention of every head's query row over the shared latent cache.

    q: (B, h_q, d_qk) = [absorbed latent query (d_v) | rotary query part (d_qk - d_v)].
    cache: (B, T_max, d_qk) = [latent C (d_v) | rotary key part kr].
    Values are cache[..., :d_v]. Token j of sequence b is visible iff j < min(kv_len[b], q_pos[b]+1)
    (q_pos defaults to kv_len - 1). ``scale`` must be the model's softmax scale (for absorbed MLA it
    is 1/sqrt(d_nope + d_rope) of the original heads, not 1/sqrt(d_qk)); default 1/sqrt(d_qk).
    Returns (o_lat (B, h_q, d_v), lse (B, h_q)), natural-log lse.
    """
    q = np.asarray(q, np.float64)
    cache = np.asarray(cache, np.float64)
    B, h_q, d_qk = q.shape
    T_max = cache.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d_qk)
    kv_len = np.full(B, T_max, np.int64) if kv_len is None else np.asarray(kv_len, np.int64)
    q_pos = kv_len - 1 if q_pos is None else np.asarray(q_pos, np.int64)
    O = np.zeros((B, h_q, d_v))
    L = np.zeros((B, h_q))
    for b in range(B):
        n = int(min(kv_len[b], q_pos[b] + 1))
        if n <= 0:
            raise ValueError("query has no visible key")
        rows = cache[b, :n]
        S = (q[b] @ rows.T) * scale  # (h_q, n): all d_qk columns
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        den = E.sum(axis=1, keepdims=True)
        O[b] = (E / den) @ rows[:, :d_v]
        L[b] = m[:, 0] + np.log(den[:, 0])
    return O, L


def absorb_query(q_nope, w_uk):
    """q_lat_h = q_nope_h U_K^h^T for every head: q_nope (B, h, d), w_uk (c, h*d) -> (B, h, c)."""
    q_nope = np.asarray(q_nope, np.float64)
    B, h, d = q_nope.shape
    U = np.asarray(w_uk, np.float64).reshape(-1, h, d)  # (c, h, d)
    return np.einsum("bhd,chd->bhc", q_nope, U)


def up_project(o_lat, w_uv):
    """o_h = o_lat_h U_V^h: o_lat (B, h, c), w_uv (c, h*d) -> (B, h, d)."""
    o_lat = np.asarray(o_lat, np.float64)
    B, h, c = o_lat.shape
    U = np.asarray(w_uv, np.float64).reshape(c, h, -1)  # (c, h, d)
    return np.einsum("bhc,chd->bhd", o_lat, U)


def mla_explicit_ref(q_nope, q_rope, c_cache, kr_cache, w_uk, w_uv, kv_len=None, scale=None):
    """Non-absorbed MLA decode: rebuild K_h = [C U_K^h, kr] and V_h = C U_V^h for every head and
    run ordinary attention. Returns o (B, h, d_v_head)."""
    q_nope = np.asarray(q_nope, np.float64)
    q_rope = np.asarray(q_rope, np.float64)
    C = np.asarray(c_cache, np.float64)
    kr = np.asarray(kr_cache, np.float64)
    B, h, d = q_nope.shape
    T = C.shape[1]
    Uk = np.asarray(w_uk, np.float64).reshape(-1, h, d)
    Uv = np.asarray(w_uv, np.float64).reshape(C.shape[2], h, -1)
    if scale is None:
        scale = 1.0 / np.sqrt(d + q_rope.shape[2])
    kv_len = np.full(B, T, np.int64) if kv_len is None else np.asarray(kv_len, np.int64)
    out = np.zeros((B, h, Uv.shape[2]))
    for b in range(B):
        n = int(kv_len[b])
        for a in range(h):
            K = np.concatenate([C[b, :n] @ Uk[:, a, :], kr[b, :n]], axis=1)  # (n, d + d_r)
            V = C[b, :n] @ Uv[:, a, :]
            s = (np.concatenate([q_nope[b, a], q_rope[b, a]]) @ K.T) * scale
            p = np.exp(s - s.max())
            out[b, a] = (p / p.sum()) @ V
    return out


def mla_cache_elements_per_token(c, d_r=0):
    """Cached numbers per token and layer: the latent plus the decoupled position key part."""
    return c + d_r
