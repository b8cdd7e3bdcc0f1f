"""The plain definition of causal grouped-query attention, in fp64 NumPy.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``): never imported by the CUDA library.

Definition followed, in the pages' notation:

* h_q query heads, h_kv K/V heads, h_q divisible by h_kv, r = h_q / h_kv query heads per group;
  query head a (counted from 0) reads K/V head g(a) = floor(a / r)
  [序列计算与存储 §分组查询注意力; 第 09 章 §09.2]. Heads of one group are adjacent
  (A, A, B, B), never interleaved (A, B, A, B) [第 09 章 §09.2].
* O_a = softmax(Q_a K_{g(a)}^T / sqrt(d_h) + M) V_{g(a)}, softmax along the key axis,
  M = 0 on visible pairs and -inf elsewhere [序列计算与存储 §分组查询注意力, display equation
  for O_a; §分块注意力, S = QK^T/sqrt(d_h) + M, P = softmax(S), O = PV].
* M is causal or padding [序列计算与存储 §分组查询注意力]. A query's causal limit is its
  absolute position, not its index inside the current call: with a cache, a single query at
  position t must see keys 0..t [第 09 章 §09.2, ptr_current_pos paragraph; 第三章 §3.3 note that
  is_causal only fits equal-length Q and K]. So query row i of batch b sits at position
  q_start[b] + i and sees key j iff j <= q_start[b] + i (causal) and j < kv_len[b] (padding).
* A query with no visible key is an error [序列计算与存储 §两块算例, the error the listing raises].
* Sliding window (optional): each query reads only a local window of the history [第三章 §3.7,
  the Sliding Window Attention row]. The page gives no formula; the reading taken here is that a
  window of W keeps the W most recent positions up to and including the query's own, i.e. key j is
  visible iff q_pos - W < j <= q_pos (and j < kv_len). W = None means no window.

The score matrix S and the weights P are materialised in full; K/V are read through g(a) and
never expanded.  ``scale`` defaults to 1/sqrt(d_h) and may be given explicitly, because the
pages' worked examples use unscaled scores.
"""

from __future__ import annotations

import numpy as np


def group_of(a: int, h_q: int, h_kv: int) -> int:
    """K/V head read by query head ``a``: floor(a / r) with r = h_q / h_kv.

    [序列计算与存储 §分组查询注意力: g(a) = floor(a / r); 第 09 章 §09.2 and its exercise 1.]
    """
    if h_kv <= 0 or h_q <= 0 or h_q % h_kv != 0:
        raise ValueError(f"h_q={h_q} must be a positive multiple of h_kv={h_kv}")
    if not 0 <= a < h_q:
        raise ValueError(f"query head {a} out of range [0, {h_q})")
    r = h_q // h_kv
    return a // r


def visible_count(q_pos: int, kv_len: int, causal: bool = True, window=None) -> int:
    """Number of keys a query at absolute position ``q_pos`` sees in a sequence of ``kv_len`` keys.

    The visible keys are j < min(kv_len, q_pos + 1) (causal) or j < kv_len (not causal); a window
    of W further requires j > q_pos - W.
    """
    hi = min(kv_len, q_pos + 1) if causal else kv_len
    lo = 0 if window is None else max(0, q_pos - window + 1)
    return max(0, hi - lo)


def head_attention(q_rows, k, v, q_pos, kv_len: int, scale: float, causal: bool = True,
                   window=None):
    """One query head against the K/V head it reads.

    q_rows: (n, d_h) queries; k, v: (T, d_h) with T >= kv_len; q_pos: (n,) absolute positions.
    Returns (O (n, d_h), lse (n,)) where lse is the natural log of sum_j exp(S_ij) over visible j.
    Keys at positions >= kv_len are never read (they may hold anything, including NaN).
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)[:kv_len]
    v = np.asarray(v, dtype=np.float64)[:kv_len]
    q_pos = np.asarray(q_pos, dtype=np.int64).reshape(-1)
    n = q_rows.shape[0]
    if q_pos.shape[0] != n:
        raise ValueError("one absolute position per query row is required")

    # S = Q K^T * scale, shape (n, kv_len): every pair, materialised.
    S = (q_rows @ k.T) * scale
    j = np.arange(kv_len)
    if causal:
        visible = j[None, :] <= q_pos[:, None]
    else:
        visible = np.ones((n, kv_len), dtype=bool)
    if window is not None:
        if window < 1:
            raise ValueError("a window holds at least one key")
        visible &= j[None, :] > q_pos[:, None] - window
    if n and not visible.any(axis=1).all():
        raise ValueError("query has no visible key")
    # M: 0 where visible, -inf elsewhere.
    S = np.where(visible, S, -np.inf)

    # softmax along the key axis; subtracting the row maximum does not change the ratio.
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    denom = E.sum(axis=1, keepdims=True)
    P = E / denom
    # O = P V. Invisible keys carry weight exactly 0 (entries of k, v below kv_len must be finite).
    O = P @ v
    lse = m[:, 0] + np.log(denom[:, 0])
    return O, lse


def attention_ref(q, k_cache, v_cache, q_start=None, kv_len=None, scale=None, causal=True,
                  window=None):
    """Grouped-query attention for a batch.

    q: (B, h_q, S_q, d_h); k_cache, v_cache: (B, h_kv, T_max, d_h).
    q_start: (B,) absolute position of query row 0 (default 0).
    kv_len: (B,) number of keys present (default T_max).
    window: None, or W >= 1: row i also needs key j > q_start + i - W.
    Returns (O (B, h_q, S_q, d_h) float64, lse (B, h_q, S_q) float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache)
    v_cache = np.asarray(v_cache)
    B, h_q, S_q, d_h = q.shape
    Bk, h_kv, T_max, d_k = k_cache.shape
    if (Bk, d_k) != (B, d_h) or v_cache.shape != k_cache.shape:
        raise ValueError("q, k_cache and v_cache shapes disagree")
    if h_q % h_kv != 0:
        raise ValueError(f"h_q={h_q} must be a multiple of h_kv={h_kv}")
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    q_start = np.zeros(B, np.int64) if q_start is None else np.asarray(q_start, np.int64)
    kv_len = np.full(B, T_max, np.int64) if kv_len is None else np.asarray(kv_len, np.int64)
    if np.any(kv_len < 0) or np.any(kv_len > T_max):
        raise ValueError("kv_len out of range")

    O = np.empty((B, h_q, S_q, d_h), np.float64)
    L = np.empty((B, h_q, S_q), np.float64)
    for b in range(B):
        pos = q_start[b] + np.arange(S_q)
        n_keys = int(kv_len[b])
        for a in range(h_q):
            g = group_of(a, h_q, h_kv)
            O[b, a], L[b, a] = head_attention(
                q[b, a], k_cache[b, g], v_cache[b, g], pos, n_keys, scale, causal, window
            )
    return O, L


def decode_ref(q, k_cache, v_cache, kv_len=None, q_pos=None, scale=None, window=None):
    """Single-token decode: one query per sequence at absolute position q_pos[b].

    q: (B, h_q, d_h). q_pos defaults to kv_len[b] - 1: the current token's K/V is already in the
    cache when it attends [MHA/MQA/GQA 逐步算例 §4: after appending, 8192 positions are visible].
    Returns (O (B, h_q, d_h), lse (B, h_q)).
    """
    q = np.asarray(q, dtype=np.float64)
    B = q.shape[0]
    T_max = np.asarray(k_cache).shape[2]
    kv_len = np.full(B, T_max, np.int64) if kv_len is None else np.asarray(kv_len, np.int64)
    q_pos = kv_len - 1 if q_pos is None else np.asarray(q_pos, np.int64)
    O, L = attention_ref(q[:, :, None, :], k_cache, v_cache, q_start=q_pos, kv_len=kv_len,
                         scale=scale, causal=True, window=window)
    return O[:, :, 0, :], L[:, :, 0]
