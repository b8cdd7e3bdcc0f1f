"""The pages' blockwise (online) softmax recurrence, in fp64, one query at a time.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``). This is a second, independent CPU path: it
follows the recurrence the pages state, in their order and notation, so that the split-KV
partial/combine arithmetic has a pinned counterpart.  It is written from the equations, not
from the page's listing.

State for one query over the keys J read so far [序列计算与存储 §在线 softmax]:
    m = max_{j in J} s_j,   l = sum_{j in J} e^{s_j - m},   u = sum_{j in J} e^{s_j - m} v_j,
starting from m = -inf, l = 0, u = 0; the output is o = u / l.
Reading a block I with block maximum m_hat: m' = max(m, m_hat),
    l' = e^{m - m'} l + sum_{j in I} e^{s_j - m'},   u' = e^{m - m'} u + sum_{j in I} e^{s_j - m'} v_j.
A block whose scores are all -inf is skipped, since -inf - (-inf) is not a number.
Two partial states over disjoint key sets merge the same way [第三章 §3.5]:
    m' = max(m_a, m_b),  l' = e^{m_a - m'} l_a + e^{m_b - m'} l_b,  u' likewise.
"""

from __future__ import annotations

import numpy as np


def _empty_state(d: int):
    return (-np.inf, 0.0, np.zeros(d, np.float64))


def online_softmax_row(scores, values, block: int, return_states: bool = False):
    """Blockwise softmax-weighted average of ``values`` (T, d) under ``scores`` (T,).

    ``scores`` are already scaled and masked (-inf marks an invisible key).
    Returns o (d,), or (o, [state after each non-skipped block]) with ``return_states``.
    Raises ValueError when no key is visible.
    """
    s_all = np.asarray(scores, np.float64).reshape(-1)
    v_all = np.asarray(values, np.float64)
    if v_all.ndim == 1:
        v_all = v_all[:, None]
    if block <= 0 or v_all.shape[0] != s_all.shape[0]:
        raise ValueError("bad block size or score/value length mismatch")
    m, l, u = _empty_state(v_all.shape[1])
    states = []
    for start in range(0, s_all.shape[0], block):
        s = s_all[start:start + block]
        v = v_all[start:start + block]
        finite = np.isfinite(s)
        if not finite.any():
            continue  # fully masked block
        s, v = s[finite], v[finite]
        m_new = max(m, float(s.max()))
        alpha = np.exp(m - m_new)          # e^{m - m'}; 0 while m is still -inf
        w = np.exp(s - m_new)              # e^{s_j - m'}
        l = alpha * l + w.sum()
        u = alpha * u + w @ v
        m = m_new
        states.append((m, l, u.copy()))
    if l == 0.0:
        raise ValueError("query has no visible key")
    o = u / l
    return (o, states) if return_states else o


def merge_states(a, b):
    """Merge two partial states (m, l, u) built over disjoint key sets [第三章 §3.5]."""
    m_a, l_a, u_a = a
    m_b, l_b, u_b = b
    m = max(m_a, m_b)
    if m == -np.inf:
        return (m, 0.0, np.zeros_like(np.asarray(u_a, np.float64)))
    fa = np.exp(m_a - m)
    fb = np.exp(m_b - m)
    return (m, fa * l_a + fb * l_b, fa * np.asarray(u_a) + fb * np.asarray(u_b))


def blockwise_attention_row(q, k, v, q_pos: int, kv_len: int, scale: float, block: int,
                            n_splits: int = 1, causal: bool = True):
    """One query row of one head, computed the way a split-KV decode does.

    The visible keys are cut into ``n_splits`` contiguous ranges; each range is reduced with the
    blockwise recurrence into a state (m, l, u); the states are merged with ``merge_states``.
    Returns (o (d,), lse) where lse = m + log(l).
    """
    q = np.asarray(q, np.float64).reshape(-1)
    k = np.asarray(k, np.float64)[:kv_len]
    v = np.asarray(v, np.float64)[:kv_len]
    n_vis = min(kv_len, q_pos + 1) if causal else kv_len
    if n_vis <= 0:
        raise ValueError("query has no visible key")
    s = (k[:n_vis] @ q) * scale
    bounds = np.linspace(0, n_vis, n_splits + 1).round().astype(int)
    total = _empty_state(v.shape[1])
    for i in range(n_splits):
        lo, hi = bounds[i], bounds[i + 1]
        if hi <= lo:
            continue
        _, states = online_softmax_row(s[lo:hi], v[lo:hi], block, return_states=True)
        total = merge_states(total, states[-1])
    m, l, u = total
    return u / l, m + np.log(l)
