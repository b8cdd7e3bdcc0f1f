"""Appending new K/V rows to an unexpanded cache, as a plain array copy.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

A decode step projects the new token's own Q/K/V, appends the new K/V to the cache and then
attends over the whole history; old queries are not needed [第三章 §3.1; MHA/MQA/GQA 逐步算例 §4].
The cache keeps the unexpanded shape (B, h_kv, T_max, d_h) [序列计算与存储 §缓存字节].
"""

from __future__ import annotations

import numpy as np


def kv_append_ref(k_cache, v_cache, k_new, v_new, pos):
    """Return copies of the caches with cache[b, g, pos[b] + t, :] = new[b, g, t, :] for t < S_new.

    Works on any element type (bf16 data is passed as its raw uint16 bits, so the copy is
    bit-exact).  Raises ValueError when a row would land outside [0, T_max).
    """
    k_cache = np.array(k_cache, copy=True)
    v_cache = np.array(v_cache, copy=True)
    k_new = np.asarray(k_new)
    v_new = np.asarray(v_new)
    B, h_kv, T_max, d_h = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape != v_new.shape:
        raise ValueError("shape mismatch")
    if k_new.shape[0] != B or k_new.shape[1] != h_kv or k_new.shape[3] != d_h:
        raise ValueError("new K/V shape does not match the cache")
    S_new = k_new.shape[2]
    pos = np.asarray(pos, np.int64).reshape(-1)
    if pos.shape[0] != B:
        raise ValueError("one position per sequence is required")
    for b in range(B):
        p = int(pos[b])
        if p < 0 or p + S_new > T_max:
            raise ValueError(f"rows [{p}, {p + S_new}) do not fit in a cache of {T_max}")
        k_cache[b, :, p:p + S_new, :] = k_new[b]
        v_cache[b, :, p:p + S_new, :] = v_new[b]
    return k_cache, v_cache
