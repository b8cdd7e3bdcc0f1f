"""Paged KV cache: the oracle's view of a cache stored as fixed-size pages plus a block table.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

The pages name page metadata and fragmentation as a deployment concern of the cache
[第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.6; MHA/MQA/GQA walkthrough, section 8,
the ledger's note on page metadata]. The layout used here: a pool of pages
``(num_pages, h_kv, page_size, d_h)``; logical position t of sequence b lives in page
``block_table[b, t // page_size]`` at row ``t % page_size``. Attention over a paged cache is, by
definition, attention over the contiguous cache these pages spell out; the oracle gathers that
contiguous cache and calls the plain definition.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import decode_ref


def gather_pages(pages, block_table, lengths, T_max=None):
    """Contiguous cache (B, h_kv, T_max, d_h) spelled out by ``block_table`` over ``pages``.

    pages: (num_pages, h_kv, page_size, d_h); block_table: (B, max_pages) int; lengths: (B,).
    Positions at or beyond lengths[b] are left as NaN (they are never read).
    """
    pages = np.asarray(pages)
    block_table = np.asarray(block_table, np.int64)
    num_pages, h_kv, page_size, d_h = pages.shape
    B, max_pages = block_table.shape
    T_max = max_pages * page_size if T_max is None else T_max
    out = np.full((B, h_kv, T_max, d_h), np.nan, dtype=np.float64)
    for b in range(B):
        n = int(lengths[b])
        if n > max_pages * page_size:
            raise ValueError("length beyond the block table")
        for t0 in range(0, n, page_size):
            page = int(block_table[b, t0 // page_size])
            if not 0 <= page < num_pages:
                raise ValueError(f"page index {page} out of range")
            m = min(page_size, n - t0)
            out[b, :, t0:t0 + m] = pages[page, :, :m]
    return out


def paged_decode_ref(q, k_pages, v_pages, block_table, kv_len, q_pos=None, scale=None, window=None):
    """Decode over a paged cache = decode over the gathered contiguous cache."""
    k = gather_pages(k_pages, block_table, kv_len)
    v = gather_pages(v_pages, block_table, kv_len)
    return decode_ref(q, k, v, kv_len=kv_len, q_pos=q_pos, scale=scale, window=window)


def paged_append_ref(k_pages, v_pages, k_new, v_new, block_table, pos):
    """Copies of the page pools with new[b, g, t] written at logical position pos[b] + t.

    Works on raw element types (bit-exact). Raises ValueError when a position falls outside the
    block table or names a page outside the pool.
    """
    k_pages = np.array(k_pages, copy=True)
    v_pages = np.array(v_pages, copy=True)
    block_table = np.asarray(block_table, np.int64)
    num_pages, h_kv, page_size, d_h = k_pages.shape
    B, max_pages = block_table.shape
    k_new = np.asarray(k_new)
    v_new = np.asarray(v_new)
    S_new = k_new.shape[2]
    for b in range(B):
        for t in range(S_new):
            p = int(pos[b]) + t
            if p < 0 or p >= max_pages * page_size:
                raise ValueError("position outside the block table")
            page = int(block_table[b, p // page_size])
            if not 0 <= page < num_pages:
                raise ValueError("page index out of range")
            k_pages[page, :, p % page_size] = k_new[b, :, t]
            v_pages[page, :, p % page_size] = v_new[b, :, t]
    return k_pages, v_pages
