"""Pins for the oracle's sliding-window mask (a query at position p sees keys p - W < j <= p).

The page lists sliding-window attention as a route where each layer reads only a local window
[第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.7, the Sliding Window Attention row];
the window's exact extent is this project's reading (W keys, the query's own included). These pins
tie that reading to things outside the oracle: a window of 1 returns the query's own value row,
a window of W equals unwindowed attention over the W-key slice of the cache, a window wider than
the history changes nothing, torch's SDPA with a band mask built from tril/triu agrees, and a
pure-Python double loop agrees on tiny inputs.
"""

import math

import numpy as np
import pytest
import torch

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_visible_count_closed_form():
    assert oracle.visible_count(10, 100, window=4) == 4     # keys 7..10
    assert oracle.visible_count(2, 100, window=4) == 3      # keys 0..2: the window is cut at 0
    assert oracle.visible_count(10, 9, window=4) == 2       # keys 7..8: cut by the length
    assert oracle.visible_count(10, 100) == 11
    assert oracle.visible_count(10, 100, window=1) == 1


def test_window_one_returns_own_value_row():
    rng = np.random.default_rng(7)
    B, h_q, h_kv, T, d = 2, 4, 2, 20, 8
    q, k, v = _rand(rng, B, h_q, d), _rand(rng, B, h_kv, T, d), _rand(rng, B, h_kv, T, d)
    q_pos = np.array([5, 19])
    O, L = oracle.decode_ref(q, k, v, q_pos=q_pos, window=1)
    r = h_q // h_kv
    for b in range(B):
        for a in range(h_q):
            g = a // r
            assert np.array_equal(O[b, a], v[b, g, q_pos[b]])
            assert math.isclose(L[b, a], float(q[b, a] @ k[b, g, q_pos[b]]) / math.sqrt(d), rel_tol=1e-14)


@pytest.mark.parametrize("W", [2, 5, 16])
def test_window_equals_attention_over_the_slice(W):
    rng = np.random.default_rng(W)
    B, h_q, h_kv, T, d = 2, 6, 3, 40, 8
    q, k, v = _rand(rng, B, h_q, d), _rand(rng, B, h_kv, T, d), _rand(rng, B, h_kv, T, d)
    for p in (0, 3, W - 1, W, 39):
        lo = max(0, p - W + 1)
        O, L = oracle.decode_ref(q, k, v, q_pos=np.full(B, p), window=W)
        Os, Ls = oracle.decode_ref(q, k[:, :, lo:p + 1], v[:, :, lo:p + 1], q_pos=np.full(B, p - lo))
        assert np.allclose(O, Os, rtol=0, atol=1e-13) and np.allclose(L, Ls, rtol=0, atol=1e-13)


def test_wide_window_changes_nothing():
    rng = np.random.default_rng(3)
    B, h_q, h_kv, S, d = 1, 4, 1, 12, 8
    q, k, v = _rand(rng, B, h_q, S, d), _rand(rng, B, h_kv, S, d), _rand(rng, B, h_kv, S, d)
    O0, L0 = oracle.attention_ref(q, k, v)
    O1, L1 = oracle.attention_ref(q, k, v, window=S)
    O2, L2 = oracle.attention_ref(q, k, v, window=10 * S)
    assert np.array_equal(O0, O1) and np.array_equal(O0, O2)
    assert np.array_equal(L0, L1) and np.array_equal(L0, L2)
    # one narrower window does change the late rows and only them
    O3, _ = oracle.attention_ref(q, k, v, window=S - 1)
    assert np.array_equal(O3[:, :, :S - 1], O0[:, :, :S - 1])
    assert not np.allclose(O3[:, :, S - 1], O0[:, :, S - 1])


@pytest.mark.parametrize("W", [1, 3, 7])
def test_matches_torch_sdpa_band_mask(W):
    rng = np.random.default_rng(11 + W)
    B, h_q, h_kv, S, d = 2, 8, 2, 24, 16
    q, k, v = _rand(rng, B, h_q, S, d), _rand(rng, B, h_kv, S, d), _rand(rng, B, h_kv, S, d)
    O, _ = oracle.attention_ref(q, k, v, window=W)
    r = h_q // h_kv
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(k).repeat_interleave(r, dim=1)
    tv = torch.from_numpy(v).repeat_interleave(r, dim=1)
    ones = torch.ones(S, S, dtype=torch.bool)
    band = torch.tril(ones) & torch.triu(ones, diagonal=-(W - 1))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=band)
    assert np.allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_brute_force_windowed_prefill_with_offset():
    """Pure-Python loops: rows at positions q_start + i, keys q_start + i - W < j <= q_start + i."""
    rng = np.random.default_rng(5)
    B, h_q, h_kv, S_q, T, d, W = 1, 2, 1, 4, 9, 3, 3
    q, k, v = _rand(rng, B, h_q, S_q, d), _rand(rng, B, h_kv, T, d), _rand(rng, B, h_kv, T, d)
    q_start, kv_len = np.array([5]), np.array([9])
    O, _ = oracle.attention_ref(q, k, v, q_start=q_start, kv_len=kv_len, window=W)
    for a in range(h_q):
        for i in range(S_q):
            pos = 5 + i
            keys = [j for j in range(9) if pos - W < j <= pos]
            s = [sum(q[0, a, i, c] * k[0, 0, j, c] for c in range(d)) / math.sqrt(d) for j in keys]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            tot = sum(w)
            for c in range(d):
                want = sum(w[n] * v[0, 0, keys[n], c] for n in range(len(keys))) / tot
                assert abs(O[0, a, i, c] - want) < 1e-12


def test_window_zero_is_rejected():
    rng = np.random.default_rng(0)
    with pytest.raises(ValueError):
        oracle.decode_ref(_rand(rng, 1, 1, 4), _rand(rng, 1, 1, 5, 4), _rand(rng, 1, 1, 5, 4), window=0)
