"""Pins for the fp64 oracle: page values, closed forms, invariants, independent library routines.

Each test names the plausible oracle mistake it would catch.  Nothing here calls the CUDA library.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import ledgers

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _round(x, digits):
    return np.round(np.asarray(x, np.float64), digits)


# ---------------------------------------------------------------------------------------------
# Page-printed worked examples
# ---------------------------------------------------------------------------------------------

def test_mqa_two_queries_page_values():
    """序列计算与存储 §头与投影: keys [1,2], values [10,20], queries 0 and 1 -> 15 and 17.310586.

    Catches: wrong softmax axis, transposed Q/K, dropped max-subtraction sign, wrong group.
    """
    g = GOLDEN["mqa_two_queries"]
    # MQA: h_q = 2 query heads, h_kv = 1; d_h = 1; one query per head at position 1 (sees both keys)
    q = np.array(g["queries"], np.float64).reshape(1, 2, 1, 1)
    k = np.array(g["keys"], np.float64).reshape(1, 1, 2, 1)
    v = np.array(g["values"], np.float64).reshape(1, 1, 2, 1)
    O, lse = oracle.attention_ref(q, k, v, q_start=[1], scale=g["scale"])
    assert np.array_equal(_round(O[0, :, 0, 0], g["printed_digits"]), np.array(g["outputs"]))
    # weights of query 1 are e^{s_j - lse}
    w = np.exp(np.array([1.0, 2.0]) * 1.0 - lse[0, 1, 0])
    assert np.array_equal(_round(w, 6), np.array(g["weights_query1"]))
    # query 0 gives equal weights: plain mean (a closed form)
    assert O[0, 0, 0, 0] == 15.0


def test_two_block_example_direct():
    """序列计算与存储 §两块算例: scores log[1,2,3,4] on values [1,2,3,4] give exactly 3."""
    g = GOLDEN["two_block_online_softmax"]
    s = np.log(np.array(g["scores_are_log_of"]))
    q = np.ones((1, 1, 1, 1))
    k = s.reshape(1, 1, 4, 1)
    v = np.array(g["values"]).reshape(1, 1, 4, 1)
    O, lse = oracle.attention_ref(q, k, v, q_start=[3], scale=1.0)
    assert abs(O[0, 0, 0, 0] - g["output"]) < 1e-14
    assert abs(lse[0, 0, 0] - math.log(10.0)) < 1e-14  # sum of weights' numerators 1+2+3+4
    w = np.exp(s - lse[0, 0, 0])
    assert np.allclose(w, g["weights"], atol=1e-15)


def test_two_block_example_online_states():
    """序列计算与存储 §两块算例: states (m=ln2, l=1.5, u=2.5) then (ln4, 2.5, 7.5); wrong mean 2.619048."""
    g = GOLDEN["two_block_online_softmax"]
    s = np.log(np.array(g["scores_are_log_of"]))
    v = np.array(g["values"])
    o, states = oracle.online_softmax_row(s, v, block=g["block"], return_states=True)
    (m1, l1, u1), (m2, l2, u2) = states
    a1, a2 = g["after_block1"], g["after_block2"]
    assert abs(m1 - math.log(a1["m_is_log_of"])) < 1e-15
    assert abs(l1 - a1["l"]) < 1e-15 and abs(u1[0] - a1["u"]) < 1e-15
    assert abs(m2 - math.log(a2["m_is_log_of"])) < 1e-15
    assert abs(l2 - a2["l"]) < 1e-14 and abs(u2[0] - a2["u"]) < 1e-14
    assert abs(o[0] - g["output"]) < 1e-14
    # averaging the two locally normalised outputs is the page's counter-example
    loc = [oracle.online_softmax_row(s[i:i + 2], v[i:i + 2], block=2)[0] for i in (0, 2)]
    assert np.allclose(loc, g["local_outputs"], atol=1e-15)
    assert round(float(np.mean(loc)), 6) == g["wrong_average"]
    assert abs(np.mean(loc) - o[0]) > 0.3


def test_merge_states_equals_single_pass():
    """第三章 §3.5: merging two partial states equals one pass over both blocks."""
    g = GOLDEN["two_block_online_softmax"]
    s = np.log(np.array(g["scores_are_log_of"]))
    v = np.array(g["values"])[:, None]
    _, sa = oracle.online_softmax_row(s[:2], v[:2], block=2, return_states=True)
    _, sb = oracle.online_softmax_row(s[2:], v[2:], block=2, return_states=True)
    m, l, u = oracle.merge_states(sa[-1], sb[-1])
    assert abs(l - 2.5) < 1e-14 and abs(u[0] - 7.5) < 1e-14 and abs(m - math.log(4)) < 1e-15
    # merge is symmetric and has the empty state as identity
    m2, l2, u2 = oracle.merge_states(sb[-1], sa[-1])
    assert (m, l) == (m2, l2) and np.array_equal(u, u2)
    e = (-np.inf, 0.0, np.zeros(1))
    assert oracle.merge_states(e, sa[-1])[1] == sa[-1][1]


def test_scores_two_zero_example_closed_form():
    """MHA/MQA/GQA 逐步算例 §2: scores [2,0] and [0,2] on values [10,20].

    The page's result line was lost in extraction; the closed form is 10 + 10*logistic(-2) and
    10 + 10*logistic(2), computed here with scipy's logistic function (not the oracle's route).
    Also pins the default scale 1/sqrt(d_h): d_h = 4 and raw dot products [4, 0] give [2, 0].
    Catches: a dropped or wrong default scale (1/d_h would give scores [1, 0]).
    """
    expected = [10 + 10 * scipy.special.expit(-2.0), 10 + 10 * scipy.special.expit(2.0)]
    assert round(expected[0], 6) == 11.192029 and round(expected[1], 6) == 18.807971
    # d_h = 4: keys (2,0,0,0) and (0,2,0,0); queries (2,0,0,0) -> raw [4,0]; (0,2,0,0) -> [0,4]
    k = np.array([[2, 0, 0, 0], [0, 2, 0, 0]], np.float64).reshape(1, 1, 2, 4)
    v = np.tile(np.array([10.0, 20.0])[:, None], (1, 4)).reshape(1, 1, 2, 4)
    q = np.array([[2, 0, 0, 0], [0, 2, 0, 0]], np.float64).reshape(1, 2, 1, 4)
    O, _ = oracle.attention_ref(q, k, v, q_start=[1])  # default scale
    assert np.allclose(O[0, :, 0, 0], expected, atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------------------------
# Masking by absolute position, padding, errors
# ---------------------------------------------------------------------------------------------

def test_causal_first_row_sees_only_key_zero():
    """Causal mask direction (j > t is invisible): row 0 of a square prefill equals v_0 exactly.

    Catches: mask applied the wrong way (j < t), or no mask.
    """
    rng = np.random.default_rng(1949)
    q = rng.standard_normal((1, 2, 5, 3))
    k = rng.standard_normal((1, 1, 5, 3))
    v = rng.standard_normal((1, 1, 5, 3))
    O, _ = oracle.attention_ref(q, k, v)
    assert np.array_equal(O[0, 0, 0], v[0, 0, 0]) and np.array_equal(O[0, 1, 0], v[0, 0, 0])
    # the last row sees everything: equal to the non-causal result for that row
    Onc, _ = oracle.attention_ref(q, k, v, causal=False)
    assert np.allclose(O[0, :, -1], Onc[0, :, -1], atol=1e-15)


def test_decode_uses_absolute_position():
    """第 09 章 §09.2: a single cached query at position T-1 sees all T keys, not just key 0.

    Catches: the zero-based-template bug (a 1 x T triangular mask that shows only key 0).
    """
    rng = np.random.default_rng(1949)
    T = 7
    q = rng.standard_normal((1, 2, 4))
    k = rng.standard_normal((1, 1, T, 4))
    v = rng.standard_normal((1, 1, T, 4))
    O, _ = oracle.decode_ref(q, k, v)
    full, _ = oracle.attention_ref(q[:, :, None], k, v, causal=False)
    assert np.allclose(O, full[:, :, 0], atol=1e-15)
    assert not np.allclose(O[0, 0], v[0, 0, 0])
    # with q_pos = 0 the query sees key 0 only
    O0, _ = oracle.decode_ref(q, k, v, q_pos=[0])
    assert np.array_equal(O0[0, 0], v[0, 0, 0])


def test_padding_tail_never_read():
    """Keys at or beyond kv_len are invisible and never read: a NaN tail leaves outputs finite and
    equal to the computation on the truncated cache."""
    rng = np.random.default_rng(5)
    k = rng.standard_normal((2, 2, 9, 4))
    v = rng.standard_normal((2, 2, 9, 4))
    q = rng.standard_normal((2, 4, 4))
    lens = np.array([3, 9])
    k2, v2 = k.copy(), v.copy()
    k2[0, :, 3:] = np.nan
    v2[0, :, 3:] = np.nan
    O, _ = oracle.decode_ref(q, k2, v2, kv_len=lens)
    assert np.isfinite(O).all()
    Ot, _ = oracle.decode_ref(q[:1], k[:1, :, :3], v[:1, :, :3])
    assert np.array_equal(O[0], Ot[0])


def test_no_visible_key_is_an_error():
    """序列计算与存储 §两块算例: a query with no visible key raises."""
    k = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_ref(np.zeros((1, 1, 1, 2)), k, k, kv_len=[0])
    with pytest.raises(ValueError):
        oracle.online_softmax_row(np.array([-np.inf, -np.inf]), np.ones(2), block=1)
    with pytest.raises(ValueError):
        oracle.group_of(0, 6, 4)


def test_chunked_prefill_equals_rows_of_full_prefill():
    """Queries at absolute positions q_start.. over a longer cache equal the matching rows of a
    full causal prefill (the offset mask is bottom-right aligned by position)."""
    rng = np.random.default_rng(11)
    T, start = 12, 8
    q = rng.standard_normal((1, 4, T, 8))
    k = rng.standard_normal((1, 2, T, 8))
    v = rng.standard_normal((1, 2, T, 8))
    full, lf = oracle.attention_ref(q, k, v)
    part, lp = oracle.attention_ref(q[:, :, start:], k, v, q_start=[start])
    assert np.array_equal(part, full[:, :, start:]) and np.array_equal(lp, lf[:, :, start:])


# ---------------------------------------------------------------------------------------------
# Group mapping
# ---------------------------------------------------------------------------------------------

def test_group_map_page_cases():
    for case in GOLDEN["group_map"]["cases"]:
        if "groups" in case:
            assert [oracle.group_of(a, case["h_q"], case["h_kv"]) for a in range(case["h_q"])] == case["groups"]
        elif "groups_first8" in case:
            assert [oracle.group_of(a, case["h_q"], case["h_kv"]) for a in range(8)] == case["groups_first8"]
        else:
            assert oracle.group_of(case["head"], case["h_q"], case["h_kv"]) == case["group"]


def test_gqa_equals_mha_on_adjacent_expansion_and_detects_interleaved():
    """第 09 章 §09.2 / §09.6: GQA equals MHA on K/V expanded A,A,B,B (error exactly 0 in fp64);
    the wrong expansion A,B,A,B is detected.  Catches: g(a) = a % h_kv."""
    rng = np.random.default_rng(1949)
    B, h_q, h_kv, T, d = 2, 6, 2, 10, 5
    q = rng.standard_normal((B, h_q, T, d))
    k = rng.standard_normal((B, h_kv, T, d))
    v = rng.standard_normal((B, h_kv, T, d))
    O, _ = oracle.attention_ref(q, k, v)
    r = h_q // h_kv
    O_mha, _ = oracle.attention_ref(q, np.repeat(k, r, axis=1), np.repeat(v, r, axis=1))
    assert np.array_equal(O, O_mha)
    O_bad, _ = oracle.attention_ref(q, np.tile(k, (1, r, 1, 1)), np.tile(v, (1, r, 1, 1)))
    assert np.abs(O_bad - O).max() > 0.1


def test_h_kv_equals_h_q_is_per_head_attention():
    """h_kv = h_q is MHA: each head equals a single-head computation with its own K/V."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 3, 6, 4))
    k = rng.standard_normal((1, 3, 6, 4))
    v = rng.standard_normal((1, 3, 6, 4))
    O, _ = oracle.attention_ref(q, k, v)
    for a in range(3):
        Oa, _ = oracle.attention_ref(q[:, a:a + 1], k[:, a:a + 1], v[:, a:a + 1])
        assert np.array_equal(O[:, a], Oa[:, 0])


# ---------------------------------------------------------------------------------------------
# Independent library routine: torch's scaled_dot_product_attention on repeat_interleave'd K/V
# (the comparator shape the pages' 第三章 §3.3 snippet uses), fp64 on the CPU.
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("h_q,h_kv", [(4, 2), (8, 8), (8, 1), (6, 3)])
def test_matches_torch_sdpa_square_causal(h_q, h_kv):
    rng = np.random.default_rng(h_q * 10 + h_kv)
    B, T, d = 2, 33, 16
    q = rng.standard_normal((B, h_q, T, d))
    k = rng.standard_normal((B, h_kv, T, d))
    v = rng.standard_normal((B, h_kv, T, d))
    O, _ = oracle.attention_ref(q, k, v)
    r = h_q // h_kv
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(r, dim=1), tv.repeat_interleave(r, dim=1), is_causal=True
    ).numpy()
    assert np.abs(O - ref).max() < 1e-12


def test_matches_torch_sdpa_offset_mask_and_lengths():
    """Absolute-position mask with q_start > 0 and per-sequence lengths, against SDPA with an
    explicit boolean mask built from the same visibility rule."""
    rng = np.random.default_rng(7)
    B, h_q, h_kv, S_q, T, d = 2, 4, 2, 5, 20, 8
    q = rng.standard_normal((B, h_q, S_q, d))
    k = rng.standard_normal((B, h_kv, T, d))
    v = rng.standard_normal((B, h_kv, T, d))
    q_start = np.array([10, 3])
    kv_len = np.array([14, 20])
    O, _ = oracle.attention_ref(q, k, v, q_start=q_start, kv_len=kv_len, scale=0.3)
    for b in range(B):
        j = np.arange(T)
        pos = q_start[b] + np.arange(S_q)
        mask = (j[None, :] <= pos[:, None]) & (j[None, :] < kv_len[b])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b:b + 1]),
            torch.from_numpy(np.repeat(k[b:b + 1], 2, axis=1)),
            torch.from_numpy(np.repeat(v[b:b + 1], 2, axis=1)),
            attn_mask=torch.from_numpy(mask), scale=0.3,
        ).numpy()
        assert np.abs(O[b:b + 1] - ref).max() < 1e-12


# ---------------------------------------------------------------------------------------------
# Invariants and special cases
# ---------------------------------------------------------------------------------------------

def test_invariants():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 4, 9, 6))
    k = rng.standard_normal((1, 2, 9, 6))
    v = rng.standard_normal((1, 2, 9, 6))
    # constant values -> constant output
    O, lse = oracle.attention_ref(q, k, np.full_like(v, 3.25))
    assert np.allclose(O, 3.25, atol=1e-14)
    # output inside the per-channel range of the visible values (convex combination)
    O, lse = oracle.attention_ref(q, k, v)
    for a in range(4):
        g = a // 2
        for i in range(9):
            vis = v[0, g, : i + 1]
            assert (O[0, a, i] >= vis.min(0) - 1e-12).all() and (O[0, a, i] <= vis.max(0) + 1e-12).all()
    # weights sum to one: sum_j exp(s_j - lse) = 1 on each row
    for a in range(4):
        g = a // 2
        S = (q[0, a] @ k[0, g].T) / math.sqrt(6)
        S = np.where(np.tril(np.ones((9, 9), bool)), S, -np.inf)
        assert np.allclose(np.exp(S - lse[0, a][:, None]).sum(1), 1.0, atol=1e-14)
    # zero query -> plain mean of the visible values
    O0, _ = oracle.attention_ref(np.zeros_like(q), k, v)
    for i in range(9):
        assert np.allclose(O0[0, 0, i], v[0, 0, : i + 1].mean(0), atol=1e-14)


def test_large_scores_are_stable():
    """Without the max subtraction exp(1000) overflows; the oracle must give v_0 exactly."""
    q = np.array([[[[1.0]]]])
    k = np.array([1000.0, 0.0]).reshape(1, 1, 2, 1)
    v = np.array([1.5, 3.0]).reshape(1, 1, 2, 1)
    O, lse = oracle.attention_ref(q, k, v, q_start=[1], scale=1.0)
    assert O[0, 0, 0, 0] == 1.5 and lse[0, 0, 0] == 1000.0


def test_key_permutation_invariance_non_causal():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 2, 3, 4))
    k = rng.standard_normal((1, 1, 7, 4))
    v = rng.standard_normal((1, 1, 7, 4))
    p = rng.permutation(7)
    O1, l1 = oracle.attention_ref(q, k, v, causal=False)
    O2, l2 = oracle.attention_ref(q, k[:, :, p], v[:, :, p], causal=False)
    assert np.allclose(O1, O2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)


def test_blockwise_split_path_equals_definition():
    """The split-KV reduction (several splits, several block sizes) reaches the plain result."""
    rng = np.random.default_rng(1949)
    T, d = 37, 8
    q = rng.standard_normal(d)
    k = rng.standard_normal((T, d))
    v = rng.standard_normal((T, d))
    ref, lref = oracle.head_attention(q[None], k, v, [T - 1], T, 0.35)
    for block in (1, 4, 16, 64):
        for n_splits in (1, 2, 3, 7):
            o, lse = oracle.blockwise_attention_row(q, k, v, T - 1, T, 0.35, block, n_splits)
            assert np.abs(o - ref[0]).max() < 1e-13 and abs(lse - lref[0]) < 1e-13


def test_brute_force_tiny_grid():
    """Pure-Python scalar loops on tiny shapes (an independent, element-by-element route)."""
    rng = np.random.default_rng(1949)
    for (B, h_q, h_kv, S_q, T, d, q0) in [(1, 2, 1, 3, 3, 2, 0), (2, 4, 2, 2, 5, 3, 3), (1, 3, 3, 4, 6, 1, 1)]:
        q = rng.standard_normal((B, h_q, S_q, d))
        k = rng.standard_normal((B, h_kv, T, d))
        v = rng.standard_normal((B, h_kv, T, d))
        O, _ = oracle.attention_ref(q, k, v, q_start=[q0] * B, scale=0.7)
        r = h_q // h_kv
        for b in range(B):
            for a in range(h_q):
                g = a // r
                for i in range(S_q):
                    n = min(T, q0 + i + 1)
                    s = [0.7 * sum(q[b, a, i, t] * k[b, g, j, t] for t in range(d)) for j in range(n)]
                    mx = max(s)
                    w = [math.exp(x - mx) for x in s]
                    z = sum(w)
                    for c in range(d):
                        ref = sum(w[j] * v[b, g, j, c] for j in range(n)) / z
                        assert abs(O[b, a, i, c] - ref) < 1e-13


# ---------------------------------------------------------------------------------------------
# kv_append
# ---------------------------------------------------------------------------------------------

def test_kv_append_ref_bit_exact():
    rng = np.random.default_rng(4)
    k = rng.integers(0, 65535, size=(2, 3, 10, 4), dtype=np.uint16)
    v = rng.integers(0, 65535, size=(2, 3, 10, 4), dtype=np.uint16)
    kn = rng.integers(0, 65535, size=(2, 3, 2, 4), dtype=np.uint16)
    vn = rng.integers(0, 65535, size=(2, 3, 2, 4), dtype=np.uint16)
    k2, v2 = oracle.kv_append_ref(k, v, kn, vn, [0, 8])
    assert np.array_equal(k2[0, :, 0:2], kn[0]) and np.array_equal(v2[1, :, 8:10], vn[1])
    mask = np.ones(k.shape, bool)
    mask[0, :, 0:2] = False
    mask[1, :, 8:10] = False
    assert np.array_equal(k2[mask], k[mask]) and np.array_equal(v2[mask], v[mask])
    with pytest.raises(ValueError):
        oracle.kv_append_ref(k, v, kn, vn, [0, 9])
    with pytest.raises(ValueError):
        oracle.kv_append_ref(k, v, kn, vn, [-1, 0])


# ---------------------------------------------------------------------------------------------
# Ledgers
# ---------------------------------------------------------------------------------------------

def test_cache_byte_ledgers():
    for key in ("cache_bytes", "kv_bytes_ch09"):
        for c in GOLDEN[key]["cases"]:
            assert ledgers.kv_cache_bytes(c["L"], c["B"], c["T"], c["h_kv"], c["d_h"], c["s"]) == c["bytes"]
    c7 = GOLDEN["kv_bytes_7b"]["cases"]
    assert ledgers.kv_cache_bytes(**{k: c7[0][k] for k in ("L", "B", "T", "h_kv", "d_h", "s")}) == c7[0]["bytes"]
    assert round(ledgers.kv_cache_bytes(**{k: c7[1][k] for k in ("L", "B", "T", "h_kv", "d_h", "s")}) / 1e9, 2) == c7[1]["bytes_approx_gb"]
    # equals the bytes of an allocated (B, h_kv, T, d_h) K and V pair times L
    k = np.zeros((1, 2, 3, 2), np.float16)
    assert 2 * (k.nbytes + k.nbytes) == 96
    assert ledgers.kv_ratio_vs_mha(4, 2) == 0.5


def test_per_token_and_intensity_ledger():
    g = GOLDEN["per_token_and_8k_ledger"]
    for row in g["rows"]:
        assert ledgers.kv_bytes_per_token_layer(row["h_kv"], g["d_h"], g["s"]) == row["per_token_bytes"]
        assert ledgers.kv_cache_bytes(1, 1, g["T"], row["h_kv"], g["d_h"], g["s"]) == row["per_layer_8k_bytes"]
        assert ledgers.kv_read_intensity(g["h_q"], row["h_kv"], g["d_h"], g["s"], g["T"]) == row["intensity"]
    assert ledgers.kv_cache_bytes(32, 1, g["T"], 32, g["d_h"], g["s"]) == g["mha_32_layers_8k_bytes"]
    assert ledgers.decode_flops(g["h_q"], g["T"], g["d_h"]) == g["decode_flops"]


def test_projection_params():
    g = GOLDEN["projection_params"]
    for c in g["cases"]:
        assert ledgers.projection_params(g["d"], g["h_q"], c["h_kv"], g["d_h"]) == c["params"]


def test_score_memory_and_tile_ledger():
    g = GOLDEN["score_memory"]
    assert ledgers.score_tensor_elements(1, 4, 1024) == g["full_elements_B1_hq4_T1024"]
    assert ledgers.score_tensor_elements(1, 4, 1024) * 4 == g["full_bytes_fp32"]
    assert 64 * 64 == g["block64_elements"] and 64 * 64 * 4 == g["block64_bytes_fp32"]
    assert ledgers.score_tensor_elements(1, 1, 4096) * 2 == g["fp16_N4096_bytes"]
    assert ledgers.score_tensor_elements(1, 1, 32768) * 2 == g["fp16_N32768_bytes"]
    assert ledgers.kv_cache_bytes(1, 1, 256, 1, 128, 2) == GOLDEN["tile_bytes"]["bytes"]


def test_prefill_flop_ledger_closed_form():
    """4 d_h per visible pair; square causal: T (T + 1) / 2 pairs per head."""
    assert ledgers.prefill_visible_pairs(256, 0, 256) == 256 * 257 // 2
    assert ledgers.prefill_flops(1, 4, 64, 256, 0, 256) == 4 * 4 * 64 * (256 * 257 // 2)
    assert ledgers.prefill_flops(1, 32, 128, 4096, 0, 4096) == 137_472_507_904
    # chunked: 512 queries at 32256.., each sees q_start + i + 1 keys
    assert ledgers.prefill_visible_pairs(512, 32256, 32768) == sum(32257 + i for i in range(512))
    assert ledgers.prefill_flops(1, 32, 128, 512, 32256, 32768) == 272_734_617_600
