"""Pins for the MLA oracle: the absorbed decode (scores against the latent cache, latent output
up-projected afterwards) equals the explicit one (rebuild K and V per head, ordinary attention) by
associativity [第 09 章 §09.3: the pages record a largest difference of 1.78e-15 for their
check]; the value rows are the latent's first c columns; the cache ledger follows the page's
example (H d = 512, c = 128: 1024 numbers per token become 128)."""

import numpy as np
import pytest

import oracle
from oracle import mla


def _weights(rng, c, h, d):
    return rng.standard_normal((c, h * d)) / np.sqrt(c), rng.standard_normal((c, h * d)) / np.sqrt(c)


@pytest.mark.parametrize("h,d,c,d_r", [(4, 16, 24, 8), (8, 32, 48, 16), (2, 8, 64, 0)])
def test_absorbed_equals_explicit(h, d, c, d_r):
    rng = np.random.default_rng(h * 100 + c)
    B, T = 2, 23
    x = rng.standard_normal((B, T, 40))
    w_d = rng.standard_normal((40, c)) / np.sqrt(40)
    C = x @ w_d                                   # latent cache C = X W_D
    kr = rng.standard_normal((B, T, d_r))
    w_uk, w_uv = _weights(rng, c, h, d)
    q_nope = rng.standard_normal((B, h, d))
    q_rope = rng.standard_normal((B, h, d_r))
    kv_len = np.array([23, 9])
    scale = 1.0 / np.sqrt(d + d_r)
    ref = mla.mla_explicit_ref(q_nope, q_rope, C, kr, w_uk, w_uv, kv_len=kv_len, scale=scale)
    q = np.concatenate([mla.absorb_query(q_nope, w_uk), q_rope], axis=2)
    cache = np.concatenate([C, kr], axis=2)
    o_lat, _ = mla.mla_decode_ref(q, cache, c, kv_len=kv_len, scale=scale)
    got = mla.up_project(o_lat, w_uv)
    assert np.abs(got - ref).max() < 1e-12


def test_latent_output_is_a_convex_combination_of_latent_rows():
    rng = np.random.default_rng(5)
    B, h, T, c, d_r = 1, 3, 11, 6, 2
    cache = rng.standard_normal((B, T, c + d_r))
    q = rng.standard_normal((B, h, c + d_r))
    o, lse = mla.mla_decode_ref(q, cache, c, scale=0.3)
    # weights recovered from lse reproduce o from the first c columns only
    s = (q[0] @ cache[0].T) * 0.3
    w = np.exp(s - lse[0][:, None])
    assert np.allclose(w.sum(axis=1), 1.0)
    assert np.allclose(o[0], w @ cache[0, :, :c])
    # one visible token: the output is that token's latent
    o1, _ = mla.mla_decode_ref(q, cache, c, q_pos=[0], scale=0.3)
    assert np.allclose(o1[0], np.broadcast_to(cache[0, 0, :c], (h, c)))


def test_equals_gqa_oracle_with_one_kv_head():
    """With d_r = 0 and the value taken as the whole row, MLA decode is MQA decode (h_kv = 1)."""
    rng = np.random.default_rng(6)
    B, h, T, c = 2, 4, 13, 8
    cache = rng.standard_normal((B, T, c))
    q = rng.standard_normal((B, h, c))
    kv_len = np.array([13, 5])
    o, lse = mla.mla_decode_ref(q, cache, c, kv_len=kv_len)
    o2, lse2 = oracle.decode_ref(q, cache[:, None], cache[:, None], kv_len=kv_len)
    assert np.allclose(o, o2, atol=1e-14) and np.allclose(lse, lse2, atol=1e-14)


def test_cache_ledger_page_example():
    # H d = 512 per K and per V: 1024 numbers per token; latent c = 128 (no rotary part in the
    # page's teaching version)
    assert 2 * 512 == 1024
    assert mla.mla_cache_elements_per_token(128) == 128
    # DeepSeek-style latent 512 + rotary 64
    assert mla.mla_cache_elements_per_token(512, 64) == 576
