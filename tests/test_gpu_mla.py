"""MLA decode (gqa_mla_decode) on the GPU against the fp64 oracle: the latent output of every
head over the shared latent cache rows (bf16: max |d| <= 2e-2, mean |d| <= 2e-3; fp32 check mode
1e-5 relative), lse, and the end-to-end absorbed path against the explicit per-head MLA."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_bf16_close, assert_fp32_close
from oracle import mla as mla_ref

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


@pytest.mark.parametrize("h_q", [16, 8, 32, 128])
def test_mla_decode_bf16(h_q):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=3, h_q=h_q, T_max=700)
    lens = [700, 333, 1]
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=h_q, lengths=lens)
    ref, lref = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=np.array(lens), scale=shape.scale)
    for splits in (1, 7, 0):
        o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), kv_len=lens, scale=shape.scale, num_splits=splits,
                                return_lse=True)
        assert_bf16_close(_f64(o), ref, f"mla h_q={h_q} splits={splits}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
        assert gqa.get_device_error() == 0
    # one visible token: every head's output is that token's latent
    assert torch.equal(o[2].cpu(), cache[2, 0, :512].expand(h_q, 512))


def test_mla_decode_query_position_inside_the_cache():
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=2, h_q=16, T_max=1000)
    q, cache, _ = workloads.mla_decode_inputs(shape, seed=3, nan_tail=False)
    q_pos = np.array([0, 611], np.int32)
    ref, _ = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, q_pos=q_pos, scale=shape.scale)
    o = gqa.mla_decode(q.cuda(), cache.cuda(), q_pos=q_pos.tolist(), scale=shape.scale, num_splits=5)
    assert_bf16_close(_f64(o), ref, "mla q_pos")


@pytest.mark.parametrize("d_qk,d_v", [(576, 512), (40, 32), (100, 100)])
def test_mla_decode_fp32_check_mode(d_qk, d_v):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=2, h_q=20, T_max=300, d_qk=d_qk, d_v=d_v)
    lens = [300, 77]
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=d_qk, dtype=torch.float32, lengths=lens)
    ref, lref = mla_ref.mla_decode_ref(_f64(q), _f64(cache), d_v, kv_len=np.array(lens), scale=0.07)
    o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), d_v, kv_len=lens, scale=0.07, num_splits=4, return_lse=True)
    assert_fp32_close(_f64(o), ref, f"fp32 mla {d_qk}/{d_v}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 1e-4
    assert gqa.get_device_error() == 0


def test_mla_absorbed_path_equals_explicit_heads():
    """End to end: absorb the query on the host, run the latent decode on the GPU, up-project on
    the host; compare with the explicit MLA that rebuilds K_h = [C U_K^h, kr] and V_h = C U_V^h."""
    import kv_cache_attention_gqa_b200 as gqa

    rng = np.random.default_rng(0)
    B, h, T, d, c, d_r = 2, 16, 500, 128, 512, 64
    C = rng.standard_normal((B, T, c)) * 0.5
    kr = rng.standard_normal((B, T, d_r))
    w_uk = rng.standard_normal((c, h * d)) / np.sqrt(c)
    w_uv = rng.standard_normal((c, h * d)) / np.sqrt(c)
    q_nope = rng.standard_normal((B, h, d))
    q_rope = rng.standard_normal((B, h, d_r))
    scale = 1.0 / np.sqrt(d + d_r)
    lens = np.array([500, 123])
    # bf16 inputs seen by both sides
    q_lat = torch.tensor(np.concatenate([mla_ref.absorb_query(q_nope, w_uk), q_rope], axis=2)).to(torch.bfloat16)
    cache = torch.tensor(np.concatenate([C, kr], axis=2)).to(torch.bfloat16)
    o_lat = gqa.mla_decode(q_lat.cuda(), cache.cuda(), kv_len=lens.tolist(), scale=scale)
    got = mla_ref.up_project(_f64(o_lat), w_uv)
    # the explicit form on the same (bf16-rounded) latent, rotary key and absorbed query
    cache64 = _f64(cache)
    ref_lat, _ = mla_ref.mla_decode_ref(_f64(q_lat), cache64, c, kv_len=lens, scale=scale)
    ref = mla_ref.up_project(ref_lat, w_uv)
    assert np.abs(got - ref).max() <= 2e-2 * max(1.0, np.abs(ref).max())
    # and the explicit per-head computation agrees with the absorbed one in fp64
    explicit = mla_ref.mla_explicit_ref(q_nope, q_rope, C, kr, w_uk, w_uv, kv_len=lens, scale=scale)
    absorbed = mla_ref.up_project(mla_ref.mla_decode_ref(
        np.concatenate([mla_ref.absorb_query(q_nope, w_uk), q_rope], axis=2), np.concatenate([C, kr], axis=2),
        c, kv_len=lens, scale=scale)[0], w_uv)
    assert np.abs(explicit - absorbed).max() < 1e-11


@pytest.mark.parametrize("h_q", [16, 128])
def test_mla_decode_8k_full_size(h_q):
    """B=8, T=8192, 576-wide rows, automatic splits (the bench's configuration), every output."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MLA_DECODE[h_q]
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=0, device="cuda")
    o = gqa.mla_decode(q, cache, kv_len=kl, scale=shape.scale)
    assert gqa.get_device_error() == 0
    ref, _ = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=kl.cpu().numpy(), scale=shape.scale)
    assert_bf16_close(_f64(o), ref, f"mla decode_8k h_q={h_q}")


@pytest.mark.parametrize("splits", [3, 0])
def test_mla_decode_bf16_two_units_per_sequence(splits):
    """256 heads: two 128-head units per sequence on the tensor-core kernel, ragged lengths with
    NaN past each, chunks that cut through units and sequences."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=2, h_q=256, T_max=1500)
    lens = [1500, 901]
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=256 + splits, lengths=lens)
    ref, lref = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=np.array(lens), scale=shape.scale)
    o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), kv_len=lens, scale=shape.scale, num_splits=splits,
                            return_lse=True)
    assert gqa.get_device_error() == 0
    assert_bf16_close(_f64(o), ref, f"mla h_q=256 splits={splits}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2


def test_mla_decode_128_heads_query_position_inside_the_cache():
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=3, h_q=128, T_max=1000)
    q, cache, _ = workloads.mla_decode_inputs(shape, seed=5, nan_tail=False)
    q_pos = np.array([0, 611, 64], np.int32)
    ref, _ = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, q_pos=q_pos, scale=shape.scale)
    for splits in (5, 0):
        o = gqa.mla_decode(q.cuda(), cache.cuda(), q_pos=q_pos.tolist(), scale=shape.scale, num_splits=splits)
        assert gqa.get_device_error() == 0
        assert_bf16_close(_f64(o), ref, f"mla 128 heads q_pos splits={splits}")


def test_mla_decode_128_heads_equal_lengths_aligned_chunks():
    """Every sequence at the same length (1000 keys, 4 sequences): the automatic plan cuts each
    unit into equal chunks that never straddle two sequences (here 2 chunks of 500 keys each, not
    16 of 256), so every CTA pair has one piece and every row two partials."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=4, h_q=128, T_max=1000)
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=11)
    ref, lref = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=kl.numpy(), scale=shape.scale)
    o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), kv_len=kl.cuda(), scale=shape.scale, return_lse=True)
    assert gqa.get_device_error() == 0
    assert_bf16_close(_f64(o), ref, "mla 128 heads, equal lengths")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2


def test_mla_decode_128_heads_more_chunks_than_pairs():
    """200 explicit splits of 2 ragged sequences (NaN past each length) on the tensor-core kernel:
    more chunks than CTA pairs, so each pair walks several chunks in turn, every chunk a piece of
    its own with a query copy, early tiles and a partial epilogue, and rows merge up to ~120
    partials."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.MlaShape(B=2, h_q=128, T_max=2500)
    lens = [2500, 1733]
    q, cache, kl = workloads.mla_decode_inputs(shape, seed=57, lengths=lens)
    ref, lref = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=np.array(lens), scale=shape.scale)
    for rep in range(2):
        o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), kv_len=lens, scale=shape.scale, num_splits=200,
                                return_lse=True)
        assert gqa.get_device_error() == 0
        assert_bf16_close(_f64(o), ref, f"mla 128 heads, 200 splits, call {rep}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2


def test_mla_decode_128_heads_many_short_sequences_and_an_empty_one():
    """40 sequences of 1-120 visible keys on the tensor-core kernel: chunks of at least 256 keys hold
    several sequences each, so a CTA pair runs piece after piece (its next piece's tiles issued
    early, its query copied before the previous piece's epilogue). One sequence has kv_len = 0: its
    rows are zeros with lse = -inf and the device error reads GQA_DEVERR_KV_LEN; every other row
    matches the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    rng = np.random.default_rng(61)
    B, bad = 40, 17
    lens = rng.integers(1, 121, size=B).astype(np.int32)
    lens[bad] = 0
    shape = workloads.MlaShape(B=B, h_q=128, T_max=120)
    q, cache, _ = workloads.mla_decode_inputs(shape, seed=61, lengths=lens)
    o, lse = gqa.mla_decode(q.cuda(), cache.cuda(), kv_len=lens.tolist(), scale=shape.scale, return_lse=True)
    assert gqa.get_device_error() == 1  # GQA_DEVERR_KV_LEN
    assert o[bad].abs().sum().item() == 0 and torch.isneginf(lse[bad]).all()
    keep = [b for b in range(B) if b != bad]
    ref, lref = mla_ref.mla_decode_ref(_f64(q[keep]), _f64(cache[keep]), 512, kv_len=lens[keep], scale=shape.scale)
    assert_bf16_close(_f64(o[keep]), ref, "mla 128 heads, 39 short sequences")
    assert np.abs(lse[keep].cpu().double().numpy() - lref).max() < 2e-2
