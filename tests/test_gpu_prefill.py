"""bf16 tcgen05 prefill on the GPU against the fp64 oracle (max |d| <= 2e-2, mean |d| <= 2e-3)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_bf16_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


def _run(B, h_q, h_kv, S_q, T, d, q_start, kv_len, causal=True, seed=0, nan_tail=False, std=1.0):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PrefillShape(B=B, h_q=h_q, h_kv=h_kv, S_q=S_q, T_max=T, d_h=d, q_start=0,
                                   kv_len=T, std=std)
    q, k, v = workloads.prefill_inputs(shape, seed=seed)
    if nan_tail:
        for b in range(B):
            k[b, :, kv_len[b]:] = float("nan")
            v[b, :, kv_len[b]:] = float("nan")
    o, lse = gqa.prefill(q.cuda(), k.cuda(), v.cuda(), q_start=list(q_start), kv_len=list(kv_len),
                         causal=causal, return_lse=True)
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v), q_start=q_start, kv_len=kv_len,
                                     causal=causal)
    assert_bf16_close(_f64(o), ref, f"prefill B={B} h_q={h_q} h_kv={h_kv} S_q={S_q} T={T} d={d}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
    assert gqa.get_device_error() == 0


def test_prefill_small_workload():
    """prefill_small: B=1, h_q=4, h_kv=2, T=256, d_h=64, causal, N(0,1)."""
    _run(1, 4, 2, 256, 256, 64, [0], [256])


@pytest.mark.parametrize("h_q,h_kv", [(4, 4), (8, 4), (16, 4), (32, 4), (6, 2), (8, 1)])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_group_widths_ragged(h_q, h_kv, d):
    # S_q not a multiple of any tile; kv_len not a multiple of the 128-key block
    _run(2, h_q, h_kv, 77, 200, d, [0, 50], [77, 127], seed=h_q + d)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_offset_and_nan_tail(d):
    # queries at absolute positions q_start.. over a longer cache; keys past kv_len are NaN
    _run(2, 8, 2, 130, 600, d, [300, 460], [431, 590], seed=7, nan_tail=True)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_rows_before_a_chains_first_block(d):
    # Few tiles, so each CTA runs one tile with its K/V blocks alternating between two chains. With
    # r=1 a tile holds 128 positions; from position 50 it spans key blocks 0 and 1, so the rows
    # before position 128 see no key of the second chain's first block (their running maximum is
    # still -inf there) and must take nothing from it.
    _run(1, 2, 2, 200, 300, d, [50], [250], seed=13)
    _run(2, 4, 4, 180, 400, d, [100, 0], [280, 180], seed=14)


@pytest.mark.parametrize("h_q,h_kv,S_q,T", [
    (64, 2, 37, 150),    # r=32: tiles of 4 positions x 32 heads; few CTAs (one tile each)
    (64, 1, 23, 90),     # r=64: 2 positions per tile
    (128, 1, 300, 300),  # r=128: 1 position per tile; 150 pairs of tiles (pair mode)
    (256, 1, 9, 140),    # r=256: two 128-head blocks per group
    (8, 2, 1, 77),       # a single query row
])
def test_prefill_wide_groups_and_tiny_tiles(h_q, h_kv, S_q, T):
    _run(1, h_q, h_kv, S_q, T, 128, [T - S_q], [T], seed=h_q + S_q)


def test_prefill_many_sequences_offsets_and_lengths():
    """B=6 with per-sequence query offsets and lengths (pair mode: enough tiles for every SM)."""
    rng = np.random.default_rng(5)
    kv = rng.integers(200, 600, size=6)
    qs = np.maximum(kv - 180, 0) - rng.integers(0, 20, size=6).clip(0, None)
    qs = np.maximum(qs, 0)
    _run(6, 16, 4, 180, 600, 128, qs.tolist(), kv.tolist(), seed=8, nan_tail=True)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_persistent_walk_mha_ragged(d):
    """More pairs than SMs, so each CTA walks several items: r=1 (tiles of 128 positions, so the
    second tile of a pair sees one more key block than the first and the first chain passes that
    block over), an odd tile count (items with one tile), per-sequence offsets and lengths, and
    NaN past every length."""
    rng = np.random.default_rng(17)
    kv = rng.integers(650, 900, size=8)
    qs = (kv - 600 - rng.integers(0, 40, size=8)).clip(0, None)
    _run(8, 8, 8, 600, 900, d, qs.tolist(), kv.tolist(), seed=21 + d, nan_tail=True)


def test_prefill_persistent_walk_many_single_block_items():
    """256 items of one K/V block each (64 short prompts x 4 groups): consecutive one-block items
    on every CTA, where the chains' turn-taking has no waits at the start of each item."""
    rng = np.random.default_rng(19)
    kv = rng.integers(40, 128, size=64)
    _run(64, 16, 4, 40, 128, 128, (kv - 40).tolist(), kv.tolist(), seed=23, nan_tail=True)


def test_prefill_not_causal():
    _run(1, 8, 2, 100, 300, 128, [0], [260], causal=False, seed=3)


def test_prefill_4k_full_size():
    """prefill_4k at full size (B=1, h_q=32, h_kv=8, T=4096, d_h=128, N(0,1)*0.5), in the bench's
    launch configuration; every output (all 32 heads, all 4096 rows) and every lse against the
    oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(shape, seed=0, device="cuda")
    o, lse = gqa.prefill(q, k, v, return_lse=True)
    assert gqa.get_device_error() == 0
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v))
    assert_bf16_close(_f64(o), ref, "prefill_4k, every head")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2


def test_chunked_prefill_full_size():
    """chunked_prefill: kv_append of 512 new K/V rows at 32256, then prefill of the 512 queries at
    absolute positions 32256.. over T=32768; every output of all 32 heads against the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.CHUNKED_PREFILL
    k, v, k_new, v_new, q = workloads.chunked_prefill_inputs(shape, seed=0, device="cuda")
    gqa.kv_append(k, v, k_new, v_new, [shape.q_start])
    o, lse = gqa.prefill(q, k, v, q_start=[shape.q_start], kv_len=[shape.kv_len], return_lse=True)
    assert gqa.get_device_error() == 0
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v), q_start=[shape.q_start], kv_len=[shape.kv_len])
    assert_bf16_close(_f64(o), ref, "chunked prefill, every head")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2


def test_prefill_equals_rows_of_decode():
    """The last prefill row equals a decode of the same query at position T-1."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PrefillShape(B=2, h_q=16, h_kv=4, S_q=300, T_max=300, d_h=128, q_start=0, kv_len=300)
    q, k, v = workloads.prefill_inputs(shape, seed=11, device="cuda")
    o = gqa.prefill(q, k, v)
    od = gqa.decode(q[:, :, -1].contiguous(), k, v)
    assert (o[:, :, -1].float() - od.float()).abs().max().item() < 2e-2
