"""Sliding-window attention on the GPU against the oracle (a row at position p sees keys
p - W < j <= p [第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.7]).

Rows below each window are overwritten with NaN in the copy the GPU reads (the oracle reads the
finite original), and on a paged cache the block-table entries of pages wholly below the window
are -1: a kernel that read outside the window would produce NaN or a page error.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_bf16_close, assert_fp32_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


def _poison_below(cache, lo):
    """Copy of a (B, h_kv, T, d) cache with rows j < lo[b] set to NaN."""
    c = cache.clone()
    for b, n in enumerate(lo):
        if n > 0:
            c[b, :, :int(n)] = float("nan")
    return c


# ------------------------------------------------------------------------------------ prefill

@pytest.mark.parametrize("W", [1, 17, 128, 130, 300, 10_000])
@pytest.mark.parametrize("h_q,h_kv,d", [(4, 2, 64), (32, 8, 128), (8, 8, 128), (16, 1, 64)])
def test_prefill_window_bf16(W, h_q, h_kv, d):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PrefillShape(B=2, h_q=h_q, h_kv=h_kv, S_q=520, T_max=520, d_h=d, q_start=0,
                                   kv_len=520)
    q, k, v = workloads.prefill_inputs(shape, seed=W + h_q)
    o, lse = gqa.prefill(q.cuda(), k.cuda(), v.cuda(), window=W, return_lse=True)
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v), window=W)
    assert_bf16_close(_f64(o), ref, f"prefill W={W} h_q={h_q} h_kv={h_kv} d={d}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
    assert gqa.get_device_error() == 0


@pytest.mark.parametrize("W", [1, 64, 200])
def test_prefill_window_offset_ragged_nan_outside(W):
    """Chunked prefill (queries at q_start..q_start+S_q-1) with ragged kv_len; keys below every
    row's window and past kv_len are NaN in the GPU's copy."""
    import kv_cache_attention_gqa_b200 as gqa

    B, h_q, h_kv, S_q, T, d = 3, 8, 2, 256, 1024, 128
    g = torch.Generator().manual_seed(W)
    q = torch.randn(B, h_q, S_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16)
    q_start = np.array([0, 500, 768], np.int32)
    kv_len = q_start + S_q
    lo = np.maximum(0, q_start - W + 1)  # the earliest row's window start
    kp, vp = _poison_below(k, lo), _poison_below(v, lo)
    for b in range(B):
        kp[b, :, kv_len[b]:] = float("nan")
        vp[b, :, kv_len[b]:] = float("nan")
    o = gqa.prefill(q.cuda(), kp.cuda(), vp.cuda(), q_start=q_start.tolist(), kv_len=kv_len.tolist(), window=W)
    ref, _ = oracle.attention_ref(_f64(q), _f64(k), _f64(v), q_start=q_start, kv_len=kv_len, window=W)
    assert_bf16_close(_f64(o), ref, f"offset W={W}")
    assert gqa.get_device_error() == 0


@pytest.mark.parametrize("W", [100, 300])
def test_prefill_window_persistent_walk(W):
    """More pairs than SMs (each CTA walks several items) under a sliding window: r=1 tiles of 128
    positions, per-sequence offsets and lengths, NaN below every sequence's earliest window and
    past its length."""
    import kv_cache_attention_gqa_b200 as gqa

    B, h_q, h_kv, S_q, T, d = 8, 8, 8, 600, 1000, 128
    g = torch.Generator().manual_seed(W + 1)
    q = torch.randn(B, h_q, S_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(W)
    q_start = rng.integers(0, T - S_q + 1, size=B).astype(np.int32)
    kv_len = np.minimum(q_start + S_q + rng.integers(0, 30, size=B), T).astype(np.int32)
    lo = np.maximum(0, q_start - W + 1)
    kp, vp = _poison_below(k, lo), _poison_below(v, lo)
    for b in range(B):
        kp[b, :, kv_len[b]:] = float("nan")
        vp[b, :, kv_len[b]:] = float("nan")
    o = gqa.prefill(q.cuda(), kp.cuda(), vp.cuda(), q_start=q_start.tolist(), kv_len=kv_len.tolist(), window=W)
    ref, _ = oracle.attention_ref(_f64(q), _f64(k), _f64(v), q_start=q_start, kv_len=kv_len, window=W)
    assert_bf16_close(_f64(o), ref, f"persistent walk W={W}")
    assert gqa.get_device_error() == 0


@pytest.mark.parametrize("W", [1, 5, 70])
def test_prefill_window_fp32_check_mode(W):
    import kv_cache_attention_gqa_b200 as gqa

    g = torch.Generator().manual_seed(W)
    B, h_q, h_kv, S_q, T, d = 2, 6, 3, 90, 200, 40
    q = torch.randn(B, h_q, S_q, d, generator=g)
    k = torch.randn(B, h_kv, T, d, generator=g)
    v = torch.randn(B, h_kv, T, d, generator=g)
    q_start = np.array([0, 110], np.int32)
    o, lse = gqa.prefill(q.cuda(), k.cuda(), v.cuda(), q_start=q_start.tolist(),
                         kv_len=(q_start + S_q).tolist(), window=W, return_lse=True)
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v), q_start=q_start, kv_len=q_start + S_q,
                                     window=W)
    assert_fp32_close(_f64(o), ref, f"fp32 W={W}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 1e-4
    assert gqa.get_device_error() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_window_rows_with_no_visible_key(dtype):
    """Rows whose window starts at or past kv_len see nothing: zero output, lse = -inf, device
    error 3; the other rows are unaffected."""
    import kv_cache_attention_gqa_b200 as gqa

    g = torch.Generator().manual_seed(1)
    B, h_q, h_kv, S_q, T, d, W = 1, 4, 2, 32, 64, 64, 5
    q = torch.randn(B, h_q, S_q, d, generator=g).to(dtype)
    k = torch.randn(B, h_kv, T, d, generator=g).to(dtype)
    v = torch.randn(B, h_kv, T, d, generator=g).to(dtype)
    # rows at positions 40..71 over 50 keys: row i sees (35 + i, 40 + i] within [0, 50) -> i < 14
    o, lse = gqa.prefill(q.cuda(), k.cuda(), v.cuda(), q_start=[40], kv_len=[50], window=W, return_lse=True)
    assert gqa.get_device_error() == 3
    assert torch.all(o[:, :, 14:] == 0) and torch.all(lse[:, :, 14:] == float("-inf"))
    ref, _ = oracle.attention_ref(_f64(q[:, :, :14]), _f64(k), _f64(v), q_start=[40], kv_len=[50], window=W)
    got = _f64(o[:, :, :14])
    if dtype == torch.float32:
        assert_fp32_close(got, ref, "visible rows")
    else:
        assert_bf16_close(got, ref, "visible rows")
    # a whole tile without visible keys
    gqa.prefill(q.cuda(), k.cuda(), v.cuda(), q_start=[200], kv_len=[50], window=W)
    assert gqa.get_device_error() == 3


def test_prefill_window_4k_full_size():
    """prefill_4k (h_q=32, h_kv=8, S=T=4096, d_h=128) with a 1024-key window: every output of all
    32 heads against the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(shape, seed=0, device="cuda")
    o = gqa.prefill(q, k, v, window=1024)
    assert gqa.get_device_error() == 0
    ref, _ = oracle.attention_ref(_f64(q), _f64(k), _f64(v), window=1024)
    assert_bf16_close(_f64(o), ref, "prefill_4k W=1024, every head")


# ------------------------------------------------------------------------------------- decode

@pytest.mark.parametrize("W", [1, 16, 100, 1000, 5000])
@pytest.mark.parametrize("h_q,h_kv", [(32, 8), (32, 32), (32, 1), (40, 5)])
def test_decode_window_bf16(W, h_q, h_kv):
    import kv_cache_attention_gqa_b200 as gqa

    B, T, d = 4, 1500, 128
    shape = workloads.DecodeShape(B=B, h_q=h_q, h_kv=h_kv, T_max=T, d_h=d)
    q, k, v, _ = workloads.decode_inputs(shape, seed=W + h_kv)
    lens = np.array([1500, 1001, 64, 1], np.int32)
    q_pos = np.array([1499, 700, 63, 0], np.int32)
    lo = np.maximum(0, q_pos - W + 1)
    kp, vp = _poison_below(k, lo), _poison_below(v, lo)
    for splits in (1, 7, 0):
        o, lse = gqa.decode(q.cuda(), kp.cuda(), vp.cuda(), kv_len=lens.tolist(), q_pos=q_pos.tolist(),
                            window=W, num_splits=splits, return_lse=True)
        ref, lref = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens, q_pos=q_pos, window=W)
        assert_bf16_close(_f64(o), ref, f"decode W={W} h_q={h_q} h_kv={h_kv} splits={splits}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
        assert gqa.get_device_error() == 0


def test_decode_window_fp32_check_mode():
    import kv_cache_attention_gqa_b200 as gqa

    B, h_q, h_kv, T, d = 3, 12, 3, 700, 72
    shape = workloads.DecodeShape(B=B, h_q=h_q, h_kv=h_kv, T_max=T, d_h=d)
    q, k, v, _ = workloads.decode_inputs(shape, seed=4, dtype=torch.float32)
    lens = np.array([700, 333, 20], np.int32)
    for W in (1, 9, 250):
        lo = np.maximum(0, lens - W)
        o, lse = gqa.decode(q.cuda(), _poison_below(k, lo).cuda(), _poison_below(v, lo).cuda(),
                            kv_len=lens.tolist(), window=W, num_splits=5, return_lse=True)
        ref, lref = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens, window=W)
        assert_fp32_close(_f64(o), ref, f"fp32 decode W={W}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 1e-4
        assert gqa.get_device_error() == 0


@pytest.mark.parametrize("page_size", [16, 48, 64])
@pytest.mark.parametrize("W", [1, 37, 100, 4000])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_paged_decode_window(page_size, W, dtype):
    """Windowed decode over a paged cache: the unit starts at the window start rounded down to the
    16- (or 64-) key granule and masks the keys before it; pages wholly below that are never read
    (their table entries are -1 here) and rows below the window are NaN."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=1200, d_h=128)
    lens = np.array([1200, 777, 130, 5], np.int32)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, page_size, seed=W, device="cpu",
                                                    dtype=dtype, lengths=lens)
    ref, lref = oracle.paged_decode_ref(_f64(q), _f64(k), _f64(v), bt.numpy(), lens, window=W)
    gran = 64 if page_size % 64 == 0 else 16
    bt_gpu = bt.clone()
    kp, vp = k.clone(), v.clone()
    for b, n in enumerate(lens):
        lo = max(0, int(n) - W)
        first_page = (lo // gran * gran) // page_size
        bt_gpu[b, :first_page] = -1
        for t in range(lo):
            page = int(bt[b, t // page_size])
            kp[page, :, t % page_size] = float("nan")
            vp[page, :, t % page_size] = float("nan")
    for splits in (1, 6, 0):
        o, lse = gqa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), bt_gpu.cuda(), kv_len=kl.cuda(),
                                  window=W, num_splits=splits, return_lse=True)
        what = f"paged page={page_size} W={W} {dtype} splits={splits}"
        if dtype == torch.float32:
            assert_fp32_close(_f64(o), ref, what)
        else:
            assert_bf16_close(_f64(o), ref, what)
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
        assert gqa.get_device_error() == 0, what


def test_decode_window_no_visible_key():
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=2, h_q=8, h_kv=2, T_max=128, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=1)
    # sequence 1: query at position 100 with a 10-key window over 50 cached keys -> nothing visible
    o, lse = gqa.decode(q.cuda(), k.cuda(), v.cuda(), kv_len=[128, 50], q_pos=[127, 100], window=10,
                        return_lse=True)
    assert gqa.get_device_error() == 3
    assert torch.all(o[1] == 0) and torch.all(lse[1] == float("-inf"))
    ref, _ = oracle.decode_ref(_f64(q[:1]), _f64(k[:1]), _f64(v[:1]), window=10)
    assert_bf16_close(_f64(o[:1]), ref, "the other sequence")


def test_decode_8k_window_full_size():
    """decode_8k (h_kv=8) with a 1024-key window, automatic splits, every output compared."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DECODE_8K[8]
    q, k, v, kv_len = workloads.decode_inputs(shape, seed=0, device="cuda")
    o = gqa.decode(q, k, v, kv_len=kv_len, window=1024)
    assert gqa.get_device_error() == 0
    ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=kv_len.cpu().numpy(), window=1024)
    assert_bf16_close(_f64(o), ref, "decode_8k W=1024")
