"""The seeded input recipe, checked without a GPU: draw order, scaling, one rounding to bf16, the
ragged lengths and the NaN sentinels past them. Small shapes with the workloads' structure."""

import numpy as np
import torch

import workloads


def _draws(seed, shapes, std=1.0):
    """Independent restatement of the recipe: fp32 normal draws in order from one CPU generator,
    scaled, then rounded to bf16."""
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(s, generator=g, dtype=torch.float32) * std).to(torch.bfloat16) for s in shapes]


def test_prefill_draw_order_and_scale():
    shape = workloads.PrefillShape(B=1, h_q=4, h_kv=2, S_q=24, T_max=24, d_h=16, q_start=0, kv_len=24,
                                   std=0.5)
    q, k, v = workloads.prefill_inputs(shape, seed=7)
    rq, rk, rv = _draws(7, [(1, 4, 24, 16), (1, 2, 24, 16), (1, 2, 24, 16)], std=0.5)
    for got, want in ((q, rq), (k, rk), (v, rv)):
        assert got.dtype == torch.bfloat16 and torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert workloads.PREFILL_4K.std == 0.5 and workloads.PREFILL_SMALL.std == 1.0


def test_chunked_prefill_draw_order_and_empty_slots():
    shape = workloads.PrefillShape(B=1, h_q=4, h_kv=2, S_q=8, T_max=40, d_h=16, q_start=32, kv_len=40)
    k, v, k_new, v_new, q = workloads.chunked_prefill_inputs(shape, seed=3)
    rk, rv, rkn, rvn, rq = _draws(3, [(1, 2, 32, 16), (1, 2, 32, 16), (1, 2, 8, 16), (1, 2, 8, 16),
                                      (1, 4, 8, 16)])
    assert torch.equal(k[:, :, :32], rk) and torch.equal(v[:, :, :32], rv)
    assert torch.equal(k_new, rkn) and torch.equal(v_new, rvn) and torch.equal(q, rq)
    # the slots the append will fill start at zero
    assert not k[:, :, 32:].any() and not v[:, :, 32:].any()
    c = workloads.CHUNKED_PREFILL
    assert (c.q_start + c.S_q, c.kv_len, c.T_max) == (32768, 32768, 32768)


def test_ragged_decode_lengths_and_nan_tail():
    lens = workloads.ragged_lengths(0)
    assert np.array_equal(lens, np.random.default_rng(0).integers(1024, 32769, size=64))
    shape = workloads.DecodeShape(B=5, h_q=4, h_kv=2, T_max=50, d_h=8, ragged=True, len_lo=3, len_hi=50)
    q, k, v, kv_len = workloads.decode_inputs(shape, seed=11)
    want = workloads.ragged_lengths(11, 5, 3, 50)
    assert np.array_equal(kv_len.numpy(), want)
    rq, rk, rv = _draws(11, [(5, 4, 8), (5, 2, 50, 8), (5, 2, 50, 8)])
    assert torch.equal(q, rq)
    for b, n in enumerate(want):
        for got, ref in ((k, rk), (v, rv)):
            assert torch.equal(got[b, :, :n], ref[b, :, :n])
            assert torch.isnan(got[b, :, n:].float()).all()


def test_decode_8k_shapes():
    for h_kv, s in workloads.DECODE_8K.items():
        assert (s.B, s.h_q, s.h_kv, s.T_max, s.d_h) == (8, 32, h_kv, 8192, 128)
    r = workloads.RAGGED_DECODE
    assert (r.B, r.h_q, r.h_kv, r.T_max, r.d_h, r.len_lo, r.len_hi) == (64, 64, 8, 32768, 128, 1024, 32768)
