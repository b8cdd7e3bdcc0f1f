"""Backward pass (gqa_prefill_backward) on the GPU against the fp64 oracle's gradients.

The forward runs through the library (gqa_prefill with lse); the backward recomputes P from that
lse. The oracle differentiates the plain definition on the same inputs. bf16 gradients within
2e-2 (max) / 2e-3 (mean) of the tensor's largest entry, fp32 check mode within 1e-5 of it; dK and
dV rows past kv_len must be exactly zero.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_grad_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


def _run(B, h_q, h_kv, S_q, T, d, dtype=torch.bfloat16, q_start=None, kv_len=None, causal=True,
         window=0, seed=0, nan_tail=False, std=0.5):
    import kv_cache_attention_gqa_b200 as gqa

    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, h_q, S_q, d, generator=g) * std).to(dtype)
    k = (torch.randn(B, h_kv, T, d, generator=g) * std).to(dtype)
    v = torch.randn(B, h_kv, T, d, generator=g).to(dtype)
    d_o = torch.randn(B, h_q, S_q, d, generator=g).to(dtype)
    kl = np.full(B, T, np.int32) if kv_len is None else np.asarray(kv_len, np.int32)
    qs = np.zeros(B, np.int32) if q_start is None else np.asarray(q_start, np.int32)
    kg, vg = k.clone(), v.clone()
    if nan_tail:
        for b in range(B):
            kg[b, :, kl[b]:] = float("nan")
            vg[b, :, kl[b]:] = float("nan")
    qd, kd, vd, dod = q.cuda(), kg.cuda(), vg.cuda(), d_o.cuda()
    o, lse = gqa.prefill(qd, kd, vd, q_start=qs.tolist(), kv_len=kl.tolist(), causal=causal,
                         window=window, return_lse=True)
    dq, dk, dv = gqa.prefill_backward(qd, kd, vd, o, dod, lse, q_start=qs.tolist(), kv_len=kl.tolist(),
                                      causal=causal, window=window)
    assert gqa.get_device_error() == 0
    rq, rk, rv = oracle.attention_backward_ref(_f64(q), _f64(k), _f64(v), _f64(d_o), q_start=qs, kv_len=kl,
                                               causal=causal, window=window or None)
    fp32 = dtype == torch.float32
    what = f"B={B} h_q={h_q} h_kv={h_kv} S={S_q} T={T} d={d} causal={causal} W={window}"
    assert_grad_close(_f64(dq), rq, "dQ " + what, fp32)
    assert_grad_close(_f64(dk), rk, "dK " + what, fp32)
    assert_grad_close(_f64(dv), rv, "dV " + what, fp32)
    for b in range(B):
        assert torch.all(dk[b, :, kl[b]:] == 0) and torch.all(dv[b, :, kl[b]:] == 0)
    return dq, dk, dv, d_o


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("h_q,h_kv", [(8, 2), (4, 4), (16, 1), (32, 8), (12, 3)])
def test_backward_bf16_group_widths(h_q, h_kv, d):
    _run(2, h_q, h_kv, 300, 300, d, seed=h_q + d)


@pytest.mark.parametrize("W", [1, 64, 130])
def test_backward_bf16_window(W):
    _run(2, 8, 2, 400, 400, 128, window=W, seed=W)


def test_backward_bf16_offsets_ragged_nan_tail():
    """Chunked-prefill rows (q_start > 0) over ragged lengths with NaN past each kv_len."""
    _run(3, 8, 2, 200, 700, 128, q_start=[0, 300, 500], kv_len=[200, 500, 700], nan_tail=True, seed=4)


def test_backward_bf16_not_causal():
    _run(2, 8, 4, 150, 260, 64, kv_len=[260, 131], causal=False, seed=5)


@pytest.mark.parametrize("window", [0, 7])
def test_backward_fp32_check_mode(window):
    _run(2, 6, 3, 70, 90, 40, dtype=torch.float32, q_start=[0, 20], kv_len=[70, 90], window=window, seed=6)


def test_backward_bf16_group_identities():
    """dK of a head sums to zero over its keys; dV sums to the group's dO (exact identities of the
    softmax), checked on the kernel's own output against the summed magnitudes (each bf16 entry
    carries a relative rounding of 2^-9)."""
    _, dk, dv, d_o = _run(1, 8, 2, 256, 256, 128, seed=9)
    dk = _f64(dk)[0]
    dv = _f64(dv)[0]
    do = _f64(d_o)[0]
    for g in range(2):
        assert np.abs(dk[g].sum(axis=0)).max() <= 1e-2 * np.abs(dk[g]).sum(axis=0).max()
        want = do[4 * g:4 * g + 4].sum(axis=(0, 1))
        assert np.abs(dv[g].sum(axis=0) - want).max() <= 1e-2 * np.abs(dv[g]).sum(axis=0).max()


def test_backward_prefill_4k_full_size():
    """prefill_4k (h_q=32, h_kv=8, S=T=4096, d_h=128): dQ of all 32 heads and dK, dV of all 8 KV
    heads against the oracle's gradients."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(shape, seed=0, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(1)
    d_o = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    o, lse = gqa.prefill(q, k, v, return_lse=True)
    dq, dk, dv = gqa.prefill_backward(q, k, v, o, d_o, lse)
    assert gqa.get_device_error() == 0
    rq, rk, rv = oracle.attention_backward_ref(_f64(q), _f64(k), _f64(v), _f64(d_o))
    assert_grad_close(_f64(dq), rq, "prefill_4k dQ")
    assert_grad_close(_f64(dk), rk, "prefill_4k dK")
    assert_grad_close(_f64(dv), rv, "prefill_4k dV")


@pytest.mark.parametrize("d", [64, 128])
def test_backward_bf16_unaligned_o(d):
    """O at an address 2 bytes past a 16-byte boundary (O is read by the row term only; dO goes
    through TMA and must be 16-byte aligned): the row term then takes its element-by-element path
    (another summation order for D); both results match the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    g = torch.Generator().manual_seed(31 + d)
    B, h_q, h_kv, S, T = 2, 8, 2, 200, 200
    q = (torch.randn(B, h_q, S, d, generator=g) * 0.5).to(torch.bfloat16).cuda()
    k = (torch.randn(B, h_kv, T, d, generator=g) * 0.5).to(torch.bfloat16).cuda()
    v = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16).cuda()
    d_o = torch.randn(B, h_q, S, d, generator=g).to(torch.bfloat16).cuda()
    o, lse = gqa.prefill(q, k, v, return_lse=True)
    ob = torch.empty(o.numel() + 1, dtype=torch.bfloat16, device="cuda")
    o_u = ob[1:].view(o.shape)
    o_u.copy_(o)
    assert o_u.data_ptr() % 16 == 2
    rq, rk, rv = oracle.attention_backward_ref(_f64(q), _f64(k), _f64(v), _f64(d_o))
    for oo, what in ((o, "aligned"), (o_u, "unaligned")):
        dq, dk, dv = gqa.prefill_backward(q, k, v, oo, d_o, lse)
        assert gqa.get_device_error() == 0
        assert_grad_close(_f64(dq), rq, f"dQ {what} d={d}", False)
        assert_grad_close(_f64(dk), rk, f"dK {what} d={d}", False)
        assert_grad_close(_f64(dv), rv, f"dV {what} d={d}", False)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_dq_runs_mha_ragged(d):
    """More dQ tiles than SMs (320 tiles of one head x 128 positions, after 512 dK/dV tiles), so
    CTAs run several dQ tiles back to back, the next tile's loads and first scores overlapping the
    previous tile's dQ write-out; per-sequence offsets and lengths make consecutive tiles of a CTA
    differ in block count and mask, and NaN sits past every length."""
    rng = np.random.default_rng(37)
    kv = rng.integers(650, 900, size=8)
    qs = (kv - 600 - rng.integers(0, 40, size=8)).clip(0, None)
    _run(8, 8, 8, 600, 900, d, q_start=qs.tolist(), kv_len=kv.tolist(), nan_tail=True, seed=41 + d)


def test_backward_dq_runs_window_gqa():
    """416 dQ tiles of 4 heads x 32 positions under a 100-key window: tiles whose first K/V block
    is partly below every row's window (K rows zeroed in the ring) follow one another on a CTA."""
    _run(16, 8, 2, 400, 400, 128, window=100, seed=43)


def test_backward_dq_runs_with_an_invalid_sequence():
    """A sequence with kv_len = 0 among 12 (384 dQ tiles): its tiles see no key block, so a CTA's
    run passes tiles with no MMA between ones with; their dQ, dK and dV are zero, the device
    error reads GQA_DEVERR_KV_LEN, and every other sequence matches the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    B, h_q, h_kv, S, T, d, bad = 12, 16, 4, 256, 256, 64, 5
    g = torch.Generator().manual_seed(47)
    q = (torch.randn(B, h_q, S, d, generator=g) * 0.5).to(torch.bfloat16)
    k = (torch.randn(B, h_kv, T, d, generator=g) * 0.5).to(torch.bfloat16)
    v = torch.randn(B, h_kv, T, d, generator=g).to(torch.bfloat16)
    d_o = torch.randn(B, h_q, S, d, generator=g).to(torch.bfloat16)
    kl = [T] * B
    kl[bad] = 0
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), d_o.cuda()
    o, lse = gqa.prefill(qd, kd, vd, kv_len=kl, return_lse=True)
    assert gqa.get_device_error() == 1
    dq, dk, dv = gqa.prefill_backward(qd, kd, vd, o, dod, lse, kv_len=kl)
    assert gqa.get_device_error() == 1
    assert dq[bad].abs().sum().item() == 0
    assert dk[bad].abs().sum().item() == 0 and dv[bad].abs().sum().item() == 0
    keep = [b for b in range(B) if b != bad]
    rq, rk, rv = oracle.attention_backward_ref(_f64(q[keep]), _f64(k[keep]), _f64(v[keep]), _f64(d_o[keep]))
    assert_grad_close(_f64(dq[keep]), rq, "dQ, the valid sequences")
    assert_grad_close(_f64(dk[keep]), rk, "dK, the valid sequences")
    assert_grad_close(_f64(dv[keep]), rv, "dV, the valid sequences")
