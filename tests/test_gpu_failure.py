"""Failure detection on the GPU without a fault: a bounded pipeline wait that runs out.

Every mbarrier wait in the kernels gives up after about 2 s of %globaltimer, records
GQA_DEVERR_TIMEOUT in the sticky device error word and returns, so a stuck pipeline ends the
kernel instead of hanging the GPU. The test hook gqa_debug_expire_waits makes CTA 0 of the bf16
prefill and of the contiguous bf16 decode wait on a barrier that nothing signals, so that bound is
reached on purpose (no trap, no bad address, no endless loop). The tests check the error status,
that the prefill tile which gave up wrote zero rows while every other row is right, that the GPU
still answers, and that the next call with the hook off matches the oracle (for decode on the same
workspace, whose work ticket must be back at zero).
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_bf16_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


def test_prefill_expired_wait_reports_timeout_and_zero_rows():
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.PrefillShape(B=1, h_q=8, h_kv=2, S_q=500, T_max=500, d_h=128, q_start=0, kv_len=500)
    q, k, v = workloads.prefill_inputs(shape, seed=41)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ref, lref = oracle.attention_ref(_f64(q), _f64(k), _f64(v))
    assert gqa.get_device_error() == 0
    gqa.debug_expire_waits(True)
    try:
        out = torch.full_like(qd, float("nan"))
        o, lse = gqa.prefill(qd, kd, vd, out=out, return_lse=True)
        code = gqa.get_device_error()
    finally:
        gqa.debug_expire_waits(False)
    assert code == 4  # GQA_DEVERR_TIMEOUT
    # h_q=8, h_kv=2: a tile holds 4 heads x 32 positions. CTA 0 takes the heaviest work, the
    # latest positions of heads 0-3 (KV group 0): one tile (positions 480..499) when each CTA holds
    # one tile, two tiles (448..499) when it holds a pair; its rows must be zeros, lse = -inf.
    got = _f64(o)
    lse_h = lse.cpu().numpy()
    zero = np.all(got == 0.0, axis=-1)
    p0s = [p0 for p0 in (480, 448) if zero[0, 0:4, p0:].all() and np.isneginf(lse_h[0, 0:4, p0:]).all()]
    assert p0s, "the rows of the work that gave up are not zeros"
    p0 = p0s[-1]
    mask = np.ones(got.shape, bool)
    mask[0, 0:4, p0:] = False
    assert_bf16_close(got[mask], ref[mask], "rows of the tiles that did not give up")
    # the GPU answers, and the next call is whole
    o2, lse2 = gqa.prefill(qd, kd, vd, return_lse=True)
    assert gqa.get_device_error() == 0
    assert_bf16_close(_f64(o2), ref, "prefill after the expired wait")
    assert np.abs(lse2.cpu().double().numpy() - lref).max() < 2e-2


@pytest.mark.parametrize("splits", [0, 400])
def test_decode_expired_wait_reports_timeout_and_workspace_stays_usable(splits):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=2048, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=42)
    lens = np.array([2048, 1500, 77, 600], np.int32)
    ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    n = gqa.decode_workspace_size(4, 32, 8, 2048, 128, torch.bfloat16, splits)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    assert gqa.get_device_error() == 0
    gqa.debug_expire_waits(True)
    try:
        gqa.decode(qd, kd, vd, kv_len=lens.tolist(), num_splits=splits, ws=ws)
        code = gqa.get_device_error()
    finally:
        gqa.debug_expire_waits(False)
    assert code == 4  # GQA_DEVERR_TIMEOUT
    assert ws[:4].view(torch.int32).item() == 0  # the merge reset the work ticket
    for rep in range(2):
        o = gqa.decode(qd, kd, vd, kv_len=lens.tolist(), num_splits=splits, ws=ws)
        assert gqa.get_device_error() == 0
        assert_bf16_close(_f64(o), ref, f"decode after the expired wait, rep {rep}")


def test_mla_tensor_core_expired_wait_reports_timeout():
    """The tensor-core MLA kernel (128 heads): CTA 0's producer waits on a barrier nothing signals;
    every other role of that CTA finds its first wait running out as well, the CTA releases its
    TMEM and ends, the call reports GQA_DEVERR_TIMEOUT, and the next call matches the oracle."""
    import kv_cache_attention_gqa_b200 as gqa
    from oracle import mla as mla_ref

    shape = workloads.MlaShape(B=2, h_q=128, T_max=1000)
    lens = [1000, 700]
    q, cache, _ = workloads.mla_decode_inputs(shape, seed=43, lengths=lens)
    ref, _ = mla_ref.mla_decode_ref(_f64(q), _f64(cache), 512, kv_len=np.array(lens), scale=shape.scale)
    qd, cd = q.cuda(), cache.cuda()
    assert gqa.get_device_error() == 0
    gqa.debug_expire_waits(True)
    try:
        gqa.mla_decode(qd, cd, kv_len=lens, scale=shape.scale)
        code = gqa.get_device_error()
    finally:
        gqa.debug_expire_waits(False)
    assert code == 4  # GQA_DEVERR_TIMEOUT
    o = gqa.mla_decode(qd, cd, kv_len=lens, scale=shape.scale)
    assert gqa.get_device_error() == 0
    assert_bf16_close(_f64(o), ref, "MLA decode after the expired wait")
