"""bf16 split-KV decode on the GPU against the fp64 oracle (max |d| <= 2e-2, mean |d| <= 2e-3)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _tol import assert_bf16_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


@pytest.mark.parametrize("h_q,h_kv", [(8, 8), (8, 4), (16, 4), (16, 2), (32, 2), (32, 1), (64, 1), (12, 3), (40, 5)])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_group_widths(h_q, h_kv, d):
    import kv_cache_attention_gqa_b200 as gqa

    B, T = 3, 333
    shape = workloads.DecodeShape(B=B, h_q=h_q, h_kv=h_kv, T_max=T, d_h=d)
    q, k, v, _ = workloads.decode_inputs(shape, seed=h_q * 7 + h_kv)
    lens = np.array([T, 200, 65], np.int32)
    for b in range(B):
        k[b, :, lens[b]:] = float("nan")
        v[b, :, lens[b]:] = float("nan")
    o, lse = gqa.decode(q.cuda(), k.cuda(), v.cuda(), kv_len=lens.tolist(), num_splits=5, return_lse=True)
    ref, lref = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens)
    assert_bf16_close(_f64(o), ref, f"h_q={h_q} h_kv={h_kv} d={d}")
    assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
    assert gqa.get_device_error() == 0


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 16, 100, 0])
def test_decode_split_counts_agree(splits):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=1000, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=11)
    lens = np.array([1000, 999, 64, 1], np.int32)
    q_pos = np.array([999, 500, 63, 0], np.int32)
    o = gqa.decode(q.cuda(), k.cuda(), v.cuda(), kv_len=lens.tolist(), q_pos=q_pos.tolist(), num_splits=splits)
    ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens, q_pos=q_pos)
    assert_bf16_close(_f64(o), ref, f"splits={splits}")
    # length-1 sequence: exactly v_0 of its group (weight 1)
    assert torch.equal(o[3].cpu(), v[3, :, 0].repeat_interleave(4, dim=0))


def test_decode_workspace_ticket_returns_to_zero():
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=2, h_q=8, h_kv=2, T_max=2048, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=3)
    n = gqa.decode_workspace_size(2, 8, 2, 2048, 128, torch.bfloat16, 37)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1 = gqa.decode(qd, kd, vd, num_splits=37, ws=ws)
    assert ws[:4].view(torch.int32).item() == 0  # the work ticket is back at zero
    o2 = gqa.decode(qd, kd, vd, num_splits=37, ws=ws)
    assert torch.equal(o1, o2)  # deterministic


@pytest.mark.parametrize("h_kv", [32, 8, 1])
def test_decode_8k_full_size(h_kv):
    """decode_8k workload at full size, in the bench's launch configuration (automatic splits),
    every output compared."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DECODE_8K[h_kv]
    q, k, v, kv_len = workloads.decode_inputs(shape, seed=0, device="cuda")
    o = gqa.decode(q, k, v, kv_len=kv_len)
    ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=kv_len.cpu().numpy())
    assert_bf16_close(_f64(o), ref, f"decode_8k h_kv={h_kv}")
    assert gqa.get_device_error() == 0


def test_ragged_decode_full_size():
    """ragged_decode workload at full size (8 GiB cache, NaN beyond each length): every head of
    every one of the 64 sequences against the oracle (one sequence at a time on the host)."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.RAGGED_DECODE
    q, k, v, kv_len = workloads.decode_inputs(shape, seed=0, device="cuda")
    o, lse = gqa.decode(q, k, v, kv_len=kv_len, return_lse=True)
    assert gqa.get_device_error() == 0
    lens = kv_len.cpu().numpy()
    assert torch.isfinite(o).all()
    for b in range(shape.B):
        n = int(lens[b])
        ref, lref = oracle.decode_ref(_f64(q[b:b + 1]), _f64(k[b:b + 1, :, :n]), _f64(v[b:b + 1, :, :n]))
        assert_bf16_close(_f64(o[b:b + 1]), ref, f"ragged b={b} len={n}")
        assert np.abs(lse[b:b + 1].cpu().double().numpy() - lref).max() < 2e-2


def test_one_workspace_shared_by_different_shapes():
    """Calls of different shapes (different workspace layouts) alternate on one workspace: the
    work ticket sits at a fixed offset and every completed call leaves it at zero."""
    import kv_cache_attention_gqa_b200 as gqa

    cases = []
    for (B, h_q, h_kv, T, splits) in [(2, 8, 2, 3000, 40), (8, 32, 32, 1500, 148), (4, 64, 8, 2500, 97)]:
        shape = workloads.DecodeShape(B=B, h_q=h_q, h_kv=h_kv, T_max=T, d_h=128)
        q, k, v, kv_len = workloads.decode_inputs(shape, seed=B + h_kv, device="cuda")
        ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=kv_len.cpu().numpy())
        cases.append((q, k, v, kv_len, splits, ref))
    need = max(gqa.decode_workspace_size(c[0].shape[0], c[0].shape[1], c[1].shape[1], c[1].shape[2], 128,
                                         torch.bfloat16, c[4]) for c in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for q, k, v, kv_len, splits, ref in cases:
            o = gqa.decode(q, k, v, kv_len=kv_len, num_splits=splits, ws=ws)
            assert_bf16_close(_f64(o), ref, f"shared workspace rep={rep}")
            assert ws[:4].view(torch.int32).item() == 0  # the work ticket


def test_decode_more_chunks_than_ctas_uses_the_ticket():
    """num_splits above the CTA count: CTAs take further chunks from the atomic work ticket."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=4096, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=12)
    lens = np.array([4096, 3000, 77, 1], np.int32)
    ref, _ = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens)
    n = gqa.decode_workspace_size(4, 32, 8, 4096, 128, torch.bfloat16, 400)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        o = gqa.decode(q.cuda(), k.cuda(), v.cuda(), kv_len=lens.tolist(), num_splits=400, ws=ws)
        assert_bf16_close(_f64(o), ref, f"400 splits rep {rep}")
        assert ws[:4].view(torch.int32).item() == 0
    o32 = gqa.decode(q.float().cuda(), k.float().cuda(), v.float().cuda(), kv_len=lens.tolist(), num_splits=400)
    from _tol import assert_fp32_close
    assert_fp32_close(_f64(o32), ref, "fp32 400 splits")
    assert gqa.get_device_error() == 0


def test_decode_maximum_batch():
    """B = 1024 (the largest batch the decode accepts) with ragged lengths, a few empty-window
    rows' neighbours and q_pos inside the cache: every output against the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    B, h_q, h_kv, T, d = 1024, 8, 2, 96, 64
    shape = workloads.DecodeShape(B=B, h_q=h_q, h_kv=h_kv, T_max=T, d_h=d)
    q, k, v, _ = workloads.decode_inputs(shape, seed=21)
    rng = np.random.default_rng(21)
    lens = rng.integers(1, T + 1, size=B).astype(np.int32)
    q_pos = np.minimum(lens - 1, rng.integers(0, T, size=B)).astype(np.int32)
    ref, lref = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens, q_pos=q_pos)
    for splits in (0, 300):
        o, lse = gqa.decode(q.cuda(), k.cuda(), v.cuda(), kv_len=lens.tolist(), q_pos=q_pos.tolist(),
                            num_splits=splits, return_lse=True)
        assert_bf16_close(_f64(o), ref, f"B=1024 splits={splits}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
    assert gqa.get_device_error() == 0
    with pytest.raises(gqa.GQAError):
        gqa.decode(q[:1].cuda().expand(1025, h_q, d).contiguous(), k[:1].cuda().expand(1025, h_kv, T, d).contiguous(),
                   v[:1].cuda().expand(1025, h_kv, T, d).contiguous())
