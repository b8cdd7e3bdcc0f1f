"""Paged KV cache on the GPU against the oracle.

Decode over K/V pools of fixed-size pages and a shuffled block table must equal the plain
definition over the contiguous cache the pages spell out (``oracle.paged_decode_ref``): bf16 within
max |d| <= 2e-2 / mean |d| <= 2e-3, fp32 check mode within 1e-5 relative. Appends into pages are
bit-exact against ``oracle.paged_append_ref``. Rows that hold no visible position (spare pages,
the tail of each sequence's last page) are NaN, and block-table entries past a sequence's last
page are -1: neither may reach an output.
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


def _ref(q, k, v, bt, kl, q_pos=None):
    return oracle.paged_decode_ref(_f64(q), _f64(k), _f64(v), bt.cpu().numpy(), kl.cpu().numpy(),
                                   q_pos=q_pos)


@pytest.mark.parametrize("page_size", [16, 48, 64, 256])
@pytest.mark.parametrize("h_q,h_kv", [(32, 8), (32, 32), (32, 1), (40, 5), (64, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_paged_decode_bf16(page_size, h_q, h_kv, d):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=h_q, h_kv=h_kv, T_max=700, d_h=d)
    lens = [700, 333, 16, 1]
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, page_size, seed=page_size + h_kv + d,
                                                    device="cuda", lengths=lens)
    ref, lref = _ref(q, k, v, bt, kl)
    for splits in (1, 7, 0):
        o, lse = gqa.decode_paged(q, k, v, bt, kv_len=kl, num_splits=splits, return_lse=True)
        assert_bf16_close(_f64(o), ref, f"page={page_size} h_q={h_q} h_kv={h_kv} d={d} splits={splits}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
        assert gqa.get_device_error() == 0
    # length-1 sequence: exactly the value row at position 0 of its group
    r = h_q // h_kv
    v0 = v[bt[3, 0].item(), :, 0]
    assert torch.equal(o[3], v0.repeat_interleave(r, dim=0))


@pytest.mark.parametrize("page_size", [16, 48, 128])
def test_paged_decode_fp32_check_mode(page_size):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=3, h_q=12, h_kv=3, T_max=500, d_h=80)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, page_size, seed=5, device="cuda",
                                                    dtype=torch.float32, lengths=[500, 129, 17])
    ref, lref = _ref(q, k, v, bt, kl)
    for splits in (1, 6, 0):
        o, lse = gqa.decode_paged(q, k, v, bt, kv_len=kl, num_splits=splits, return_lse=True)
        assert_fp32_close(_f64(o), ref, f"fp32 page={page_size} splits={splits}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 1e-4
        assert gqa.get_device_error() == 0


def test_paged_decode_query_position_inside_the_cache():
    """q_pos before the last cached row: keys after it are masked, whichever page they sit in."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=3, h_q=16, h_kv=4, T_max=1024, d_h=128)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 32, seed=8, device="cuda",
                                                    lengths=[1024, 1000, 500])
    q_pos = np.array([0, 517, 31], np.int32)
    ref, _ = _ref(q, k, v, bt, kl, q_pos=q_pos)
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl, q_pos=q_pos.tolist(), num_splits=9)
    assert_bf16_close(_f64(o), ref, "paged q_pos")
    assert gqa.get_device_error() == 0


def test_paged_decode_shared_prefix_pages():
    """Two sequences whose tables name the same first pages (a shared prompt prefix): each reads
    them as its own positions."""
    import kv_cache_attention_gqa_b200 as gqa

    page, d = 16, 128
    g = torch.Generator(device="cuda").manual_seed(21)
    num_pages = 12
    k = torch.randn(num_pages, 2, page, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(num_pages, 2, page, d, generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn(2, 8, d, generator=g, device="cuda").to(torch.bfloat16)
    bt = torch.tensor([[7, 2, 9, 4], [7, 2, 11, 0]], dtype=torch.int32, device="cuda")
    kl = torch.tensor([64, 50], dtype=torch.int32, device="cuda")
    ref, _ = _ref(q, k, v, bt, kl)
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl, num_splits=3)
    assert_bf16_close(_f64(o), ref, "shared prefix")
    assert gqa.get_device_error() == 0


def test_paged_decode_matches_contiguous_decode():
    """The same keys stored contiguously and in pages give the same attention (both against the
    oracle; results differ from each other only by the chunk boundaries' rounding)."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=2048, d_h=128)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 64, seed=2, device="cuda",
                                                    lengths=[2048, 1500, 777, 64])
    kc = torch.from_numpy(oracle.gather_pages(_f64(k), bt.cpu().numpy(), kl.cpu().numpy(), 2048))
    vc = torch.from_numpy(oracle.gather_pages(_f64(v), bt.cpu().numpy(), kl.cpu().numpy(), 2048))
    kc, vc = kc.to(torch.bfloat16).cuda(), vc.to(torch.bfloat16).cuda()  # exact: bf16 values
    o_paged = gqa.decode_paged(q, k, v, bt, kv_len=kl)
    o_flat = gqa.decode(q, kc, vc, kv_len=kl)
    ref, _ = _ref(q, k, v, bt, kl)
    assert_bf16_close(_f64(o_paged), ref, "paged")
    assert_bf16_close(_f64(o_flat), ref, "contiguous")
    assert (o_paged.float() - o_flat.float()).abs().max().item() <= 2e-2


def test_paged_decode_bad_page_entry_is_flagged():
    """A needed block-table entry outside the pool sets GQA_DEVERR_PAGE (5); the kernel reads
    page 0 in its place, so nothing outside the pool is touched."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=2, h_q=8, h_kv=2, T_max=256, d_h=128)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 16, seed=3, device="cuda",
                                                    lengths=[256, 100])
    assert gqa.get_device_error() == 0
    bad = bt.clone()
    bad[1, 2] = k.shape[0] + 5
    gqa.decode_paged(q, k, v, bad, kv_len=kl, num_splits=4)
    assert gqa.get_device_error() == 5
    bad = bt.clone()
    bad[0, 0] = -3
    gqa.decode_paged(q.float(), k.float(), v.float(), bad, kv_len=kl, num_splits=4)
    assert gqa.get_device_error() == 5
    # the good table still works afterwards
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl, num_splits=4)
    assert_bf16_close(_f64(o), _ref(q, k, v, bt, kl)[0], "after bad entry")
    assert gqa.get_device_error() == 0


def _bits(t):
    t = t.cpu()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.view(torch.int32).numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("page_size,S_new,d", [(16, 1, 128), (16, 37, 128), (5, 7, 64), (64, 200, 3)])
def test_paged_append_bit_exact(dtype, page_size, S_new, d):
    import kv_cache_attention_gqa_b200 as gqa

    B, h_kv = 3, 2
    lens = np.array([300, 64, 5], np.int64)
    cap = lens + S_new
    table, num_pages = workloads.paged_block_table(cap, page_size, seed=page_size + S_new,
                                                   spare_pages=2)
    g = torch.Generator().manual_seed(page_size * 7 + S_new)
    k = torch.randn(num_pages, h_kv, page_size, d, generator=g).to(dtype)
    v = torch.randn(num_pages, h_kv, page_size, d, generator=g).to(dtype)
    kn = torch.randn(B, h_kv, S_new, d, generator=g).to(dtype)
    vn = torch.randn(B, h_kv, S_new, d, generator=g).to(dtype)
    kd, vd = k.cuda(), v.cuda()
    gqa.kv_append_paged(kd, vd, kn.cuda(), vn.cuda(), lens.astype(np.int32).tolist(),
                        torch.from_numpy(table).cuda())
    assert gqa.get_device_error() == 0
    kr, vr = oracle.paged_append_ref(_bits(k), _bits(v), _bits(kn), _bits(vn), table, lens)
    assert np.array_equal(_bits(kd), kr) and np.array_equal(_bits(vd), vr)


def test_paged_append_then_decode():
    """One decode step on a paged cache: append the new token's K/V into its page, then attend
    over everything up to and including it."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=3, h_q=32, h_kv=8, T_max=512, d_h=128)
    lens = np.array([511, 200, 31], np.int32)  # cached positions before this step
    q, k, v, bt, _ = workloads.paged_decode_inputs(shape, 32, seed=13, device="cuda",
                                                   lengths=lens + 1)
    g = torch.Generator(device="cuda").manual_seed(5)
    kn = torch.randn(3, 8, 1, 128, generator=g, device="cuda").to(torch.bfloat16)
    vn = torch.randn(3, 8, 1, 128, generator=g, device="cuda").to(torch.bfloat16)
    gqa.kv_append_paged(k, v, kn, vn, lens.tolist(), bt)
    kl = torch.from_numpy(lens + 1).cuda()
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl)
    assert gqa.get_device_error() == 0
    ref, _ = _ref(q, k, v, bt, kl)
    assert_bf16_close(_f64(o), ref, "append then decode")


def test_paged_append_bad_entries_write_nothing():
    import kv_cache_attention_gqa_b200 as gqa

    k = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    kn = torch.ones(2, 2, 1, 64, dtype=torch.bfloat16, device="cuda")
    bt = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")
    gqa.kv_append_paged(k, v, kn, kn, [16, 40], bt)  # b0 -> page 9 (outside), b1 -> beyond table
    code = gqa.get_device_error()
    assert code in (2, 5)
    assert k.abs().sum().item() == 0 and v.abs().sum().item() == 0


@pytest.mark.parametrize("page_size", [16, 256])
def test_paged_decode_8k_full_size(page_size):
    """decode_8k (h_q=32, h_kv=8, T=8192, d_h=128, B=8) in pages, automatic splits as the bench
    runs it; every output compared with the oracle."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DECODE_8K[8]
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, page_size, seed=0, device="cuda")
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl)
    assert gqa.get_device_error() == 0
    assert_bf16_close(_f64(o), _ref(q, k, v, bt, kl)[0], f"paged decode_8k page={page_size}")


def test_paged_ragged_decode_full_size():
    """ragged_decode (B=64, h_q=64, h_kv=8, lengths 1024..32768) in 16-token pages: every head of
    every sequence against the oracle (one sequence at a time on the host)."""
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.RAGGED_DECODE
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 16, seed=0, device="cuda")
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl)
    assert gqa.get_device_error() == 0
    assert torch.isfinite(o).all()
    lens = kl.cpu().numpy()
    btn = bt.cpu().numpy()
    for b in range(shape.B):
        # hand the oracle only this sequence's pages (in table order) and the matching table
        n_pages = (int(lens[b]) + 15) // 16
        idx = torch.from_numpy(btn[b, :n_pages].astype(np.int64)).cuda()
        table = np.arange(n_pages, dtype=np.int32)[None]
        ref, _ = oracle.paged_decode_ref(_f64(q[b:b + 1]), _f64(k[idx]), _f64(v[idx]), table,
                                         lens[b:b + 1])
        assert_bf16_close(_f64(o[b:b + 1]), ref, f"paged ragged b={b} len={lens[b]}")


def test_paged_and_mla_decode_more_chunks_than_ctas():
    import kv_cache_attention_gqa_b200 as gqa
    from oracle import mla as mla_ref

    shape = workloads.DecodeShape(B=3, h_q=16, h_kv=4, T_max=3000, d_h=128)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 16, seed=30, device="cuda", lengths=[3000, 1234, 9])
    o = gqa.decode_paged(q, k, v, bt, kv_len=kl, num_splits=400)
    assert_bf16_close(_f64(o), _ref(q, k, v, bt, kl)[0], "paged 400 splits")
    mshape = workloads.MlaShape(B=2, h_q=16, T_max=3000)
    mq, mc, mkl = workloads.mla_decode_inputs(mshape, seed=31, lengths=[3000, 500])
    om = gqa.mla_decode(mq.cuda(), mc.cuda(), kv_len=[3000, 500], scale=mshape.scale, num_splits=400)
    mref, _ = mla_ref.mla_decode_ref(_f64(mq), _f64(mc), 512, kv_len=np.array([3000, 500]), scale=mshape.scale)
    assert_bf16_close(_f64(om), mref, "mla 400 splits")
    assert gqa.get_device_error() == 0
