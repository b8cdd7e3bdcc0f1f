"""kv_append on the GPU against the oracle's array copy: bit-exact."""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.cpu()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.view(torch.int32).numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,h_kv,S_new,T_max,d", [(2, 3, 1, 17, 128), (3, 2, 5, 40, 64), (1, 8, 512, 1024, 128),
                                                  (2, 1, 3, 9, 3), (4, 2, 1, 8, 2)])
def test_append_bit_exact(dtype, B, h_kv, S_new, T_max, d):
    import kv_cache_attention_gqa_b200 as gqa

    g = torch.Generator().manual_seed(B * 100 + d)
    k = torch.randn(B, h_kv, T_max, d, generator=g).to(dtype)
    v = torch.randn(B, h_kv, T_max, d, generator=g).to(dtype)
    kn = torch.randn(B, h_kv, S_new, d, generator=g).to(dtype)
    vn = torch.randn(B, h_kv, S_new, d, generator=g).to(dtype)
    pos = np.array([(7 * b) % (T_max - S_new + 1) for b in range(B)], np.int32)
    pos[-1] = T_max - S_new  # last rows of the cache
    kd, vd = k.cuda(), v.cuda()
    gqa.kv_append(kd, vd, kn.cuda(), vn.cuda(), torch.from_numpy(pos).cuda())
    kr, vr = oracle.kv_append_ref(_bits(k), _bits(v), _bits(kn), _bits(vn), pos)
    assert np.array_equal(_bits(kd), kr) and np.array_equal(_bits(vd), vr)
    assert gqa.get_device_error() == 0


def test_append_out_of_range_is_flagged_and_writes_nothing():
    import kv_cache_attention_gqa_b200 as gqa

    k = torch.zeros(2, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    kn = torch.ones(2, 2, 2, 64, dtype=torch.bfloat16, device="cuda")
    gqa.kv_append(k, v, kn, kn, torch.tensor([7, 0], dtype=torch.int32, device="cuda"))
    assert gqa.get_device_error() == 2
    assert k[0].abs().sum().item() == 0  # sequence 0 did not fit: untouched
    assert torch.equal(k[1, :, 0:2], kn[1])  # sequence 1 was written
    assert gqa.get_device_error() == 0  # the word was cleared by the read


def test_append_of_zero_rows_is_a_no_op():
    import kv_cache_attention_gqa_b200 as gqa

    k = torch.randn(2, 2, 8, 64).to(torch.bfloat16).cuda()
    v = torch.randn(2, 2, 8, 64).to(torch.bfloat16).cuda()
    k0, v0 = k.clone(), v.clone()
    empty = torch.empty(2, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    gqa.kv_append(k, v, empty, empty, [3, 8])
    torch.cuda.synchronize()
    assert torch.equal(k, k0) and torch.equal(v, v0)
    assert gqa.get_device_error() == 0
