"""gqa_decode_noalloc (the decode whose scratch space is the library's own fixed device array, for
callers that cannot allocate device memory) against gqa_decode with a caller workspace.

This file sorts last so that a run stopping at the first failure has already run every other test.
It must pass both alone in a fresh process and after the other tests.
"""

import numpy as np
import pytest
import torch

import workloads
from _tol import assert_bf16_close, assert_fp32_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return workloads.to_f64(t)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_decode_twice(dtype):
    import kv_cache_attention_gqa_b200 as gqa

    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=3000, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=5, device="cuda", dtype=dtype)
    kv_len = torch.tensor([3000, 1777, 64, 901], dtype=torch.int32, device="cuda")
    ref, ref_lse = gqa.decode(q, k, v, kv_len=kv_len, return_lse=True)
    check = assert_bf16_close if dtype == torch.bfloat16 else assert_fp32_close
    for call in range(2):  # two calls in a row share the scratch array
        out = torch.full_like(q, float("nan"))
        o, lse = gqa.decode_noalloc(q, k, v, kv_len=kv_len, out=out, return_lse=True)
        check(_f64(o), _f64(ref), f"no-alloc decode, call {call}")
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() < 2e-2
    assert gqa.get_device_error() == 0


def test_noalloc_rejects_shapes_beyond_the_scratch_size():
    import kv_cache_attention_gqa_b200 as gqa

    # (B=512, h_q=h_kv=64) needs far more than the fixed scratch: rejected before any launch
    q = torch.zeros(512, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(512, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gqa.GQAError) as ei:
        gqa.decode_noalloc(q, k, k, num_splits=100000)
    assert ei.value.status == 5
