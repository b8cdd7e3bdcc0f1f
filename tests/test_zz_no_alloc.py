"""gqa_decode_noalloc: the split-KV decode whose scratch space is a fixed array the library keeps in
device memory, for callers that cannot allocate device memory (a plugin whose host framework owns
every device allocation, or a loop that must not risk the synchronisation an allocation can bring).

Each call is checked against the fp64 oracle and against gqa_decode with a caller workspace, on
several calls in a row that share the array: with automatic splitting, and with four chunks per SM,
where CTAs take further chunks from the work ticket that lives in the shared array and must be
cleared before every call.

This file sorts last so that a run stopping at the first failure has already run every other test.
It must pass both alone in a fresh process and after the other tests.
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("chunks_per_sm", [0, 4])
def test_noalloc_matches_oracle_and_workspace_decode(dtype, chunks_per_sm):
    import kv_cache_attention_gqa_b200 as gqa

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    splits = chunks_per_sm * sms  # 0: automatic (one chunk per SM)
    shape = workloads.DecodeShape(B=4, h_q=32, h_kv=8, T_max=3000, d_h=128)
    q, k, v, _ = workloads.decode_inputs(shape, seed=5, dtype=dtype)
    lens = np.array([3000, 1777, 64, 901], np.int32)
    for b in range(4):  # keys past each length never contribute
        k[b, :, lens[b]:] = float("nan")
        v[b, :, lens[b]:] = float("nan")
    ref, lref = oracle.decode_ref(_f64(q), _f64(k), _f64(v), kv_len=lens)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kv_len = torch.from_numpy(lens).cuda()
    check = assert_bf16_close if dtype == torch.bfloat16 else assert_fp32_close
    ws_out = gqa.decode(qd, kd, vd, kv_len=kv_len, num_splits=splits)
    for call in range(3):  # calls in a row share the scratch array and its ticket
        out = torch.full_like(qd, float("nan"))
        o, lse = gqa.decode_noalloc(qd, kd, vd, kv_len=kv_len, num_splits=splits, out=out, return_lse=True)
        check(_f64(o), ref, f"no-alloc decode vs oracle, splits={splits}, call {call}")
        check(_f64(o), _f64(ws_out), f"no-alloc vs workspace decode, splits={splits}, call {call}")
        assert np.abs(lse.cpu().double().numpy() - lref).max() < 2e-2
    assert gqa.get_device_error() == 0


def test_noalloc_rejects_shapes_beyond_the_scratch_size():
    import kv_cache_attention_gqa_b200 as gqa

    # (B=512, h_q=h_kv=64) with 100000 chunks needs far more than the fixed scratch array: rejected
    # with GQA_ERR_WORKSPACE before any launch
    q = torch.zeros(512, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(512, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gqa.GQAError) as ei:
        gqa.decode_noalloc(q, k, k, num_splits=100000)
    assert ei.value.status == 5
    # a batch beyond the decode limit is UNSUPPORTED, as in gqa_decode
    q = torch.zeros(2000, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(2000, 8, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gqa.GQAError) as ei:
        gqa.decode_noalloc(q, k, k)
    assert ei.value.status == 2
