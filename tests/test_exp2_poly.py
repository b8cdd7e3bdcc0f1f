"""The polynomial 2^x used for part of the prefill softmax: its coefficients (read from the CUDA
header) meet the stated relative error bound on [-1/2, 1/2], and the full range reduction,
restated in NumPy fp32, agrees with 2^x to that bound over the softmax's input range."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_attention_gqa_b200", "csrc", "exp2_poly.cuh")


def _coeffs():
    text = open(HDR).read()
    found = dict(re.findall(r"#define GQA_EXP2_POLY_C(\d) (0x[0-9a-fA-F]+)u", text))
    bits = [int(found[str(i)], 16) for i in range(4)]
    return np.array(bits, np.uint32).view(np.float32)


def test_polynomial_relative_error_bound():
    c = _coeffs().astype(np.float64)
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs((c[0] + f * (c[1] + f * (c[2] + f * c[3]))) / 2.0 ** f - 1.0)
    assert rel.max() < 8e-5


def test_range_reduction_in_fp32():
    c = _coeffs()
    x = np.concatenate([np.linspace(-126.0, 8.0, 500001, dtype=np.float32),
                        np.array([-126.0, -0.5, 0.5, 0.0, 8.0], np.float32)])
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    p = p.astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + ((t.view(np.uint32).astype(np.int64) << 23) & 0xFFFFFFFF)
    y = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    ref = 2.0 ** x.astype(np.float64)
    normal = x >= -125.0
    assert np.all(np.abs(y[normal] / ref[normal] - 1.0) < 1e-4)
    assert np.all(y >= 0) and np.all(np.isfinite(y))
