"""Tolerances of the parity tests.

bf16 inputs with fp32 accumulation: max |out - ref| <= 2e-2 and mean |out - ref| <= 2e-3 (absolute).
fp32 check mode: max |out - ref| <= 1e-5 * max |ref| (relative to the largest reference value).
Integer and byte work (append, indexing): bit-exact.
"""

import numpy as np

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_REL = 1e-5


def bf16_errors(out, ref):
    d = np.abs(np.asarray(out, np.float64) - np.asarray(ref, np.float64))
    return float(d.max()), float(d.mean())


def assert_bf16_close(out, ref, what=""):
    out = np.asarray(out, np.float64)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    mx, mean = bf16_errors(out, ref)
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"


def assert_fp32_close(out, ref, what=""):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    scale = max(float(np.abs(ref).max()), 1e-30)
    mx = float(np.abs(out - ref).max())
    assert mx <= FP32_REL * scale, f"{what}: max {mx:.3e} > {FP32_REL} * {scale:.3e}"
