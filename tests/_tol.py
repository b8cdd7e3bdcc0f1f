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


# Gradients (backward pass) are not O(1) like attention outputs, so their bounds scale with the
# tensor's largest reference entry. bf16: P and dS are rounded to bf16 before the tensor-core sums
# over up to S_q (or r * S_q) terms. fp32 check mode: the same 1e-5 relative bound as the forward
# check mode; the scalar sums run over at most r * S_q terms (a few hundred in the tests), whose
# rounding stays near 1e-6 of the largest entry.
GRAD_BF16_MAX = 2e-2
GRAD_BF16_MEAN = 2e-3
GRAD_FP32_REL = 1e-5


GRAD_SCALE_FLOOR = 1e-3  # where the exact gradient vanishes (e.g. a window of one key: P = 1, dS = 0)


def assert_grad_close(out, ref, what="", fp32=False):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(out).all(), f"{what}: non-finite gradient"
    scale = max(float(np.abs(ref).max()), GRAD_SCALE_FLOOR)
    d = np.abs(out - ref)
    if fp32:
        assert d.max() <= GRAD_FP32_REL * scale, f"{what}: max {d.max():.3e} > {GRAD_FP32_REL} * {scale:.3e}"
    else:
        assert d.max() <= GRAD_BF16_MAX * scale and d.mean() <= GRAD_BF16_MEAN * scale, \
            f"{what}: max {d.max():.3e} mean {d.mean():.3e} (scale {scale:.3e})"
