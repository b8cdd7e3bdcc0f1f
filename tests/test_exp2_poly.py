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


def _remez_relative(deg, a=-0.5, b=0.5, iters=30, grid=200001):
    """Minimax fit of 2^f in relative error by Remez exchange: solve for the coefficients that make
    the relative error equioscillate at deg + 2 reference points, then move the points to the
    extrema of the error's sign-constant runs."""
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    xs = np.linspace(a, b, grid)
    for _ in range(iters):
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)
        A[:, deg + 1] = (-1.0) ** np.arange(n) * 2.0 ** x
        c = np.linalg.solve(A, 2.0 ** x)[:deg + 1]
        err = np.polyval(c[::-1], xs) / 2.0 ** xs - 1.0
        runs = np.split(np.arange(grid), np.flatnonzero(np.diff(np.sign(err))) + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) > n:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:n]
        if len(ext) == n:
            x = np.sort(xs[ext])
    return c


def test_coefficients_are_the_minimax_fit():
    """The header's constants are the degree-3 relative-error minimax fit, rounded to fp32."""
    fit = _remez_relative(3).astype(np.float32)
    assert np.array_equal(fit.view(np.uint32), _coeffs().view(np.uint32))
