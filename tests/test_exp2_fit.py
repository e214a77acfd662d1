"""Where the constants of the kernels' FMA-pipe exp2 come from.

The prefill softmax computes one exponential pair in eight as 2^x = 2^j * 2^f with j = rint(x),
f in [-0.5, 0.5], and 2^f ~ 1 + c1 f + c2 f^2 + c3 f^3.  The coefficients are a minimax fit of the
relative error on that interval with the constant term held at 1 (so integer x, the row maximum
among them, map to exact powers of two), computed by iteratively reweighted least squares.  This
test re-runs the fit, checks that the constants in ptx.cuh are its float32 rounding, and bounds the
relative error of the float32 evaluation the kernel performs (the GPU test checks the device)."""
import os
import re

import numpy as np

PTX = os.path.join(os.path.dirname(os.path.dirname(__file__)), "exact_long_context_tmem_b200", "csrc", "ptx.cuh")


def fit_exp2(degree=3, n=20001, iters=300):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    a = np.stack([f ** k for k in range(1, degree + 1)], 1)
    w = np.ones(n)
    for _ in range(iters):
        ww = w / y  # relative error: scale each row by 1/y
        c, *_ = np.linalg.lstsq(a * ww[:, None], (y - 1) * ww, rcond=None)
        err = np.abs((1 + a @ c) / y - 1)
        w = w * (1 + 50 * err / err.max())  # push weight towards the worst points (minimax)
        w /= w.mean()
    return c


def kernel_constants():
    src = open(PTX).read()
    body = src[src.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"make_float2\(([-0-9.e]+)f,", body)]
    # Horner order in the source: c3 (times f) + c2, then c1, then the constant 1
    return vals


def eval_f32(x, c1, c2, c3):
    x = np.maximum(x.astype(np.float32), np.float32(-127))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    q = (np.float32(c3) * f + np.float32(c2)).astype(np.float32)
    q = (q * f + np.float32(c1)).astype(np.float32)
    q = (q * f + np.float32(1.0)).astype(np.float32)
    bits = (q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_constants_are_the_fit():
    c1, c2, c3 = fit_exp2(3)
    kc = kernel_constants()
    assert len(kc) >= 4 and kc[3] == 1.0, kc
    k3, k2, k1 = kc[0], kc[1], kc[2]
    for got, want in ((k1, c1), (k2, c2), (k3, c3)):
        assert np.float32(got) == np.float32(want), (got, want)


def test_float32_evaluation_error_bound():
    _, _, _, one = kernel_constants()[:4]
    k3, k2, k1 = kernel_constants()[:3]
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(eval_f32(x, k1, k2, k3).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 1.1e-4, rel.max()
    ints = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(eval_f32(ints, k1, k2, k3), np.exp2(ints))
    assert np.all(eval_f32(np.array([-np.inf, -1000, -200, -127], dtype=np.float32), k1, k2, k3) == 0)
