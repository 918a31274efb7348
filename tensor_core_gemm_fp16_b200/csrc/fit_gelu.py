"""Fit the polynomial used by the erf-GELU epilogue (tg_kernels.cuh, gelu_erf).

GELU(v) = v * Phi(v) = max(v, 0) - a * T(a) for a = |v|, where
T(a) = Phi(-a) is the standard normal lower tail.  Its logarithm is the
Gaussian exponent plus a slowly varying remainder (the logarithm of the
Mills ratio, which falls like -log2(a sqrt(2 pi)) for large a):

    log2 T(a) = -a^2 * log2(e) / 2 + R(a),   R(0) = -1,

a smooth function on [0, A_MAX] that a polynomial fits closely.  The kernel
evaluates

    T(a) = 2^( Q(x) ),   x = min(a, A_MAX) / (A_MAX/2) - 1,   and T = 0 for a > A_MAX,

with Q a polynomial of degree DEGREE in x in [-1, 1] (Horner form) fitted to
the whole log2 T, Gaussian term included, so one GELU costs one base-2
exponential, no division and DEGREE + 2 fused multiply-adds.  Past A_MAX,
a * T is below half the smallest fp16 subnormal for every fp16 input, so
setting T to zero there changes no fp16 result (at most the sign of a zero).

Q is fitted here by iteratively reweighted least squares (towards minimax) on
a in [0, A_MAX] against scipy's log_ndtr; the coefficients are our own.  The
script then evaluates the kernel's fp32 formula (each fused multiply-add
rounded once, the exponential exact) on every finite fp16 input in
[-16, 16] and reports its largest distance, in fp16 units in the last place,
from the correctly rounded GELU.

    python tensor_core_gemm_fp16_b200/csrc/fit_gelu.py [DEGREE]
"""
import sys

import numpy as np
from scipy.special import log_ndtr, ndtr

DEGREE = 7
A_MAX = 6.0
LOG2E = 1.0 / np.log(2.0)


def target(a):
    return log_ndtr(-a) * LOG2E


def fit(degree=DEGREE, iters=40):
    a = np.linspace(0.0, A_MAX, 200001)
    x = a / (A_MAX / 2.0) - 1.0
    y = target(a)
    V = np.polynomial.chebyshev.chebvander(x, degree)
    w = np.ones_like(a)
    coef = np.linalg.lstsq(V, y, rcond=None)[0]
    for _ in range(iters):
        err = np.abs(V @ coef - y)
        w = w * (err / err.max() + 1e-3)
        w /= w.max()
        sw = np.sqrt(w)
        coef = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)[0]
    mono = np.polynomial.chebyshev.cheb2poly(coef)   # power basis in x, increasing
    return mono.astype(np.float32), float(np.abs(V @ coef - y).max())


def f32(x):
    return np.float32(x)


def fma32(a, b, c):
    """fp32 fused multiply-add: the product and sum exact in fp64 for fp32
    operands of these magnitudes, then one rounding to fp32."""
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) +
            np.asarray(c, np.float64)).astype(np.float32)


def gelu_kernel_model(v, q):
    """The kernel's fp32 evaluation, operation by operation."""
    v = np.asarray(v, np.float32)
    a = np.abs(v)
    x = fma32(np.minimum(a, f32(A_MAX)), f32(2.0 / A_MAX), f32(-1.0))
    p = np.full_like(x, q[-1])
    for c in q[-2::-1]:
        p = fma32(p, x, c)
    t = np.exp2(p.astype(np.float64)).astype(np.float32)
    t = np.where(a > f32(A_MAX), f32(0.0), t)
    return fma32(-a, t, np.maximum(v, f32(0.0)))


def ulp_check(q):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    keep = np.isfinite(vals) & (np.abs(vals.astype(np.float64)) <= 16)
    v = vals[keep]
    vd = v.astype(np.float64)
    exact = vd * ndtr(vd)
    got = gelu_kernel_model(v.astype(np.float32), q).astype(np.float16)
    want = exact.astype(np.float16)
    gb = got.view(np.uint16).astype(np.int32)
    wb = want.view(np.uint16).astype(np.int32)
    same = (gb & 0x8000) == (wb & 0x8000)
    dist = np.where(same, np.abs(gb - wb), (gb & 0x7FFF) + (wb & 0x7FFF))
    return int(dist.max()), float((dist > 0).mean())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else DEGREE
    q, max_err = fit(deg)
    for i, c in enumerate(q):
        print(f"q{i} = {c:.9e}f")
    print(f"max |Q_fit - log2 T| on [0, {A_MAX}] = {max_err:.3e} (log2 units)")
    worst, frac = ulp_check(q)
    print(f"fp32 model vs correctly rounded GELU on fp16 [-16, 16]: max {worst} ulp, "
          f"{100 * frac:.3f}% of inputs off by one")
