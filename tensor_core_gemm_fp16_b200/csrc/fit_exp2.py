"""Fit the polynomial of the attention kernel's FMA-pipe base-2 exponential
(tg_attention.cu, exp2_fma).

The softmax computes 2^x for most scores with the SFU's ex2 and for a fixed
share of them on the FMA pipe, so that both units work at once.  The FMA form
splits x into an integer and a fraction, x = n + r with n = round(x) and
r in [-1/2, 1/2], and returns 2^n * R(r), R a polynomial of degree DEGREE:

    x' = max(x, -125)                  (masked scores, -inf, give ~2^-125)
    t  = x' + 1.5 * 2^23               (n sits in the low mantissa bits of t)
    n  = t - 1.5 * 2^23
    r  = x' - n
    2^x ~ R(r) * 2^n: the bits of R(r) plus n << 23, i.e. plus t_bits << 23
    (the rounding constant's own bits fall off the top)

R is fitted here by iteratively reweighted least squares towards the minimax
relative error on [-1/2, 1/2]; the coefficients are our own.  The script then
evaluates the kernel's fp32 sequence (each fused multiply-add rounded once)
on a dense grid and reports the largest relative error.  P enters the second
product as fp16 (relative rounding up to 2^-11 = 4.9e-4), so a relative error
near 1e-4 is below what that rounding already adds.

    python tensor_core_gemm_fp16_b200/csrc/fit_exp2.py [DEGREE]
"""
import sys

import numpy as np

DEGREE = 3
MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def fit(degree=DEGREE, iters=60):
    """R(r) = 1 + c1 r + ... + cD r^D: the constant term is fixed at 1, so
    that an integer x gives 2^x exactly (as the SFU's ex2 does)."""
    r = np.linspace(-0.5, 0.5, 200001)
    y = np.exp2(r)
    V = np.vander(r, degree + 1, increasing=True)[:, 1:]
    w = np.ones_like(r)
    c = np.linalg.lstsq(V / y[:, None], (y - 1.0) / y, rcond=None)[0]
    for _ in range(iters):
        e = np.abs(1.0 + V @ c - y) / y
        w = w * (e / e.max() + 1e-3)
        w /= w.max()
        sw = np.sqrt(w) / y
        c = np.linalg.lstsq(V * sw[:, None], (y - 1.0) * sw, rcond=None)[0]
    return np.concatenate([[1.0], c]).astype(np.float32)


def fma32(a, b, c):
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) +
            np.asarray(c, np.float64)).astype(np.float32)


def exp2_kernel_model(x, c):
    """The kernel's fp32 sequence, operation by operation."""
    x = np.asarray(x, np.float32)
    xc = np.maximum(x, np.float32(-125.0)).astype(np.float32)
    t = (xc + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    r = fma32(n, np.float32(-1.0), xc)
    p = np.full_like(r, c[-1])
    for k in c[-2::-1]:
        p = fma32(p, r, k)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def max_rel_error(c, lo=-125.0, hi=16.0, n=2000001):
    x = np.linspace(lo, hi, n).astype(np.float32)
    got = exp2_kernel_model(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got - want) / want))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else DEGREE
    c = fit(deg)
    for i, v in enumerate(c):
        print(f"c{i} = {v:.9e}f")
    print(f"max relative error of the fp32 sequence on [-125, 16]: {max_rel_error(c):.3e}")
