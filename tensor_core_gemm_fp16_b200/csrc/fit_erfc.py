"""Fit the polynomial used by the GELU epilogue (tg_kernels.cuh).

The epilogue needs Phi(-a) = erfc(z)/2 for a = |v| >= 0, z = a / sqrt(2).  It
uses the Chebyshev-type representation of the complementary error function
of Numerical Recipes (2nd ed., section 6.2),

    erfc(z) = t * exp(-z^2 + P(t)),   t = 1 / (1 + z/2),

with base-2 exponent and the factor 1/2 folded into the polynomial, so that
the kernel evaluates

    Phi(-a) = t * 2^( -a^2 * log2(e)/2 + Q(t) ),   Q(t) = log2(erfcx(z) / (2 t)),

with one reciprocal, DEGREE fused multiply-adds and one base-2 exponential.
Q is fitted here by iteratively reweighted least squares (towards minimax) on
z in [0, 9] against scipy's scaled complementary error function erfcx; the
coefficients are our own.

    python tensor_core_gemm_fp16_b200/csrc/fit_erfc.py [DEGREE]

prints q0 .. qDEGREE and the fit's maximum error in Q (log2 units; the
relative error of Phi(-a) is about ln(2) times that) before fp32 rounding.
"""
import sys

import numpy as np
from scipy.special import erfcx

DEGREE = 6
Z_MAX = 9.0


def fit(degree=DEGREE, z_max=Z_MAX, iters=40):
    z = np.linspace(0.0, z_max, 400001)
    t = 1.0 / (1.0 + 0.5 * z)
    target = np.log2(erfcx(z) / (2.0 * t))
    V = np.vander(t, degree + 1, increasing=True)
    w = np.ones_like(z)
    coef = np.linalg.lstsq(V, target, rcond=None)[0]
    for _ in range(iters):
        err = np.abs(V @ coef - target)
        w = w * (err / err.max() + 1e-3)
        w /= w.max()
        sw = np.sqrt(w)
        coef = np.linalg.lstsq(V * sw[:, None], target * sw, rcond=None)[0]
    return coef, float(np.abs(V @ coef - target).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else DEGREE
    coef, max_err = fit(deg)
    for i, c in enumerate(coef):
        print(f"q{i} = {c:.9e}f")
    print(f"max |Q_fit - Q| on [0, {Z_MAX}] = {max_err:.3e} (log2 units)")
