"""Fit the erfc approximation used by the GELU epilogue (tg_kernels.cuh).

Form (the Chebyshev-type representation of the complementary error function
used in Numerical Recipes, 2nd ed., section 6.2, with our own coefficients):

    erfc(z) ~= t * exp(-z^2 + P(t)),   t = 1 / (1 + z/2),   z >= 0,

P a degree-7 polynomial in t, fitted here by iteratively reweighted least
squares (towards minimax) to log(erfcx(z) / t) on z in [0, 9], with scipy's
scaled complementary error function erfcx as the reference.  For z < 0 the
kernel uses erfc(z) = 2 - erfc(-z).

    python tensor_core_gemm_fp16_b200/csrc/fit_erfc.py

prints the coefficients (c0 .. c7) and the fit's maximum error in P, which is
the maximum relative error of erfc before fp32 rounding.
"""
import numpy as np
from scipy.special import erfcx

DEGREE = 7
Z_MAX = 9.0


def fit(degree=DEGREE, z_max=Z_MAX, iters=40):
    z = np.linspace(0.0, z_max, 400001)
    t = 1.0 / (1.0 + 0.5 * z)
    target = np.log(erfcx(z) / t)
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
    coef, max_err = fit()
    for i, c in enumerate(coef):
        print(f"c{i} = {c:.9e}f")
    print(f"max |P_fit - P| on [0, {Z_MAX}] = {max_err:.3e}")
