"""The erf-GELU epilogue's fitted constants, checked on the host.

The kernel evaluates GELU(v) = max(v, 0) - a * T(a), a = |v|, with the lower
normal tail T = 2^Q(x), x = min(a, 6)/3 - 1 (T = 0 past a = 6), and Q a
degree-7 polynomial fitted by csrc/fit_gelu.py to the whole of log2 T.  This test
reads the coefficients as compiled into tg_kernels.cuh, replays the kernel's
fp32 operations on every finite fp16 input in [-16, 16] (each fused
multiply-add rounded once), and requires the fp16 result to be within one
unit in the last place of the correctly rounded GELU (scipy's normal CDF in
fp64).  The GPU test of the epilogue checks the compiled kernel itself the
same way against the oracle.
"""
import importlib.util
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "tensor_core_gemm_fp16_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_gelu", os.path.join(CSRC, "fit_gelu.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    text = open(os.path.join(CSRC, "tg_kernels.cuh")).read()
    q = {int(i): float(v) for i, v in re.findall(r"kGeluQ(\d) = ([-+0-9.e]+)f", text)}
    assert sorted(q) == list(range(8)), q
    amax = float(re.search(r"kGeluAMax = ([0-9.]+)f", text).group(1))
    return np.array([q[i] for i in range(8)], dtype=np.float32), amax


def test_compiled_coefficients_keep_gelu_within_one_ulp():
    fit = _fit_module()
    q, amax = _kernel_coefficients()
    assert amax == fit.A_MAX
    worst, frac = fit.ulp_check(q)
    assert worst <= 1, worst
    assert frac < 0.01, frac


def test_fit_reproduces_the_compiled_coefficients():
    fit = _fit_module()
    q_fit, max_err = fit.fit(7)
    q, _ = _kernel_coefficients()
    assert max_err < 1e-5
    np.testing.assert_allclose(q, q_fit, rtol=1e-6, atol=1e-9)
