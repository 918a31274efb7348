"""The attention softmax's FMA-pipe exponential, checked on the host.

With head width 128 a quarter of the softmax's exponentials are computed on
the FMA pipe instead of the SFU: x = n + r, n = round(x) taken from the low
bits of x + 1.5 * 2^23, 2^x ~ R(r) with n added to R's exponent field, and
R(r) = 1 + c1 r + c2 r^2 + c3 r^3 fitted by csrc/fit_exp2.py.  This test reads
the coefficients and constants as compiled into tg_attention.cu, replays the
kernel's fp32 sequence (each fused multiply-add rounded once), and compares it
with 2^x from numpy in fp64.  The GPU parity tests of head width 128 check the
compiled kernel against the oracle.
"""
import importlib.util
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "tensor_core_gemm_fp16_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_source():
    return open(os.path.join(CSRC, "tg_attention.cu")).read()


def _kernel_coefficients():
    text = _kernel_source()
    c = {int(i): float(v) for i, v in re.findall(r"kExp2C(\d) = ([-+0-9.e]+)f", text)}
    assert sorted(c) == [1, 2, 3], c
    return np.array([1.0, c[1], c[2], c[3]], dtype=np.float32)


def test_kernel_constants_match_the_model():
    fit = _fit_module()
    text = _kernel_source()
    assert float(re.search(r"kExp2Round = ([0-9.]+)f", text).group(1)) == float(fit.MAGIC)
    body = text[text.index("uint64_t exp2_fma2("):]
    body = body[:body.index("\n}\n")]
    assert "fmaxf(x0, -125.f)" in body and "fmaxf(x1, -125.f)" in body
    assert "f2(1.f, 1.f)" in body   # the constant term of R is exactly 1
    assert body.count("<< 23") == 2


def test_relative_error_against_exp2():
    c = _kernel_coefficients()
    fit = _fit_module()
    assert fit.max_rel_error(c) < 1.1e-4


def test_integer_arguments_are_exact_powers_of_two():
    c = _kernel_coefficients()
    fit = _fit_module()
    x = np.arange(-125, 17, dtype=np.float32)
    got = fit.exp2_kernel_model(x, c)
    np.testing.assert_array_equal(got.astype(np.float64), np.exp2(x.astype(np.float64)))


def test_masked_scores_vanish_in_fp16():
    c = _kernel_coefficients()
    fit = _fit_module()
    x = np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32)
    got = fit.exp2_kernel_model(x, c)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124)
    assert np.all(got.astype(np.float16) == 0)


def test_fit_reproduces_the_compiled_coefficients():
    fit = _fit_module()
    np.testing.assert_allclose(_kernel_coefficients(), fit.fit(3), rtol=1e-6, atol=1e-9)
