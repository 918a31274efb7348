"""Pins for the CPU oracle, checked against facts outside the oracle itself.

Each pin is a function of a GEMM callable so that ``test_pins_catch_mutants``
can run the same pin on deliberately broken oracles (mistakes planted on the
CPU) and show that every planted mistake fails at least one pin.

Independent sources used: numpy's float16 conversions (exhaustive codec
check), exact rational arithmetic (``fractions.Fraction``), closed forms for
identity / permutation / rank-1 operands, numpy int64 matmul, scipy's normal
CDF (Cephes ``ndtr``) and the tabulated normal CDF in tests/golden.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import ndtr

import oracle
from tensor_core_gemm_fp16_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# ---------------------------------------------------------------------------
# fp16 codecs


def test_decoder_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    # sign of zero survives
    assert math.copysign(1.0, mine[0x8000]) == -1.0


def test_encoder_roundtrips_every_finite_half():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    back = oracle.double_to_half_rne(vals[finite])
    assert np.array_equal(back, bits[finite])


def test_encoder_ties_to_even_at_every_midpoint():
    # All positive finite halves in increasing order; midpoints are exact doubles.
    pos = np.arange(0, 0x7C00, dtype=np.uint16)
    v = pos.view(np.float16).astype(np.float64)
    mid = (v[:-1] + v[1:]) / 2.0
    got = oracle.double_to_half_rne(mid)
    even = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:])
    assert np.array_equal(got, even)
    # just below / above a midpoint goes to the nearer neighbour
    below = oracle.double_to_half_rne(np.nextafter(mid, -np.inf))
    above = oracle.double_to_half_rne(np.nextafter(mid, np.inf))
    assert np.array_equal(below, pos[:-1])
    assert np.array_equal(above, pos[1:])


def test_encoder_matches_numpy_on_random_doubles():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
                        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -25,
                         2.0 ** -25 + 2.0 ** -60, 3 * 2.0 ** -26]])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.double_to_half_rne(x), ref)


# ---------------------------------------------------------------------------
# GELU


def _golden_cdf():
    rows = []
    with open(os.path.join(GOLDEN, "normal_cdf.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                x, p = line.split()
                rows.append((float(x), float(p)))
    return rows


def test_gelu_tabulated_values():
    for x, phi in _golden_cdf():
        assert oracle.gelu([x])[0] == pytest.approx(x * phi, rel=1e-13, abs=1e-300)


def test_gelu_matches_scipy_normal_cdf():
    x = np.linspace(-12, 12, 48001)
    assert np.allclose(oracle.gelu(x), x * ndtr(x), rtol=1e-13, atol=0)


def test_gelu_invariants():
    x = np.linspace(-9, 9, 9001)
    g = oracle.gelu(x)
    gm = oracle.gelu(-x)
    # g(x) - g(-x) = x * (Phi(x) + Phi(-x)) = x
    assert np.allclose(g - gm, x, rtol=0, atol=1e-14)
    assert oracle.gelu([0.0])[0] == 0.0
    assert np.all(np.abs(oracle.gelu(np.array([8.0, 10.0, 20.0])) - [8.0, 10.0, 20.0]) < 1e-13)
    assert np.all(np.abs(oracle.gelu(np.array([-8.0, -10.0, -20.0]))) < 1e-13)


def test_gelu_is_the_erf_form_not_tanh():
    x = np.linspace(-4, 4, 801)
    tanh_form = 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))
    assert np.max(np.abs(oracle.gelu(x) - tanh_form)) > 1e-4


# ---------------------------------------------------------------------------
# GEMM pins; each takes gemm(A, B, bias, epilogue) -> float64 (M, N)


def _dec(t):
    return t.to(torch.float64).numpy()


def pin_identity(gemm):
    A, B, _ = wl.make_inputs(37, 45, 37, seed=11)
    I = torch.eye(37, dtype=torch.float16)
    ok1 = np.array_equal(gemm(I, B, None, oracle.EPI_NONE), _dec(B))
    I2 = torch.eye(45, dtype=torch.float16)
    A2, _, _ = wl.make_inputs(29, 1, 45, seed=12)
    ok2 = np.array_equal(gemm(A2, I2, None, oracle.EPI_NONE), _dec(A2))
    return ok1 and ok2


def pin_permutation(gemm):
    M = K = 41
    N = 23
    _, B, _ = wl.make_inputs(M, N, K, seed=13)
    p = wl.permutation(M, seed=14)
    P = torch.zeros(M, K, dtype=torch.float16)
    P[np.arange(M), p] = 1.0          # (P B)[i] = B[p[i]]
    ok1 = np.array_equal(gemm(P, B, None, oracle.EPI_NONE), _dec(B)[p])
    A, _, _ = wl.make_inputs(19, 1, 31, seed=15)
    q = wl.permutation(31, seed=16)
    Q = torch.zeros(31, 31, dtype=torch.float16)
    Q[q, np.arange(31)] = 1.0         # (A Q)[:, j] = A[:, q[j]]
    ok2 = np.array_equal(gemm(A, Q, None, oracle.EPI_NONE), _dec(A)[:, q])
    return ok1 and ok2


def pin_rank1(gemm):
    M, N, K = 13, 17, 96
    u = 2.0 ** np.arange(-3, 10, dtype=np.float64)[:M]
    v = np.array([(-1) ** j * 2.0 ** (j % 7 - 5) for j in range(N)])
    A = torch.tensor(np.repeat(u[:, None], K, axis=1), dtype=torch.float16)
    B = torch.tensor(np.repeat(v[None, :], K, axis=0), dtype=torch.float16)
    exact = K * np.outer(u, v)
    ok1 = np.array_equal(gemm(A, B, None, oracle.EPI_NONE), exact)
    bias = torch.tensor(np.linspace(-3, 3, N), dtype=torch.float16)
    b = _dec(bias)
    ok2 = np.array_equal(gemm(A, B, bias, oracle.EPI_BIAS), exact + b)
    Bs = torch.tensor(np.repeat((v / 64)[None, :], K, axis=0), dtype=torch.float16)
    As = torch.tensor(np.repeat((u / 256)[:, None], K, axis=1), dtype=torch.float16)
    z = K * np.outer(u / 256, v / 64) + b
    got = gemm(As, Bs, bias, oracle.EPI_BIAS_GELU)
    ok3 = np.allclose(got, z * ndtr(z), rtol=1e-13, atol=1e-300)
    return ok1 and ok2 and ok3


def pin_integer_exact(gemm):
    A, B, bias = wl.integer_inputs(33, 29, 70, seed=17, lo=-3, hi=3, bias=True)
    ref = A.to(torch.int64).numpy() @ B.to(torch.int64).numpy()
    ok1 = np.array_equal(gemm(A, B, None, oracle.EPI_NONE), ref.astype(np.float64))
    ok2 = np.array_equal(gemm(A, B, bias, oracle.EPI_BIAS),
                         (ref + bias.to(torch.int64).numpy()).astype(np.float64))
    return ok1 and ok2


def pin_exact_rational(gemm):
    """Tiny random shapes against exact rational sums; error within the fp64 bound."""
    ok = True
    for (M, N, K, seed) in [(1, 1, 1, 20), (2, 3, 5, 21), (5, 4, 3, 22), (3, 7, 9, 23),
                            (6, 5, 17, 24)]:
        for epi in (oracle.EPI_NONE, oracle.EPI_BIAS, oracle.EPI_BIAS_GELU):
            A, B, bias = wl.make_inputs(M, N, K, seed=seed, bias=True)
            a, b, bb = _dec(A), _dec(B), _dec(bias)
            got = gemm(A, B, bias, epi)
            for i in range(M):
                for j in range(N):
                    s = sum(Fraction(a[i, k]) * Fraction(b[k, j]) for k in range(K))
                    if epi != oracle.EPI_NONE:
                        s += Fraction(bb[j])
                    mag = sum(abs(a[i, k] * b[k, j]) for k in range(K)) + abs(bb[j])
                    v = float(s)
                    if epi == oracle.EPI_BIAS_GELU:
                        want = v * ndtr(v)
                        tol = 1e-13 * abs(want) + 4 * K * 2.0 ** -52 * mag + 1e-300
                    else:
                        want = v
                        tol = (K + 1) * 2.0 ** -52 * mag
                    ok &= abs(got[i, j] - want) <= tol
    return ok


def pin_bias_and_k0(gemm):
    N = 9
    bias = torch.tensor(np.linspace(-4, 4, N), dtype=torch.float16)
    A = torch.zeros(3, 0, dtype=torch.float16)
    B = torch.zeros(0, N, dtype=torch.float16)
    b = _dec(bias)
    ok1 = np.array_equal(gemm(A, B, bias, oracle.EPI_NONE), np.zeros((3, N)))
    ok2 = np.array_equal(gemm(A, B, bias, oracle.EPI_BIAS), np.tile(b, (3, 1)))
    ok3 = np.allclose(gemm(A, B, bias, oracle.EPI_BIAS_GELU), np.tile(b * ndtr(b), (3, 1)),
                      rtol=1e-13, atol=1e-300)
    return ok1 and ok2 and ok3


def pin_numpy_fp64(gemm):
    A, B, bias = wl.make_inputs(70, 130, 257, seed=25, dist="uniform", bias=True)
    a, b, bb = _dec(A), _dec(B), _dec(bias)
    ref = a @ b
    bound = 257 * 2.0 ** -51 * (np.abs(a) @ np.abs(b))
    ok1 = np.all(np.abs(gemm(A, B, None, oracle.EPI_NONE) - ref) <= bound)
    z = ref + bb
    ok2 = np.all(np.abs(gemm(A, B, bias, oracle.EPI_BIAS_GELU) - z * ndtr(z))
                 <= 2 * bound + 1e-13 * np.abs(z))
    return ok1 and ok2


PINS = [pin_identity, pin_permutation, pin_rank1, pin_integer_exact, pin_exact_rational,
        pin_bias_and_k0, pin_numpy_fp64]


def _oracle_gemm(A, B, bias, epi):
    return oracle.gemm(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), epi)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    assert pin(_oracle_gemm)


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant must fail at least one pin.


def _mutant_transposed_b(A, B, bias, epi):      # reads B as if it were N x K
    M, K = A.shape
    N = B.shape[1]
    Bt = B.reshape(-1)[: K * N].reshape(N, K).t().contiguous() if K * N else B
    return _oracle_gemm(A, Bt, bias, epi)


def _mutant_drop_last_k(A, B, bias, epi):       # k loop one short
    if A.shape[1] == 0:
        return _oracle_gemm(A, B, bias, epi)
    return _oracle_gemm(A[:, :-1].contiguous(), B[:-1].contiguous(), bias, epi)


def _mutant_no_bias(A, B, bias, epi):           # bias ignored
    return _oracle_gemm(A, B, None, epi)


def _mutant_bias_after_gelu(A, B, bias, epi):   # GELU(acc) + bias
    if epi != oracle.EPI_BIAS_GELU or bias is None:
        return _oracle_gemm(A, B, bias, epi)
    return _oracle_gemm(A, B, None, epi) + _dec(bias)


def _mutant_tanh_gelu(A, B, bias, epi):         # tanh approximation of GELU
    if epi != oracle.EPI_BIAS_GELU:
        return _oracle_gemm(A, B, bias, epi)
    z = _oracle_gemm(A, B, bias, oracle.EPI_BIAS)
    return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))


def _mutant_sign(A, B, bias, epi):              # subtracts the bias
    if bias is None or epi == oracle.EPI_NONE:
        return _oracle_gemm(A, B, bias, epi)
    return _oracle_gemm(A, B, (-bias.float()).half(), epi)


def _mutant_fp32_accumulate(A, B, bias, epi):   # sums in float32 instead of double
    out = (A.float() @ B.float()).double().numpy()
    if epi != oracle.EPI_NONE and bias is not None:
        out = out + _dec(bias)
    if epi == oracle.EPI_BIAS_GELU:
        out = out * ndtr(out)
    return out


def _mutant_fp16_output(A, B, bias, epi):       # rounds the reference to fp16
    with np.errstate(over="ignore"):              # large values overflow fp16: expected here
        return _oracle_gemm(A, B, bias, epi).astype(np.float16).astype(np.float64)


MUTANTS = [_mutant_transposed_b, _mutant_drop_last_k, _mutant_no_bias,
           _mutant_bias_after_gelu, _mutant_tanh_gelu, _mutant_sign,
           _mutant_fp32_accumulate, _mutant_fp16_output]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__ for m in MUTANTS])
def test_pins_catch_mutants(mutant):
    failed = [p.__name__ for p in PINS if not p(mutant)]
    assert failed, f"no pin catches {mutant.__name__}"


# ---------------------------------------------------------------------------
# Other oracle behaviour


def test_rows_mode_equals_full():
    A, B, bias = wl.make_inputs(67, 45, 33, seed=30, bias=True)
    full = _oracle_gemm(A, B, bias, oracle.EPI_BIAS_GELU)
    rows = [66, 0, 31, 32, 5]
    part = oracle.gemm(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), oracle.EPI_BIAS_GELU,
                       rows=rows)
    assert np.array_equal(part, full[rows])


def test_int_exact_mode():
    A, B, bias = wl.integer_inputs(40, 50, 600, seed=31, lo=-2, hi=2, bias=True)
    ref = A.to(torch.int64).numpy() @ B.to(torch.int64).numpy()
    got = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B))
    assert np.array_equal(got, ref.astype(np.float64).astype(np.float16).view(np.uint16))
    got_b = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), oracle.EPI_BIAS)
    refb = ref + bias.to(torch.int64).numpy()
    assert np.array_equal(got_b, refb.astype(np.float64).astype(np.float16).view(np.uint16))
    # sums beyond 2048 need rounding: make one
    A2 = torch.full((1, 3000), 1.0, dtype=torch.float16)
    B2 = torch.ones(3000, 1, dtype=torch.float16)
    assert oracle.gemm_int_exact(wl.to_bits(A2), wl.to_bits(B2))[0, 0] == \
        np.array([3000.0]).astype(np.float16).view(np.uint16)[0]


def test_int_exact_rejects_non_integers_and_gelu():
    A, B, _ = wl.make_inputs(4, 4, 4, seed=32)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B))
    Ai, Bi, bi = wl.integer_inputs(4, 4, 4, seed=33, bias=True)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_int_exact(wl.to_bits(Ai), wl.to_bits(Bi), wl.to_bits(bi),
                              oracle.EPI_BIAS_GELU)


def test_empty_shapes():
    A = torch.zeros(0, 5, dtype=torch.float16)
    B = torch.zeros(5, 7, dtype=torch.float16)
    assert _oracle_gemm(A, B, None, oracle.EPI_NONE).shape == (0, 7)
    A = torch.zeros(4, 5, dtype=torch.float16)
    B = torch.zeros(5, 0, dtype=torch.float16)
    assert _oracle_gemm(A, B, None, oracle.EPI_NONE).shape == (4, 0)


def test_bad_arguments():
    A, B, _ = wl.make_inputs(4, 4, 4, seed=34)
    with pytest.raises(oracle.OracleError):
        oracle.gemm(wl.to_bits(A), wl.to_bits(B), None, 7)
    with pytest.raises(oracle.OracleError):
        oracle.gemm(wl.to_bits(A), wl.to_bits(B), None, oracle.EPI_NONE, rows=[4])


# ---------------------------------------------------------------------------
# tanh-approximation GELU and the row-softmax epilogue


def test_gelu_tanh_closed_point():
    """Where sqrt(2/pi)(x + 0.044715 x^3) = atanh(1/2), g(x) = 3x/4 exactly."""
    from scipy.optimize import brentq
    c = math.sqrt(2 / math.pi)
    target = math.atanh(0.5)
    x = brentq(lambda t: c * (t + 0.044715 * t ** 3) - target, 0.0, 2.0, xtol=1e-15)
    assert oracle.gelu_tanh([x])[0] == pytest.approx(0.75 * x, rel=1e-14)
    y = brentq(lambda t: c * (t + 0.044715 * t ** 3) + target, -2.0, 0.0, xtol=1e-15)
    assert oracle.gelu_tanh([y])[0] == pytest.approx(0.25 * y, rel=1e-14)


def test_gelu_tanh_invariants_and_distance_to_erf_form():
    x = np.linspace(-9, 9, 18001)
    g = oracle.gelu_tanh(x)
    assert np.allclose(g - oracle.gelu_tanh(-x), x, rtol=0, atol=1e-14)
    assert oracle.gelu_tanh([0.0])[0] == 0.0
    d = np.abs(g - x * ndtr(x))
    assert d.max() < 5e-4 and d.max() > 1e-4     # close to, and distinct from, erf GELU


def _scipy_softmax_rows(z):
    from scipy.special import softmax
    return softmax(z, axis=1)


def _exact_logits(A, B, bias):
    a, b, bb = _dec(A), _dec(B), _dec(bias) if bias is not None else None
    M, K = a.shape
    N = b.shape[1]
    z = np.empty((M, N))
    for i in range(M):
        for j in range(N):
            s = sum(Fraction(a[i, k]) * Fraction(b[k, j]) for k in range(K))
            if bb is not None:
                s += Fraction(bb[j])
            z[i, j] = float(s)
    return z


def test_softmax_matches_scipy_on_exact_logits():
    for (M, N, K, seed) in [(3, 5, 4, 40), (4, 17, 9, 41), (2, 1, 3, 42)]:
        A, B, bias = wl.make_inputs(M, N, K, seed=seed, bias=True)
        got = _oracle_gemm(A, B, bias, oracle.EPI_BIAS_SOFTMAX)
        assert np.allclose(got, _scipy_softmax_rows(_exact_logits(A, B, bias)), rtol=1e-13,
                           atol=1e-300)


def test_softmax_rows_sum_to_one_shift_invariance_and_uniform():
    A, B, _ = wl.make_inputs(20, 40, 30, seed=43)
    # bias on a 1/64 grid in [-2, 2): adding 4 keeps every value exact in fp16
    bias = (torch.arange(40, dtype=torch.float32).mul(37).remainder(256).sub(128) / 64).half()
    p = _oracle_gemm(A, B, bias, oracle.EPI_BIAS_SOFTMAX)
    assert np.allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    shifted = (bias.float() + 4.0).half()      # every value stays exact
    assert np.array_equal(_dec(shifted), _dec(bias) + 4.0)
    assert np.allclose(_oracle_gemm(A, B, shifted, oracle.EPI_BIAS_SOFTMAX), p, rtol=1e-12,
                       atol=1e-300)
    Z = torch.zeros(6, 8, dtype=torch.float16)
    Bz = torch.zeros(8, 13, dtype=torch.float16)
    assert np.allclose(_oracle_gemm(Z, Bz, None, oracle.EPI_BIAS_SOFTMAX), 1 / 13, rtol=1e-15)


def test_softmax_large_logits_stay_finite():
    # z up to ~2000: without subtracting the row maximum exp() would overflow
    A = torch.full((2, 64), 30.0, dtype=torch.float16)
    B = torch.ones(64, 5, dtype=torch.float16)
    bias = torch.tensor([0.0, 1.0, 2.0, 3.0, -1.0], dtype=torch.float16)
    p = _oracle_gemm(A, B, bias, oracle.EPI_BIAS_SOFTMAX)
    e = np.exp(np.array([0.0, 1.0, 2.0, 3.0, -1.0]))
    assert np.allclose(p, np.tile(e / e.sum(), (2, 1)), rtol=1e-14)


def test_softmax_rank1_closed_form():
    M, N, K = 4, 9, 32
    u = np.array([2.0 ** -6, -2.0 ** -5, 2.0 ** -4, 0.0])
    v = np.array([(-1) ** j * 2.0 ** (j % 4 - 3) for j in range(N)])
    A = torch.tensor(np.repeat(u[:, None], K, axis=1), dtype=torch.float16)
    B = torch.tensor(np.repeat(v[None, :], K, axis=0), dtype=torch.float16)
    z = K * np.outer(u, v)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    assert np.allclose(_oracle_gemm(A, B, None, oracle.EPI_BIAS_SOFTMAX),
                       e / e.sum(axis=1, keepdims=True), rtol=1e-14)


def test_softmax_k0_is_softmax_of_bias():
    bias = torch.tensor([0.5, -1.0, 2.0, 0.0], dtype=torch.float16)
    A = torch.zeros(3, 0, dtype=torch.float16)
    B = torch.zeros(0, 4, dtype=torch.float16)
    e = np.exp(_dec(bias) - 2.0)
    assert np.allclose(_oracle_gemm(A, B, bias, oracle.EPI_BIAS_SOFTMAX),
                       np.tile(e / e.sum(), (3, 1)), rtol=1e-15)


def test_thread_count_changes_no_result():
    """The oracle's threads only split the output rows: one thread gives the
    same bits as all of them (the bench's single-core timing relies on it)."""
    A, B, bias = wl.make_inputs(37, 29, 301, seed=77, bias=True)
    a, b, bb = wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias)
    many = oracle.gemm(a, b, bb, oracle.EPI_BIAS_GELU)
    prev = oracle.set_num_threads(1)
    try:
        assert oracle.num_threads() == 1
        one = oracle.gemm(a, b, bb, oracle.EPI_BIAS_GELU)
    finally:
        oracle.set_num_threads(prev)
    assert oracle.num_threads() == prev
    assert np.array_equal(many, one)


def test_brute_force_every_tiny_shape_exact():
    """Every (M, N, K) in {1..9}^3, plus 17 x 31 x 17 and 31 x 17 x 31, random
    fp16 operands and bias: the oracle against the exact sum, computed in
    integers (each fp16 value times 2^24 is an integer, so every product is
    an exact integer multiple of 2^-48).  NONE and BIAS within the fp64 bound
    of a K-term sum; BIAS_GELU within that bound carried through v Phi(v)."""
    import itertools
    shapes = list(itertools.product(range(1, 10), repeat=3)) + [(17, 31, 17), (31, 17, 31)]
    scale = 1 << 24
    for idx, (M, N, K) in enumerate(shapes):
        A, B, bias = wl.make_inputs(M, N, K, seed=10_000 + idx, bias=True)
        a, b, bb = _dec(A), _dec(B), _dec(bias)
        ai = [[int(a[i, k] * scale) for k in range(K)] for i in range(M)]
        bi = [[int(b[k, j] * scale) for j in range(N)] for k in range(K)]
        epis = (oracle.EPI_NONE, oracle.EPI_BIAS) if idx % 7 else \
            (oracle.EPI_NONE, oracle.EPI_BIAS, oracle.EPI_BIAS_GELU)
        got = {epi: _oracle_gemm(A, B, bias, epi) for epi in epis}
        for i in range(M):
            for j in range(N):
                exact = Fraction(sum(ai[i][k] * bi[k][j] for k in range(K)), scale * scale)
                mag = float(sum(abs(ai[i][k] * bi[k][j]) for k in range(K))) / scale ** 2
                for epi in epis:
                    s = exact + (Fraction(bb[j]) if epi != oracle.EPI_NONE else 0)
                    v = float(s)
                    bound = (K + 1) * 2.0 ** -52 * (mag + abs(bb[j]))
                    if epi == oracle.EPI_BIAS_GELU:
                        want = v * ndtr(v)
                        bound = 2 * bound + 1e-13 * abs(want) + 1e-300
                    else:
                        want = v
                    assert abs(got[epi][i, j] - want) <= bound, (M, N, K, epi, i, j)
