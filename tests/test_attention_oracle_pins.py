"""Pins for the attention oracle (CPU only).

The oracle computes softmax(scale * Q K^T) V per (batch, head), with the
causal (lower-triangular, top-left) mask as an option, in float64.  These
tests hold it to what the mathematics fixes without a second implementation:
uniform weights when Q = 0, the single visible key of the first causal row,
a closed form for one-hot queries and keys, invariance under a joint
permutation of keys and values and under a shift of every key, equivariance
under a shift of every value, and the scale.  Planted mistakes must each
fail at least one pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tensor_core_gemm_fp16_b200 import workloads as wl


def _dec(t):
    return t.to(torch.float64).numpy()


def _grid(shape, seed, lo=-4.0, hi=4.0, step=1 / 64):
    """Values on a 1/64 grid: sums with small integers stay exact in fp16."""
    rng = np.random.default_rng(seed)
    n = int(round((hi - lo) / step))
    return torch.tensor(lo + step * rng.integers(0, n + 1, size=shape), dtype=torch.float16)


def _oracle_attn(Q, K, V, causal, scale=None):
    return oracle.attention(wl.to_bits(Q), wl.to_bits(K), wl.to_bits(V), causal, scale)


# ---------------------------------------------------------------------------
# pins; each takes attn(Q, K, V, causal, scale) -> float64 (B, H, Sq, D)


def pin_uniform(attn):
    """Q = 0: every visible key has the same score, so O is the mean of the
    visible values (all of them, or the first i + 1 with the causal mask)."""
    B, H, S, D = 2, 3, 19, 16
    _, K, V = wl.attention_inputs(B, H, S, S, D, seed=30)
    Q = torch.zeros(B, H, S, D, dtype=torch.float16)
    v = _dec(V)
    full = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    causal = np.cumsum(v, axis=2) / np.arange(1, S + 1)[None, None, :, None]
    ok1 = np.allclose(attn(Q, K, V, False), full, rtol=0, atol=1e-13)
    ok2 = np.allclose(attn(Q, K, V, True), causal, rtol=0, atol=1e-13)
    return ok1 and ok2


def pin_causal_first_row(attn):
    """The first query sees only key 0 under the causal mask: O = V[0] exactly."""
    Q, K, V = wl.attention_inputs(1, 2, 7, 7, 16, seed=31)
    return np.array_equal(attn(Q, K, V, True)[:, :, 0, :], _dec(V)[:, :, 0, :])


def pin_one_hot_closed_form(attn):
    """Keys c e_pi(j), queries c e_pi(t_i): the matching score is scale c^2 and
    every other is 0, so O_i = (e^a V_t + sum_{j != t} V_j) / (e^a + n - 1)
    over the n visible keys (a = scale c^2; default scale 1/sqrt(D) = 1/4 and
    c = 2 give a = 1).  Causal rows whose target is not yet visible see only
    zero scores: the mean of the visible values."""
    S, D = 11, 16
    rng = np.random.default_rng(32)
    perm = rng.permutation(D)[:S]
    targets = rng.integers(0, S, size=S)
    K = torch.zeros(1, 1, S, D, dtype=torch.float16)
    Q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    for j in range(S):
        K[0, 0, j, perm[j]] = 2.0
    for i in range(S):
        Q[0, 0, i, perm[targets[i]]] = 2.0
    _, _, V = wl.attention_inputs(1, 1, S, S, D, seed=33)
    v = _dec(V)[0, 0]
    ok = True
    for causal in (False, True):
        got = attn(Q, K, V, causal)[0, 0]
        for i in range(S):
            n = i + 1 if causal else S
            t = targets[i]
            if t < n:
                want = (math.e * v[t] + v[:n].sum(axis=0) - v[t]) / (math.e + n - 1)
            else:
                want = v[:n].mean(axis=0)
            ok &= np.allclose(got[i], want, rtol=0, atol=1e-13)
    return ok


def pin_permutation(attn):
    """Permuting keys and values together leaves O unchanged; permuting the
    queries permutes the rows of O (non-causal)."""
    Q, K, V = wl.attention_inputs(2, 2, 13, 17, 32, seed=34)
    base = attn(Q, K, V, False)
    p = wl.permutation(17, seed=35)
    ok1 = np.allclose(attn(Q, K[:, :, p].contiguous(), V[:, :, p].contiguous(), False), base,
                      rtol=0, atol=1e-13)
    q = wl.permutation(13, seed=36)
    ok2 = np.array_equal(attn(Q[:, :, q].contiguous(), K, V, False), base[:, :, q])
    return ok1 and ok2


def pin_value_shift(attn):
    """Each row of weights sums to one: adding w to every value row adds w to O."""
    B, H, S, D = 1, 2, 21, 16
    Q, K, _ = wl.attention_inputs(B, H, S, S, D, seed=37)
    V = _grid((B, H, S, D), seed=38)
    w = torch.tensor(np.random.default_rng(39).integers(-2, 3, size=D), dtype=torch.float16)
    ok = True
    for causal in (False, True):
        ok &= np.allclose(attn(Q, K, V + w, causal), attn(Q, K, V, causal) + _dec(w),
                          rtol=0, atol=1e-12)
    return ok


def pin_key_shift(attn):
    """Adding u to every key adds scale q_i.u to every score of row i: the
    softmax, hence O, does not change."""
    B, H, S, D = 1, 2, 15, 16
    Q = _grid((B, H, S, D), seed=40, lo=-1, hi=1)
    K = _grid((B, H, S, D), seed=41, lo=-1, hi=1)
    _, _, V = wl.attention_inputs(B, H, S, S, D, seed=42)
    u = torch.tensor(np.random.default_rng(43).integers(-2, 3, size=D), dtype=torch.float16)
    ok = True
    for causal in (False, True):
        ok &= np.allclose(attn(Q, K + u, V, causal), attn(Q, K, V, causal), rtol=0, atol=1e-12)
    return ok


def pin_scale(attn):
    """The scale multiplies the scores: scale 2s on Q equals scale s on 2Q
    (both exact doublings), and the default is 1/sqrt(D)."""
    Q, K, V = wl.attention_inputs(1, 2, 9, 12, 64, seed=44)
    ok1 = np.array_equal(attn(Q, K, V, False, 0.25), attn(Q * 2, K, V, False, 0.125))
    ok2 = np.array_equal(attn(Q, K, V, True), attn(Q, K, V, True, 1 / 8))
    return ok1 and ok2


PINS = [pin_uniform, pin_causal_first_row, pin_one_hot_closed_form, pin_permutation,
        pin_value_shift, pin_key_shift, pin_scale]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    assert pin(_oracle_attn)


# ---------------------------------------------------------------------------
# Planted mistakes


def _np_attn(Q, K, V, causal, scale, *, mask_offset=0, normalise=True, over_queries=False):
    """A deliberately configurable numpy attention used only to build mutants."""
    q, k, v = _dec(Q), _dec(K), _dec(V)
    D = q.shape[-1]
    sc = 1 / math.sqrt(D) if scale is None else scale
    s = sc * np.einsum("bhid,bhjd->bhij", q, k)
    Sq, Sk = s.shape[-2:]
    if causal:
        i = np.arange(Sq)[:, None]
        j = np.arange(Sk)[None, :]
        s = np.where(j <= i + mask_offset, s, -np.inf)
    axis = -2 if over_queries else -1
    m = np.max(s, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = e / e.sum(axis=axis, keepdims=True) if normalise else e
    p = np.nan_to_num(p)
    return np.einsum("bhij,bhjd->bhid", p, v)


def _m_no_scale(Q, K, V, causal, scale=None):
    return _oracle_attn(Q, K, V, causal, 1.0)


def _m_causal_ignored(Q, K, V, causal, scale=None):
    return _oracle_attn(Q, K, V, False, scale)


def _m_causal_strict(Q, K, V, causal, scale=None):     # masks the diagonal too
    return _np_attn(Q, K, V, causal, scale, mask_offset=-1)


def _m_unnormalised(Q, K, V, causal, scale=None):
    return _np_attn(Q, K, V, causal, scale, normalise=False)


def _m_softmax_over_queries(Q, K, V, causal, scale=None):
    return _np_attn(Q, K, V, causal, scale, over_queries=True)


def _m_mean_values(Q, K, V, causal, scale=None):        # ignores the scores
    return _oracle_attn(torch.zeros_like(Q), K, V, causal, scale)


def _m_fp16_output(Q, K, V, causal, scale=None):
    return _oracle_attn(Q, K, V, causal, scale).astype(np.float16).astype(np.float64)


def _m_transposed_k(Q, K, V, causal, scale=None):      # reads K as [D, Sk]
    B, H, Sk, D = K.shape
    Kt = K.reshape(B, H, D, Sk).transpose(2, 3).contiguous() if Sk * D else K
    return _oracle_attn(Q, Kt, V, causal, scale)


MUTANTS = [_m_no_scale, _m_causal_ignored, _m_causal_strict, _m_unnormalised,
           _m_softmax_over_queries, _m_mean_values, _m_fp16_output, _m_transposed_k]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__ for m in MUTANTS])
def test_pins_catch_mutants(mutant):
    failed = []
    for p in PINS:
        try:
            if not p(mutant):
                failed.append(p.__name__)
        except (ValueError, IndexError, RuntimeError):
            failed.append(p.__name__)
    assert failed, f"no pin catches {mutant.__name__}"


# ---------------------------------------------------------------------------
# Other behaviour


def test_rows_mode_equals_full():
    Q, K, V = wl.attention_inputs(2, 3, 10, 12, 16, seed=45)
    full = _oracle_attn(Q, K, V, True).reshape(-1, 16)
    rows = [0, 5, 17, 29, 59]
    got = oracle.attention(wl.to_bits(Q), wl.to_bits(K), wl.to_bits(V), True, rows=rows)
    assert np.array_equal(got, full[rows])


def test_empty_and_degenerate_shapes():
    Q, K, V = wl.attention_inputs(1, 1, 4, 0, 8, seed=46)
    assert np.array_equal(_oracle_attn(Q, K, V, False), np.zeros((1, 1, 4, 8)))
    Q, K, V = wl.attention_inputs(0, 2, 4, 4, 8, seed=47)
    assert _oracle_attn(Q, K, V, True).shape == (0, 2, 4, 8)
    # more queries than keys, causal: rows past the last key see every key
    Q, K, V = wl.attention_inputs(1, 1, 6, 3, 8, seed=48)
    o = _oracle_attn(Q, K, V, True)
    assert np.allclose(o[0, 0, 5], _oracle_attn(Q[:, :, 5:], K, V, False)[0, 0, 0], atol=1e-15)


def test_bad_arguments():
    Q, K, V = wl.attention_inputs(1, 1, 4, 4, 8, seed=49)
    with pytest.raises(ValueError):
        oracle.attention(wl.to_bits(Q), wl.to_bits(K[..., :4]), wl.to_bits(V), False)
    with pytest.raises(oracle.OracleError):
        oracle.attention(wl.to_bits(Q), wl.to_bits(K), wl.to_bits(V), False, rows=[4])
