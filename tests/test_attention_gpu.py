"""GPU parity of the fused attention forward (tg_attention_fwd) against the
fp64 oracle, through the C ABI.

Acceptance is the library's rule: relative Frobenius error <= 2e-3 and every
element within 1e-2 * max(1, |ref|), no NaN/Inf.  The probabilities enter the
second product as fp16 (relative rounding 2^-11) and O is rounded to fp16 once,
so the expected error is a few 1e-4.  Cases the mathematics makes exact are
compared exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl
from gpu_helpers import assert_close, assert_close_blocked

pytestmark = pytest.mark.gpu


def run_attn(Q, K, V, causal, scale=0.0, **kw):
    dev = torch.device("cuda:0")
    o = binding.attention(Q.to(dev), K.to(dev), V.to(dev), causal, scale, **kw)
    torch.cuda.synchronize()
    st = binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream)
    assert st == binding.TG_OK, binding.tg_status_string(st)
    return o.cpu()


def oracle_attn(Q, K, V, causal, scale=None, rows=None):
    return oracle.attention(wl.to_bits(Q), wl.to_bits(K), wl.to_bits(V), causal, scale, rows=rows)


def check(Q, K, V, causal, what, scale=0.0):
    O = run_attn(Q, K, V, causal, scale)
    ref = oracle_attn(Q, K, V, causal, None if scale == 0.0 else scale)
    D = Q.shape[-1]
    return assert_close(O.reshape(-1, D), ref.reshape(-1, D), what)


SHAPES = [  # B, H, Sq, Sk, D
    (1, 1, 128, 128, 64),
    (1, 1, 128, 128, 128),
    (2, 3, 200, 333, 64),      # ragged query and key tiles
    (1, 2, 384, 256, 128),
    (1, 1, 1, 1, 64),          # one query, one key
    (1, 1, 257, 129, 128),     # more queries than keys
    (3, 1, 64, 700, 64),       # a single partial query tile, many key tiles
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=["x".join(map(str, s)) for s in SHAPES])
def test_parity_shapes(shape, causal):
    B, H, Sq, Sk, D = shape
    Q, K, V = wl.attention_inputs(B, H, Sq, Sk, D, seed=100 + Sq + Sk + D)
    check(Q, K, V, causal, f"{shape} causal={causal}")


@pytest.mark.parametrize("D", [64, 128])
def test_explicit_scale_and_large_scores(D):
    """A large scale makes the softmax nearly one-hot and exercises the lazy
    rescale (the running maximum moves by far more than 2^8 across tiles)."""
    Q, K, V = wl.attention_inputs(1, 2, 256, 640, D, seed=150 + D)
    check(Q, K, V, False, f"scale 1.0 D={D}", scale=1.0)
    check(Q, K, V, True, f"scale 0.3 causal D={D}", scale=0.3)
    check(Q, K, V, True, f"scale -0.2 causal D={D}", scale=-0.2)   # the maximum is -0.2 x min


def test_increasing_scores_force_rescales():
    """Scores that grow with the key index: every key tile raises each row's
    maximum by more than 8 (log2 units), so O is rescaled in TMEM on every tile."""
    B, H, S, D = 1, 1, 128, 64
    Q = torch.zeros(B, H, S, D, dtype=torch.float16)
    Q[..., 0] = 1.0
    K = torch.zeros(B, H, 1024, D, dtype=torch.float16)
    K[..., 0] = torch.linspace(0, 60, 1024, dtype=torch.float32).half()
    _, _, V = wl.attention_inputs(B, H, S, 1024, D, seed=160)
    check(Q, K, V, False, "increasing scores", scale=1.0)


def test_uniform_weights_when_q_is_zero():
    B, H, S, D = 1, 2, 300, 64
    _, K, V = wl.attention_inputs(B, H, S, S, D, seed=161)
    Q = torch.zeros(B, H, S, D, dtype=torch.float16)
    v = V.to(torch.float64).numpy()
    for causal in (False, True):
        O = run_attn(Q, K, V, causal).to(torch.float64).numpy()
        want = np.cumsum(v, axis=2) / np.arange(1, S + 1)[None, None, :, None] if causal else \
            np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        assert_close(O.reshape(-1, D), want.reshape(-1, D), f"uniform causal={causal}")


def test_first_causal_row_is_v0_exactly():
    """Query 0 sees only key 0: its weight is exactly 1, so O[0] = V[0] bit for bit."""
    Q, K, V = wl.attention_inputs(2, 2, 130, 130, 128, seed=162)
    O = run_attn(Q, K, V, True)
    assert torch.equal(O[:, :, 0], V[:, :, 0])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("key", [6, 7, 70])
def test_nan_key_makes_every_row_that_sees_it_nan(D, key):
    """A NaN in one key makes every score against it NaN; the exact softmax is
    then NaN for each row that sees the key, and stays finite for causal rows
    before it.  With head width 128, keys 6, 7 and 70 fall among those whose
    exponentials run on the FMA pipe, so the row maximum must carry the NaN."""
    B, H, S = 1, 2, 200
    Q, K, V = wl.attention_inputs(B, H, S, S, D, seed=164 + key)
    K[:, :, key, 3] = float("nan")
    O = run_attn_unchecked(Q, K, V, False)
    assert torch.isnan(O.float()).any(dim=-1).all()
    O = run_attn_unchecked(Q, K, V, True)
    rows = torch.isnan(O.float()).any(dim=-1)
    assert rows[:, :, key:].all() and not rows[:, :, :key].any()
    assert torch.isfinite(O[:, :, :key].float()).all()


def run_attn_unchecked(Q, K, V, causal):
    dev = torch.device("cuda:0")
    o = binding.attention(Q.to(dev), K.to(dev), V.to(dev), causal, 0.0)
    torch.cuda.synchronize()
    assert binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream) == binding.TG_OK
    return o.cpu()


def test_empty_and_zero_keys():
    dev = torch.device("cuda:0")
    q = torch.randn(1, 2, 5, 64, device=dev).half()
    k = torch.empty(1, 2, 0, 64, device=dev, dtype=torch.float16)
    o = torch.full_like(q, 7.0)
    binding.attention(q, k, k, False, out=o)
    torch.cuda.synchronize()
    assert torch.count_nonzero(o).item() == 0
    q0 = torch.empty(0, 2, 5, 64, device=dev, dtype=torch.float16)
    binding.attention(q0, q0, q0, True)


def test_deterministic():
    Q, K, V = wl.attention_inputs(2, 4, 512, 512, 128, seed=163)
    a = run_attn(Q, K, V, True)
    b = run_attn(Q, K, V, True)
    assert torch.equal(a, b)


def test_rejects_bad_calls():
    dev = torch.device("cuda:0")
    q = torch.randn(1, 1, 8, 96, device=dev).half()
    with pytest.raises(binding.TgError) as e:
        binding.attention(q, q.clone(), q.clone())
    assert e.value.status == binding.TG_ERR_INVALID_ARG
    q = torch.randn(1, 1, 8, 64, device=dev).half()
    st = binding.tg_attention_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), 1, 1,
                                  8, 8, 64, 0, 0.0)
    assert st == binding.TG_ERR_INVALID_ARG          # O overlaps Q
    buf = torch.zeros(1 + 8 * 64 * 4, device=dev, dtype=torch.float16)
    st = binding.tg_attention_fwd(buf[1:].data_ptr(), q.data_ptr(), q.data_ptr(),
                                  torch.empty_like(q).data_ptr(), 1, 1, 8, 8, 64, 0, 0.0)
    assert st == binding.TG_ERR_MISALIGNED


def test_timeout_injection_reports_and_recovers():
    """The first CTA skips its first key-tile load: the MMA issuer's bounded wait
    (50 ms) expires, the kernel exits cleanly, the status says so, and the
    next call is correct.  Nothing faults: the load is simply never issued."""
    Q, K, V = wl.attention_inputs(1, 2, 256, 256, 64, seed=164)
    dev = torch.device("cuda:0")
    binding.attention(Q.to(dev), K.to(dev), V.to(dev), False, wait_limit_ns=50_000_000,
                      inject=binding.TG_INJECT_SKIP_FIRST_LOAD)
    torch.cuda.synchronize()
    st = binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream)
    assert st == binding.TG_ERR_TIMEOUT
    check(Q, K, V, False, "after timeout")


# ---------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("name", list(wl.ATTN_WORKLOADS))
def test_workload_full_output(name):
    """The full launch of each attention workload (the benchmark's shapes),
    every output element against the whole fp64 oracle result (a few seconds
    of oracle time on the host cores)."""
    w = wl.ATTN_WORKLOADS[name]
    Q, K, V = wl.attn_workload_inputs(w)
    O = run_attn(Q, K, V, w.causal)
    ref = oracle_attn(Q, K, V, w.causal).reshape(-1, w.D)
    assert_close_blocked(O.reshape(-1, w.D), ref, f"{name} full output", block_rows=65536)


# ---------------------------------------------------------------- key-half split

SPLIT_SHAPES = [  # B, H, Sq, Sk, D (non-causal; at least two key tiles)
    (2, 3, 200, 333, 64),      # three key tiles: halves of one and two
    (1, 2, 384, 256, 128),     # two key tiles
    (1, 1, 257, 129, 128),     # the second half holds one valid key
    (3, 1, 64, 700, 64),       # six key tiles, one partial query tile
    (1, 4, 1000, 1000, 128),
]


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=["x".join(map(str, s)) for s in SPLIT_SHAPES])
def test_kv_split_modes_match_the_oracle(shape):
    """Every unit split in two key halves (merged by the half that finishes
    second), no split, and the automatic choice: each against the oracle."""
    B, H, Sq, Sk, D = shape
    Q, K, V = wl.attention_inputs(B, H, Sq, Sk, D, seed=300 + Sq + Sk + D)
    ref = oracle_attn(Q, K, V, False).reshape(-1, D)
    for mode in (binding.TG_ATTN_SPLIT_ALL, binding.TG_ATTN_SPLIT_NEVER,
                 binding.TG_ATTN_SPLIT_AUTO):
        O = run_attn(Q, K, V, False, kv_split=mode)
        assert_close(O.reshape(-1, D), ref, f"{shape} kv_split={mode}")


def test_kv_split_not_applied_where_it_cannot_be():
    """Causal calls and a single key tile never split: forcing the split gives
    the unsplit result bit for bit."""
    for (B, H, Sq, Sk, D), causal in (((1, 2, 384, 384, 64), True),
                                      ((2, 2, 300, 128, 128), False)):
        Q, K, V = wl.attention_inputs(B, H, Sq, Sk, D, seed=400 + Sq)
        a = run_attn(Q, K, V, causal, kv_split=binding.TG_ATTN_SPLIT_ALL)
        b = run_attn(Q, K, V, causal, kv_split=binding.TG_ATTN_SPLIT_NEVER)
        assert torch.equal(a, b)


def test_kv_split_workspace_growth_and_reuse():
    """Split calls of growing and shrinking unit counts on one stream (the
    workspace grows in stream order, each launch takes a fresh epoch), then
    the first call again: the same result bit for bit."""
    small = wl.attention_inputs(1, 1, 256, 512, 64, seed=501)
    big = wl.attention_inputs(2, 8, 1024, 512, 64, seed=502)
    first = run_attn(*small, False, kv_split=binding.TG_ATTN_SPLIT_ALL)
    for Q, K, V in (big, small, big):
        O = run_attn(Q, K, V, False, kv_split=binding.TG_ATTN_SPLIT_ALL)
        assert_close(O.reshape(-1, 64), oracle_attn(Q, K, V, False).reshape(-1, 64), "regrow")
    again = run_attn(*small, False, kv_split=binding.TG_ATTN_SPLIT_ALL)
    assert torch.equal(first, again)


def test_kv_split_on_two_streams_at_once():
    """Split launches on two streams overlap in time; each stream has its own
    workspace and flags, so both results match the oracle."""
    dev = torch.device("cuda:0")
    cases = [wl.attention_inputs(2, 4, 512, 768, 64, seed=601),
             wl.attention_inputs(2, 4, 512, 768, 64, seed=602)]
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    outs = []
    torch.cuda.synchronize()
    dev_in = [tuple(x.to(dev) for x in c) for c in cases]
    torch.cuda.synchronize()
    for _ in range(3):
        outs = []
        for (q, k, v), s in zip(dev_in, streams):
            with torch.cuda.stream(s):
                outs.append(binding.attention(q, k, v, False, kv_split=binding.TG_ATTN_SPLIT_ALL))
    torch.cuda.synchronize()
    for s in streams:
        assert binding.tg_gemm_check_error(s.cuda_stream) == binding.TG_OK
    for (Q, K, V), o in zip(cases, outs):
        ref = oracle_attn(Q, K, V, False).reshape(-1, 64)
        assert_close(o.cpu().reshape(-1, 64), ref, "two streams")
