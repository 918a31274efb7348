"""Operands that TMA cannot address (a row pitch or base that is not a
multiple of 16 bytes) are repacked by one kernel before the GEMM, which also
gathers B's last columns for the thin N-remainder kernel; that kernel runs
alongside the GEMM, launched after it.  tg_gemm (scratch kept per stream) and
tg_gemm_noalloc (the fixed scratch array) take the same steps and must give
the same C, bit for bit; on integer inputs C is exact.  The same calls
captured in a CUDA graph replay correctly on new inputs.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, run_oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NONE = binding.TG_EPILOGUE_NONE
BIAS = binding.TG_EPILOGUE_BIAS
GELU = binding.TG_EPILOGUE_BIAS_GELU


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield


def _call(entry, a, b, bias, c, M, N, K, epi, stream):
    st = entry(a.data_ptr(), b.data_ptr(), bias.data_ptr() if bias is not None else None,
               c.data_ptr(), M, N, K, epi, stream)
    assert st == binding.TG_OK, binding.tg_status_string(st)


def _check(stream):
    torch.cuda.synchronize()
    st = binding.tg_gemm_check_error(stream)
    assert st == binding.TG_OK, binding.tg_status_string(st)


@pytest.mark.parametrize("M,N,K,epi,seed", [
    (3000, 1537, 2050, GELU, 1),   # A and B repacked, one thin column (tail kernel)
    (1000, 777, 1030, BIAS, 2),    # A and B repacked, no tail
    (640, 256, 390, NONE, 3),      # A alone repacked
    (700, 333, 512, BIAS, 4),      # B alone repacked
    (2048, 2306, 64, NONE, 5),     # two thin columns (the tail kernel's RT = 2 form)
    (2048, 2307, 64, BIAS, 7),     # three thin columns (RT = 4)
    (3000, 1544, 2048, NONE, 6),   # aligned, 8 columns past 1536: whole tiles, nothing repacked
])
def test_tg_gemm_and_noalloc_agree_bit_exact(M, N, K, epi, seed):
    dev = torch.device("cuda:0")
    A, B, bias = wl.integer_inputs(M, N, K, seed=600 + seed, bias=True)
    a, b, bb = A.to(dev), B.to(dev), bias.to(dev)
    stream = torch.cuda.current_stream().cuda_stream
    c1 = torch.empty(M, N, dtype=torch.float16, device=dev)
    c2 = torch.full((M, N), 7.0, dtype=torch.float16, device=dev)
    _call(binding.tg_gemm, a, b, bb, c1, M, N, K, epi, stream)
    _call(binding.tg_gemm_noalloc, a, b, bb, c2, M, N, K, epi, stream)
    _check(stream)
    assert torch.equal(c1, c2), "tg_gemm and tg_gemm_noalloc differ"
    ref = run_oracle(A, B, bias, epi)
    if epi == GELU:
        assert_close(c1.cpu(), ref, f"{M}x{N}x{K}")
    else:   # integer sums of integer products: exact
        assert np.array_equal(c1.cpu().double().numpy(), ref)


def test_thin_remainder_matches_oracle():
    # normal-distributed values: the tail column's fp32 sums within the rule
    M, N, K = 3000, 1537, 2050
    A, B, bias = wl.make_inputs(M, N, K, seed=610, dist="normal", bias=True)
    assert binding.tg_gemm_launch_count(0x1000, 0x100000, None, 0x1000000, M, N, K, GELU) == 3
    dev = torch.device("cuda:0")
    c = binding.gemm(A.to(dev), B.to(dev), bias.to(dev), epilogue=GELU)
    _check(torch.cuda.current_stream().cuda_stream)
    assert_close(c.cpu(), run_oracle(A, B, bias, GELU), "thin remainder")


def test_back_to_back_calls_on_one_stream():
    # each tail kernel overlaps its own GEMM and completes after it; the next
    # call's kernels follow in stream order
    M, N, K = 3000, 1537, 2050
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    ins = [wl.integer_inputs(M, N, K, seed=615 + i, bias=True) for i in range(3)]
    outs = []
    for A, B, bias in ins:
        c = torch.empty(M, N, dtype=torch.float16, device=dev)
        _call(binding.tg_gemm, A.to(dev), B.to(dev), bias.to(dev), c, M, N, K, BIAS, stream)
        outs.append(c)
    _check(stream)
    for (A, B, bias), c in zip(ins, outs):
        assert np.array_equal(c.cpu().double().numpy(), run_oracle(A, B, bias, BIAS))


@pytest.mark.parametrize("M,N,K", [(1000, 777, 1030), (3000, 1537, 2050)])
def test_graph_capture_replays_on_new_inputs(M, N, K):
    dev = torch.device("cuda:0")
    A, B, bias = wl.integer_inputs(M, N, K, seed=630, bias=True)
    a, b, bb = A.to(dev), B.to(dev), bias.to(dev)
    c = torch.empty(M, N, dtype=torch.float16, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up outside the capture (one-time set-up)
        _call(binding.tg_gemm, a, b, bb, c, M, N, K, BIAS, s.cuda_stream)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _call(binding.tg_gemm, a, b, bb, c, M, N, K, BIAS,
              torch.cuda.current_stream().cuda_stream)
    for seed in (631, 632):
        A2, B2, bias2 = wl.integer_inputs(M, N, K, seed=seed, bias=True)
        a.copy_(A2.to(dev))
        b.copy_(B2.to(dev))
        bb.copy_(bias2.to(dev))
        c.fill_(7.0)
        g.replay()
        _check(torch.cuda.current_stream().cuda_stream)
        assert np.array_equal(c.cpu().double().numpy(), run_oracle(A2, B2, bias2, BIAS)), seed
    del g


def test_kept_scratch_grows_and_is_reused_in_stream_order():
    # calls in a row on one stream, without synchronising: the scratch kept
    # for the stream grows for the second call and is reused by the third
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    shapes = [(300, 777, 130), (3000, 1537, 2050), (500, 333, 514), (3000, 1537, 2050)]
    runs = []
    for i, (M, N, K) in enumerate(shapes):
        A, B, bias = wl.integer_inputs(M, N, K, seed=650 + i, bias=True)
        c = torch.empty(M, N, dtype=torch.float16, device=dev)
        _call(binding.tg_gemm, A.to(dev), B.to(dev), bias.to(dev), c, M, N, K, BIAS, stream)
        runs.append((A, B, bias, c))
    _check(stream)
    for A, B, bias, c in runs:
        assert np.array_equal(c.cpu().double().numpy(), run_oracle(A, B, bias, BIAS))


def test_two_streams_keep_separate_scratch():
    M, N, K = 1000, 777, 1030
    dev = torch.device("cuda:0")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    ins = [wl.integer_inputs(M, N, K, seed=660 + i, bias=True) for i in range(2)]
    dins = [(A.to(dev), B.to(dev), bias.to(dev)) for A, B, bias in ins]
    torch.cuda.synchronize()
    outs = [torch.empty(M, N, dtype=torch.float16, device=dev) for _ in range(2)]
    for _ in range(3):
        for s, (a, b, bb), c in zip((s1, s2), dins, outs):
            _call(binding.tg_gemm, a, b, bb, c, M, N, K, BIAS, s.cuda_stream)
    torch.cuda.synchronize()
    for s in (s1, s2):
        assert binding.tg_gemm_check_error(s.cuda_stream) == binding.TG_OK
    for (A, B, bias), c in zip(ins, outs):
        assert np.array_equal(c.cpu().double().numpy(), run_oracle(A, B, bias, BIAS))
