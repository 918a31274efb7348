"""Stream-K work split on the GPU (through the C ABI) against the oracle.

With stream-K the K loops of the tiles are divided over all units; partial
fp32 tiles are added by the unit holding each tile's first k-block.  Integer
inputs make every partial sum exact, so a missing, doubled or misplaced
partial shows up bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bits_equal, assert_close, run_gpu, run_oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SK, TILES = binding.TG_SPLIT_STREAM_K, binding.TG_SPLIT_TILES
NONE, BIAS, GELU = binding.TG_EPILOGUE_NONE, binding.TG_EPILOGUE_BIAS, binding.TG_EPILOGUE_BIAS_GELU
TANH, SOFTMAX = binding.TG_EPILOGUE_BIAS_GELU_TANH, binding.TG_EPILOGUE_BIAS_SOFTMAX


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield


@pytest.mark.parametrize("config_id", [0, 1, 3, 6])
@pytest.mark.parametrize("M,N,K", [(512, 512, 4096), (3000, 1537, 2050), (256, 256, 256)])
def test_streamk_integer_inputs_bit_exact(config_id, M, N, K):
    A, B, bias = wl.integer_inputs(M, N, K, seed=M + N + K + config_id, lo=-1, hi=1, bias=True)
    exp = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), oracle.EPI_BIAS)
    C = run_gpu(A, B, bias, BIAS, config_id=config_id, split=SK)
    assert_bits_equal(C, exp, f"stream-K int cfg{config_id} {M}x{N}x{K}")


def test_streamk_identity_bit_exact():
    M = K = 768
    _, B, _ = wl.make_inputs(1, 520, K, seed=1100)
    A = torch.eye(M, dtype=torch.float16)
    assert_bits_equal(run_gpu(A, B, None, NONE, config_id=0, split=SK), wl.to_bits(B), "I @ B")


@pytest.mark.parametrize("epilogue", [GELU, TANH, SOFTMAX])
def test_streamk_epilogues_match_oracle(epilogue):
    N = 200 if epilogue == SOFTMAX else 700
    A, B, bias = wl.make_inputs(1500, N, 3000, seed=1200 + epilogue, bias=True,
                                b_scale=1 / 3000 ** 0.5)
    cfg = 6 if epilogue == SOFTMAX else 0
    C = run_gpu(A, B, bias, epilogue, config_id=cfg, split=SK)
    assert_close(C, run_oracle(A, B, bias, epilogue), f"stream-K epilogue {epilogue}")


@pytest.mark.parametrize("config_id", [0, 3, 5])
def test_streamk_more_units_than_iterations(config_id):
    """Tiny problems: most units own no iterations and must not be waited on."""
    for (M, N, K) in [(100, 64, 64), (256, 256, 128), (17, 9, 300)]:
        A, B, bias = wl.make_inputs(M, N, K, seed=M * N + K, bias=True)
        C = run_gpu(A, B, bias, GELU, config_id=config_id, split=SK)
        assert_close(C, run_oracle(A, B, bias, GELU), f"tiny stream-K {M}x{N}x{K}")


def test_streamk_is_deterministic_and_close_to_whole_tiles():
    A, B, bias = wl.make_inputs(2048, 2048, 2048, seed=1300, bias=True)
    c1 = run_gpu(A, B, bias, GELU, config_id=0, split=SK)
    c2 = run_gpu(A, B, bias, GELU, config_id=0, split=SK)
    assert torch.equal(c1, c2)
    c3 = run_gpu(A, B, bias, GELU, config_id=0, split=TILES)
    # different fp32 summation orders: both meet the acceptance rule, and
    # they differ by at most 1e-2 * max(1, |C|) elementwise
    ref = run_oracle(A, B, bias, GELU)
    assert_close(c1, ref, "stream-K")
    assert_close(c3, ref, "whole tiles")
    d = (c1.double() - c3.double()).abs().numpy()
    assert np.all(d <= 1e-2 * np.maximum(1.0, np.abs(ref)))


def test_streamk_flag_wait_times_out_cleanly():
    dev = torch.device("cuda:0")
    A, B, bias = wl.make_inputs(1024, 1024, 4096, seed=1400, bias=True)
    a, b, bb = A.to(dev), B.to(dev), bias.to(dev)
    c = torch.empty(1024, 1024, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    assert binding.tg_gemm_check_error(stream) == binding.TG_OK
    st = binding.tg_gemm_ex(a.data_ptr(), b.data_ptr(), bb.data_ptr(), c.data_ptr(), 1024, 1024,
                            4096, GELU, config_id=0, wait_limit_ns=50_000_000,
                            inject=binding.TG_INJECT_SKIP_STREAMK_FLAGS, split=SK, stream=stream)
    assert st == binding.TG_OK
    assert binding.tg_gemm_check_error(stream) == binding.TG_ERR_TIMEOUT
    assert binding.tg_gemm_check_error(stream) == binding.TG_OK
    C = run_gpu(A, B, bias, GELU, config_id=0, split=SK)
    assert_close(C, run_oracle(A, B, bias, GELU), "after stream-K timeout")
