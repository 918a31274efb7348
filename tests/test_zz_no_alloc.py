"""tg_gemm_noalloc, the allocation-free entry point, against tg_gemm.

Callers that must not allocate device memory (an engine whose own allocator
owns nearly all of HBM, a latency-critical loop that must stay out of the
driver's allocator) use tg_gemm_noalloc: repacking scratch for unaligned
operands comes from a fixed device array inside the library instead of a
memory pool.  These tests call it through the C ABI and compare its output
with tg_gemm's, under the same acceptance rule as the parity tests, on calls
in a row that reuse the shared scratch array.  The file is named so that
pytest collects it last.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _device_inputs(M, N, K, seed, dist="uniform"):
    A, B, bias = wl.make_inputs(M, N, K, seed=seed, dist=dist, bias=True)
    dev = torch.device("cuda:0")
    return A.to(dev), B.to(dev), bias.to(dev)


def _run(entry, a, b, bias, M, N, K, epilogue):
    c = torch.empty(M, N, dtype=torch.float16, device=a.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = entry(a.data_ptr(), b.data_ptr(), bias.data_ptr(), c.data_ptr(), M, N, K, epilogue,
               stream)
    assert st == binding.TG_OK, binding.tg_status_string(st)
    torch.cuda.synchronize()
    assert binding.tg_gemm_check_error(stream) == binding.TG_OK
    return c.cpu()


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield


def test_noalloc_matches_tg_gemm_on_two_calls_in_a_row():
    # 3000 x 1537 x 2050: neither A's nor B's row pitch is a multiple of 16
    # bytes, so both are repacked (about 18.7 MB of scratch).
    M, N, K = 3000, 1537, 2050
    epi = binding.TG_EPILOGUE_BIAS_GELU
    a, b, bias = _device_inputs(M, N, K, seed=3)
    ref = _run(binding.tg_gemm, a, b, bias, M, N, K, epi).double().numpy()
    for call in range(2):
        got = _run(binding.tg_gemm_noalloc, a, b, bias, M, N, K, epi)
        assert_close(got, ref, f"tg_gemm_noalloc call {call + 1}")


def test_noalloc_after_a_larger_call_and_with_aligned_operands():
    # A smaller unaligned problem after a larger one (the scratch keeps the
    # larger call's bytes), then an aligned problem that needs no scratch.
    for (M, N, K, seed) in [(1000, 777, 1030, 11), (512, 1024, 768, 12)]:
        a, b, bias = _device_inputs(M, N, K, seed=seed, dist="normal")
        ref = _run(binding.tg_gemm, a, b, bias, M, N, K, binding.TG_EPILOGUE_BIAS).double().numpy()
        got = _run(binding.tg_gemm_noalloc, a, b, bias, M, N, K, binding.TG_EPILOGUE_BIAS)
        assert_close(got, ref, f"tg_gemm_noalloc {M}x{N}x{K}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # A needs repacking (K not a multiple of 8): 2 * M * K8 bytes > the limit.
    limit = binding.noalloc_scratch_bytes()
    K = 4001
    M = limit // (2 * 4008) + 1
    st = binding.tg_gemm_noalloc(0x100000, 0x40000000000, None, 0x80000000000, M, 8, K,
                                 binding.TG_EPILOGUE_NONE, None)
    assert st == binding.TG_ERR_SCRATCH_LIMIT
    assert "TG_NOALLOC_SCRATCH_BYTES" in binding.tg_status_string(st)
