"""tg_gemm_noalloc, the allocation-free entry point, against tg_gemm.

Callers that must not allocate device memory (an engine whose own allocator
owns nearly all of HBM, a latency-critical loop that must stay out of the
driver's allocator) use tg_gemm_noalloc: repacking scratch for unaligned
operands comes from a fixed device array inside the library instead of a
memory pool.  These tests call it through the C ABI and compare its output
with tg_gemm's, under the same acceptance rule as the parity tests, on calls
in a row that reuse the shared scratch array.  Every buffer handed to the
library is a real device allocation of the size the call implies, including
in the calls that are expected to be rejected.  The file is named so that
pytest collects it last.
"""
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


def _scratch_needed(M, N, K):
    """Bytes of repacking scratch a call with 16-byte aligned bases and no
    thin N remainder needs, as the header states it: 2*M*K8 rounded up to 256
    when K % 8 != 0, plus 2*K*N8 rounded up to 256 when N % 8 != 0."""
    k8, n8 = -(-K // 8) * 8, -(-N // 8) * 8
    a = 0 if K % 8 == 0 else -(-(2 * M * k8) // 256) * 256
    b = 0 if N % 8 == 0 else -(-(2 * K * n8) // 256) * 256
    return a + b


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


@pytest.mark.parametrize("M,N,K,seed", [
    (1000, 777, 1030, 11),   # A and B repacked, after a larger call
    (700, 333, 512, 13),     # B alone repacked: it starts at the array's first byte
    (640, 256, 390, 14),     # A alone repacked
    (512, 1024, 768, 12),    # aligned: no scratch
])
def test_noalloc_repacking_cases(M, N, K, seed):
    # The scratch keeps the bytes of whatever call ran before.
    a, b, bias = _device_inputs(M, N, K, seed=seed, dist="normal")
    ref = _run(binding.tg_gemm, a, b, bias, M, N, K, binding.TG_EPILOGUE_BIAS).double().numpy()
    got = _run(binding.tg_gemm_noalloc, a, b, bias, M, N, K, binding.TG_EPILOGUE_BIAS)
    assert_close(got, ref, f"tg_gemm_noalloc {M}x{N}x{K}")


def test_noalloc_accepts_exactly_its_scratch_and_rejects_one_block_more():
    # K = 127 repacks A into 128-element rows: 256 bytes of scratch per row.
    # 131072 rows need exactly TG_NOALLOC_SCRATCH_BYTES (accepted); 131073
    # rows need 256 bytes more (rejected before anything is launched).
    limit = binding.noalloc_scratch_bytes()
    K, N = 127, 8
    M_fit = limit // 256
    assert _scratch_needed(M_fit, N, K) == limit
    assert _scratch_needed(M_fit + 1, N, K) == limit + 256
    epi = binding.TG_EPILOGUE_NONE
    a, b, bias = _device_inputs(M_fit + 1, N, K, seed=15, dist="normal")
    a_fit = a[:M_fit]
    ref = _run(binding.tg_gemm, a_fit, b, bias, M_fit, N, K, epi).double().numpy()
    got = _run(binding.tg_gemm_noalloc, a_fit, b, bias, M_fit, N, K, epi)
    assert_close(got, ref, "tg_gemm_noalloc at exactly its scratch size")

    c = torch.full((M_fit + 1, N), 7.0, dtype=torch.float16, device=a.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = binding.tg_gemm_noalloc(a.data_ptr(), b.data_ptr(), None, c.data_ptr(), M_fit + 1, N, K,
                                 epi, stream)
    assert st == binding.TG_ERR_SCRATCH_LIMIT, binding.tg_status_string(st)
    assert "TG_NOALLOC_SCRATCH_BYTES" in binding.tg_status_string(st)
    torch.cuda.synchronize()
    assert bool((c == 7.0).all()), "a rejected call must launch nothing"
