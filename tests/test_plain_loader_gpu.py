"""The plain operand loader (configurations with loader == 1): four loader
warps copy A and B tiles with ordinary global loads into the tensor core's
swizzled shared-memory layout, for any row pitch, instead of TMA after a
repacking pass.  Parity against the oracle through the C ABI, on shapes and
views whose rows are not 16-byte aligned, with both work divisions.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bits_equal, assert_close, run_gpu, run_oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NONE, BIAS, GELU, SOFTMAX = 0, 1, 2, 4


def plain_configs():
    return [i for i in range(binding.tg_num_configs()) if binding.tg_config_info(i)["loader"] == 1]


def test_there_are_plain_configs():
    ids = plain_configs()
    assert ids, "no plain-loader configuration"
    for i in ids:
        c = binding.tg_config_info(i)
        assert c["cta_pair"] == 0 and c["epi_warps"] == 4


def _views(A, B, bias, off_a, off_b, off_c=0):
    """Device copies of A, B, bias whose first element sits off_* elements
    past a 16-byte boundary; C likewise.  Returns (a, b, bias, c, c_buf)."""
    dev = torch.device("cuda:0")
    M, K = A.shape
    N = B.shape[1]
    a_buf = torch.zeros(M * K + 8, dtype=torch.float16, device=dev)
    b_buf = torch.zeros(K * N + 8, dtype=torch.float16, device=dev)
    c_buf = torch.zeros(M * N + 8, dtype=torch.float16, device=dev)
    a = a_buf[off_a:off_a + M * K].view(M, K)
    b = b_buf[off_b:off_b + K * N].view(K, N)
    c = c_buf[off_c:off_c + M * N].view(M, N)
    a.copy_(A.to(dev))
    b.copy_(B.to(dev))
    bb = bias.to(dev) if bias is not None else None
    return a, b, bb, c, c_buf


SHAPES = [(300, 257, 199), (129, 1537, 2050), (517, 64, 71), (1, 1, 1), (256, 256, 256),
          (130, 300, 1)]


@pytest.mark.parametrize("split", [1, 2])
@pytest.mark.parametrize("shape", SHAPES, ids=["x".join(map(str, s)) for s in SHAPES])
def test_integer_inputs_bit_exact(shape, split):
    """Integer-valued inputs: every partial sum is exact, so the fp16 result
    must equal the correctly rounded exact sum bit for bit."""
    M, N, K = shape
    A, B, bias = wl.integer_inputs(M, N, K, seed=900 + M + N + K, lo=-2, hi=2, bias=True)
    exact = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), BIAS)
    for cfg in plain_configs():
        C = run_gpu(A, B, bias, BIAS, config_id=cfg, split=split)
        assert_bits_equal(C, exact, f"config {cfg} split {split} {shape}")


@pytest.mark.parametrize("offsets", [(1, 1), (2, 3), (4, 0), (0, 1), (3, 6)])
def test_offset_views(offsets):
    """A and B views starting 2, 4, 6, 8 or 12 bytes past a 16-byte boundary,
    so that rows mix 16-byte, 4-byte and 2-byte alignment."""
    M, N, K = 333, 181, 259
    A, B, bias = wl.make_inputs(M, N, K, seed=910 + sum(offsets), bias=True)
    ref = run_oracle(A, B, bias, GELU)
    for cfg in plain_configs():
        a, b, bb, c, c_buf = _views(A, B, bias, offsets[0], offsets[1], 1)
        binding.gemm(a, b, bb, epilogue=GELU, out=c, config_id=cfg)
        torch.cuda.synchronize()
        assert binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream) == 0
        assert c_buf[0].item() == 0.0, "wrote before C"
        assert_close(c.cpu(), ref, f"config {cfg} offsets {offsets}")


@pytest.mark.parametrize("split", [1, 2])
def test_ragged_workload(split):
    w = wl.WORKLOADS["ragged_fused"]
    A, B, bias = wl.workload_inputs(w)
    ref = run_oracle(A, B, bias, w.epilogue)
    for cfg in plain_configs():
        C = run_gpu(A, B, bias, w.epilogue, config_id=cfg, split=split)
        assert_close(C, ref, f"ragged_fused config {cfg} split {split}")


def test_softmax_epilogue_on_unaligned_rows():
    M, N, K = 700, 201, 333
    A, B, bias = wl.make_inputs(M, N, K, seed=920, bias=True, b_scale=1 / np.sqrt(K))
    ref = run_oracle(A, B, bias, SOFTMAX)
    for cfg in plain_configs():
        if binding.tg_config_info(cfg)["block_n"] < N:
            continue
        C = run_gpu(A, B, bias, SOFTMAX, config_id=cfg)
        assert_close(C, ref, f"softmax config {cfg}")


def test_default_choice_for_unaligned_shapes_repacks_for_tma():
    """The plain loader's loads are latency-bound (8 to 20 times slower than
    repacking plus TMA on B200), so shapes outside the tuned table whose rows
    are not 16-byte aligned are repacked by default; forcing the plain loader
    gives the same result."""
    M, N, K = 1000, 777, 1030
    c = binding.tg_gemm_select_config(M, N, K, GELU, 148)
    assert c["loader"] == 0
    assert binding.tg_gemm_launch_count(0x1000, 0x2000, None, 0x10000000, M, N, K, GELU) == 2
    A, B, bias = wl.make_inputs(M, N, K, seed=930, dist="uniform", bias=True)
    ref = run_oracle(A, B, bias, GELU)
    assert_close(run_gpu(A, B, bias, GELU), ref, "default choice")
    for cfg in plain_configs():
        assert_close(run_gpu(A, B, bias, GELU, config_id=cfg), ref, f"forced config {cfg}")
