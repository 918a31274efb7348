"""Randomised parity sweep through the C ABI: seeded random shapes (tiny,
ragged, unaligned K and N), every configuration able to run the shape, both
work divisions and every epilogue, against the fp64 oracle.  Integer-valued
inputs with the bias-only epilogue are compared bit for bit; the rest under
the acceptance rule."""
import numpy as np
import pytest

import oracle
from gpu_helpers import assert_bits_equal, assert_close, run_gpu, run_oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu

EPILOGUES = [0, 1, 2, 3, 4]


def _cases(n, seed=2024):
    rng = np.random.default_rng(seed)
    n_cfg = binding.tg_num_configs()
    out = []
    for i in range(n):
        M = int(rng.choice([1, 7, 64, 129, 255, 300, 513, 1000]))
        N = int(rng.choice([1, 8, 63, 64, 130, 200, 256, 384, 777]))
        K = int(rng.choice([1, 9, 16, 64, 65, 200, 333, 1024]))
        epi = int(rng.choice(EPILOGUES))
        if epi == 4 and N > 256:
            N = int(rng.choice([8, 64, 200, 256]))
        cfg = int(rng.integers(0, n_cfg))
        info = binding.tg_config_info(cfg)
        if epi == 4 and (info["epi_warps"] != 4 or info["block_n"] < N):
            cfg = -1
        split = int(rng.choice([0, 1, 2]))
        out.append((i, M, N, K, epi, cfg, split))
    return out


@pytest.mark.parametrize("case", _cases(30), ids=lambda c: "r%d_%dx%dx%d_e%d_c%d_s%d" % c)
def test_random_shapes(case):
    i, M, N, K, epi, cfg, split = case
    A, B, bias = wl.make_inputs(M, N, K, seed=5000 + i, bias=True,
                                b_scale=1.0 / np.sqrt(max(K, 1)))
    C = run_gpu(A, B, bias, epi, config_id=cfg, split=split)
    assert_close(C, run_oracle(A, B, bias, epi), f"random case {case}")


@pytest.mark.parametrize("case", _cases(12, seed=77), ids=lambda c: "i%d_%dx%dx%d_c%d_s%d" % (
    c[0], c[1], c[2], c[3], c[5], c[6]))
def test_random_integer_bit_exact(case):
    i, M, N, K, _, cfg, split = case
    A, B, bias = wl.integer_inputs(M, N, K, seed=6000 + i, lo=-2, hi=2, bias=True)
    exact = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), 1)
    C = run_gpu(A, B, bias, 1, config_id=cfg, split=split)
    assert_bits_equal(C, exact, f"integer case {case}")
