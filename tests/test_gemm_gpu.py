"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every test here launches kernels on cuda:0 and is marked ``gpu``.  Inputs are
the seeded synthetic workloads; expected values come only from ``oracle``.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (assert_bits_equal, assert_close, assert_close_blocked, run_gpu,
                         run_oracle)
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NONE, BIAS, GELU = binding.TG_EPILOGUE_NONE, binding.TG_EPILOGUE_BIAS, binding.TG_EPILOGUE_BIAS_GELU
CONFIG_IDS = list(range(binding.tg_num_configs()))


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    torch.cuda.synchronize()


# ---------------------------------------------------------------- exact layouts

@pytest.mark.parametrize("config_id", CONFIG_IDS)
@pytest.mark.parametrize("M,N", [(128, 256), (300, 200), (257, 520)])
def test_identity_left_bit_exact(config_id, M, N):
    """A = I: C must equal B bit for bit (pins A/B layouts and descriptors)."""
    K = M
    _, B, _ = wl.make_inputs(1, N, K, seed=100 + M)
    A = torch.eye(M, dtype=torch.float16)
    C = run_gpu(A, B, None, NONE, config_id=config_id)
    assert_bits_equal(C, wl.to_bits(B), f"I @ B cfg{config_id}")


@pytest.mark.parametrize("config_id", CONFIG_IDS)
@pytest.mark.parametrize("M,K", [(128, 64), (200, 136), (129, 264)])
def test_identity_right_bit_exact(config_id, M, K):
    A, _, _ = wl.make_inputs(M, 1, K, seed=200 + K)
    B = torch.eye(K, dtype=torch.float16)
    C = run_gpu(A, B, None, NONE, config_id=config_id)
    assert_bits_equal(C, wl.to_bits(A), f"A @ I cfg{config_id}")


@pytest.mark.parametrize("config_id", [0, 1, 2])
def test_permutations_bit_exact(config_id):
    M = K = 384
    N = 328
    _, B, _ = wl.make_inputs(1, N, K, seed=300)
    p = wl.permutation(M, seed=301)
    P = torch.zeros(M, K, dtype=torch.float16)
    P[np.arange(M), p] = 1.0
    C = run_gpu(P, B, None, NONE, config_id=config_id)
    assert_bits_equal(C, wl.to_bits(B)[p], "P @ B")
    A, _, _ = wl.make_inputs(200, 1, 264, seed=302)
    q = wl.permutation(264, seed=303)
    Q = torch.zeros(264, 264, dtype=torch.float16)
    Q[q, np.arange(264)] = 1.0
    C = run_gpu(A, Q, None, NONE, config_id=config_id)
    assert_bits_equal(C, wl.to_bits(A)[:, q], "A @ Q")


@pytest.mark.parametrize("config_id", CONFIG_IDS)
def test_integer_inputs_bit_exact(config_id):
    A, B, bias = wl.integer_inputs(333, 520, 1000, seed=400, lo=-1, hi=1, bias=True)
    exp = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B))
    assert_bits_equal(run_gpu(A, B, None, NONE, config_id=config_id), exp, "int NONE")
    exp_b = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), oracle.EPI_BIAS)
    assert_bits_equal(run_gpu(A, B, bias, BIAS, config_id=config_id), exp_b, "int BIAS")


def test_integer_inputs_large_sums_round_like_the_oracle():
    # {-2..2} with K = 4096: sums reach beyond 2048, where fp16 spacing is 2+
    A, B, _ = wl.integer_inputs(256, 256, 4096, seed=401, lo=0, hi=2)
    exp = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B))
    assert_bits_equal(run_gpu(A, B, None, NONE), exp, "int large sums")


def test_rank1_closed_form():
    M, N, K = 256, 512, 1024
    u = torch.tensor([2.0 ** (i % 9 - 6) for i in range(M)])
    v = torch.tensor([(-1) ** j * 2.0 ** (j % 5 - 4) for j in range(N)])
    A = u[:, None].expand(M, K).to(torch.float16).contiguous()
    B = v[None, :].expand(K, N).to(torch.float16).contiguous()
    exact = (K * torch.outer(u, v).double()).numpy()
    C = run_gpu(A, B, None, NONE)
    assert_bits_equal(C, exact.astype(np.float16).view(np.uint16), "rank-1")


# ---------------------------------------------------------------- epilogue

def test_gelu_epilogue_within_one_ulp():
    """A = 0, so C = fp16(GELU(bias)): every finite fp16 value in [-16, 16]
    as the bias (all inputs the epilogue can see from a zero product)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    keep = np.isfinite(vals) & (np.abs(vals.astype(np.float64)) <= 16)
    bias = torch.from_numpy(vals[keep].copy())
    M, N, K = 128, bias.numel(), 64
    A = torch.zeros(M, K, dtype=torch.float16)
    B = torch.zeros(K, N, dtype=torch.float16)
    C = run_gpu(A, B, bias, GELU)
    ref = run_oracle(A, B, bias, oracle.EPI_BIAS_GELU)
    exp_bits = oracle.double_to_half_rne(ref).astype(np.int32)
    got_bits = wl.to_bits(C).astype(np.int32)
    # fp16 bit patterns of same-sign values are monotone: ulp distance = |diff|
    same_sign = (exp_bits & 0x8000) == (got_bits & 0x8000)
    dist = np.where(same_sign, np.abs(exp_bits - got_bits),
                    (exp_bits & 0x7FFF) + (got_bits & 0x7FFF))
    assert dist.max() <= 1, f"max ulp distance {dist.max()}"
    assert_close(C, ref, "gelu sweep")


def test_bias_epilogue_exact_when_representable():
    M, N, K = 200, 300, 128
    A, B, _ = wl.integer_inputs(M, N, K, seed=500, lo=-1, hi=1)
    bias = torch.arange(N, dtype=torch.float32).remainder(17).sub(8).to(torch.float16)
    exp = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), oracle.EPI_BIAS)
    assert_bits_equal(run_gpu(A, B, bias, BIAS), exp, "bias exact")


def test_gelu_without_bias_is_gelu_of_product():
    A, B, _ = wl.make_inputs(192, 320, 256, seed=501)
    C = run_gpu(A, B, None, GELU)
    assert_close(C, run_oracle(A, B, None, oracle.EPI_BIAS_GELU), "gelu no bias")


def test_none_epilogue_ignores_bias():
    A, B, bias = wl.make_inputs(130, 136, 200, seed=502, bias=True)
    c1 = run_gpu(A, B, bias, NONE)
    c2 = run_gpu(A, B, None, NONE)
    assert torch.equal(c1, c2)


# ---------------------------------------------------------------- shapes

RAGGED = [(1, 1, 1), (1, 8, 8), (7, 9, 13), (63, 65, 64), (64, 64, 65), (65, 63, 127),
          (127, 129, 128), (128, 128, 129), (129, 257, 255), (255, 255, 257), (300, 1, 70),
          (1, 300, 300), (17, 31, 1), (256, 264, 72)]


@pytest.mark.parametrize("M,N,K", RAGGED)
@pytest.mark.parametrize("epilogue", [NONE, GELU])
def test_ragged_shapes(M, N, K, epilogue):
    A, B, bias = wl.make_inputs(M, N, K, seed=M * 7919 + N * 31 + K, bias=True)
    C = run_gpu(A, B, bias, epilogue)
    assert_close(C, run_oracle(A, B, bias, epilogue), f"{M}x{N}x{K}")


@pytest.mark.parametrize("config_id", CONFIG_IDS)
def test_every_config_multi_tile_ragged(config_id):
    A, B, bias = wl.make_inputs(517, 777, 333, seed=600, dist="uniform", bias=True)
    C = run_gpu(A, B, bias, GELU, config_id=config_id)
    assert_close(C, run_oracle(A, B, bias, GELU), f"cfg{config_id}")


def test_k_zero_gives_epilogue_of_bias():
    M, N = 70, 90
    bias = torch.linspace(-3, 3, N).to(torch.float16)
    A = torch.zeros(M, 0, dtype=torch.float16)
    B = torch.zeros(0, N, dtype=torch.float16)
    for epi in (NONE, BIAS, GELU):
        C = run_gpu(A, B, bias, epi)
        assert_close(C, run_oracle(A, B, bias, epi), f"K=0 epi{epi}")


def test_empty_m_or_n_is_a_no_op():
    dev = torch.device("cuda:0")
    for (M, N, K) in [(0, 5, 7), (5, 0, 7), (0, 0, 0)]:
        a = torch.zeros(M, K, dtype=torch.float16, device=dev)
        b = torch.zeros(K, N, dtype=torch.float16, device=dev)
        c = binding.gemm(a, b)
        assert c.shape == (M, N)


@pytest.mark.parametrize("config_id", [-1, 0, 3, 9])
def test_misaligned_operands(config_id):
    """Views one element off a 16-byte boundary for A, B, bias and C: the
    default choice and forced TMA configurations (which repack A and B
    first), and the plain loader (which reads them in place)."""
    dev = torch.device("cuda:0")
    M, N, K = 300, 260, 200
    A, B, bias = wl.make_inputs(M, N, K, seed=700, bias=True)
    a_buf = torch.zeros(M * K + 1, dtype=torch.float16, device=dev)
    b_buf = torch.zeros(K * N + 1, dtype=torch.float16, device=dev)
    bias_buf = torch.zeros(N + 1, dtype=torch.float16, device=dev)
    c_buf = torch.zeros(M * N + 1, dtype=torch.float16, device=dev)
    a = a_buf[1:].view(M, K)
    b = b_buf[1:].view(K, N)
    bb = bias_buf[1:]
    c = c_buf[1:].view(M, N)
    a.copy_(A.to(dev))
    b.copy_(B.to(dev))
    bb.copy_(bias.to(dev))
    binding.gemm(a, b, bb, epilogue=GELU, out=c, config_id=config_id)
    torch.cuda.synchronize()
    assert c_buf[0].item() == 0.0, "wrote before C"
    assert_close(c.cpu(), run_oracle(A, B, bias, GELU), f"misaligned views, config {config_id}")


REPACK_CASES = [((200, 131, 133), 1, 0), ((200, 131, 133), 0, 1), ((64, 70, 262), 2, 3),
                ((257, 1537, 2050), 3, 5), ((130, 9, 17), 7, 6), ((96, 250, 90), 4, 4),
                ((33, 1, 7), 5, 2)]


@pytest.mark.parametrize("shape,off_a,off_b", REPACK_CASES,
                         ids=[f"{'x'.join(map(str, c[0]))}-a{c[1]}-b{c[2]}" for c in REPACK_CASES])
def test_repacked_operands_bit_exact(shape, off_a, off_b):
    """Operands whose base sits off_* elements past a 16-byte boundary and
    whose pitches are not multiples of 8 elements go through the repacking
    kernel (every load alignment and every count of valid elements in a
    row's last 16-byte group); integer-valued inputs make the exact result
    an fp16 value, so C must match it bit for bit."""
    M, N, K = shape
    dev = torch.device("cuda:0")
    A, B, _ = wl.integer_inputs(M, N, K, seed=450 + M + off_a, lo=-1, hi=1)
    a_buf = torch.zeros(M * K + 8, dtype=torch.float16, device=dev)
    b_buf = torch.zeros(K * N + 8, dtype=torch.float16, device=dev)
    a = a_buf[off_a:off_a + M * K].view(M, K)
    b = b_buf[off_b:off_b + K * N].view(K, N)
    a.copy_(A.to(dev))
    b.copy_(B.to(dev))
    c = binding.gemm(a, b, None, epilogue=NONE)
    torch.cuda.synchronize()
    assert binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream) == binding.TG_OK
    assert_bits_equal(c.cpu(), oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B)),
                      f"repacked {M}x{N}x{K} offsets {off_a},{off_b}")


@pytest.mark.parametrize("config_id", [c for c in CONFIG_IDS if binding.tg_config_info(c)["loader"] == 0])
@pytest.mark.parametrize("off_c", [1, 2, 3, 4, 5, 6, 7])
def test_unaligned_c_rows_bit_exact(config_id, off_c):
    """C whose base sits off_c elements past a 16-byte boundary, with an odd
    N (every row starts at a different alignment): each row leaves through
    aligned 16-byte vector stores plus element stores at the ends of each
    warp's run of columns.  Integer-valued inputs make the exact result an
    fp16 value, so every element must match bit for bit, and nothing before
    or after C may be written."""
    M, N, K = 130, 333, 72
    dev = torch.device("cuda:0")
    A, B, _ = wl.integer_inputs(M, N, K, seed=470 + off_c, lo=-2, hi=2)
    c_buf = torch.full((M * N + 16,), -7.0, dtype=torch.float16, device=dev)
    c = c_buf[off_c:off_c + M * N].view(M, N)
    binding.gemm(A.to(dev), B.to(dev), None, epilogue=NONE, out=c, config_id=config_id)
    torch.cuda.synchronize()
    assert binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream) == binding.TG_OK
    assert_bits_equal(c.cpu(), oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B)),
                      f"unaligned C offset {off_c} config {config_id}")
    guard = torch.cat([c_buf[:off_c], c_buf[off_c + M * N:]]).cpu()
    assert bool((guard == -7.0).all()), "wrote outside C"


TAIL_CASES = [((3000, 1537, 2050), 1, NONE), ((2048, 2306, 64), 0, BIAS), ((3000, 1552, 130), 1, BIAS),
              ((2048, 2307, 64), 0, NONE), ((1100, 2051, 96), 0, NONE)]


@pytest.mark.parametrize("shape,config_id,epi", TAIL_CASES,
                         ids=["x".join(map(str, c[0])) for c in TAIL_CASES])
def test_thin_n_remainder_bit_exact(shape, config_id, epi):
    """N = q * 256 + r where the last column of 256-wide tiles would add a
    wave: for r <= 4 the GEMM covers q * 256 columns and the CUDA-core tail
    kernel the last r (r = 1, 2, 3); a wider remainder (r = 16) and a shape
    whose extra column of tiles fits the wave keep whole tiles.  Integer-valued
    inputs make the exact result an fp16 value."""
    M, N, K = shape
    A, B, bias = wl.integer_inputs(M, N, K, seed=480 + N, lo=-1, hi=1, bias=True)
    exp = oracle.gemm_int_exact(wl.to_bits(A), wl.to_bits(B),
                                wl.to_bits(bias) if epi == BIAS else None,
                                oracle.EPI_BIAS if epi == BIAS else oracle.EPI_NONE)
    C = run_gpu(A, B, bias if epi == BIAS else None, epi, config_id=config_id)
    assert_bits_equal(C, exp, f"tail {M}x{N}x{K} config {config_id}")


# ---------------------------------------------------------------- the workloads

@pytest.mark.parametrize("name", ["gemm_256", "gemm_2048", "fused_2048", "ragged_fused",
                                  "fused_tanh_2048", "softmax_8192x256x4096",
                                  "deepk_fused_1024x1024x8192", "deepk_512x512x16384"])
def test_workload_full_parity(name):
    w = wl.WORKLOADS[name]
    A, B, bias = wl.workload_inputs(w)
    C = run_gpu(A, B, bias, w.epilogue)
    assert_close(C, run_oracle(A, B, bias, w.epilogue), name)


@pytest.mark.parametrize("name", ["fused_8192", "fused_8192_literal"])
def test_large_workload_full_parity(name):
    """Full-size 8192^3 launch in the benchmark's configuration, every one of
    the 67,108,864 outputs against the whole fp64 oracle result (about 40 s
    of oracle time on 16 host cores per workload)."""
    w = wl.WORKLOADS[name]
    A, B, bias = wl.workload_inputs(w)
    C = run_gpu(A, B, bias, w.epilogue)
    ref = run_oracle(A, B, bias, w.epilogue)
    assert ref.shape == (w.M, w.N)
    assert_close_blocked(C, ref, name)


def test_deterministic():
    A, B, bias = wl.make_inputs(1000, 1100, 900, seed=800, bias=True)
    c1 = run_gpu(A, B, bias, GELU)
    c2 = run_gpu(A, B, bias, GELU)
    assert torch.equal(c1, c2)


# ---------------------------------------------------------------- host entry, errors

def test_host_entry_matches_device_entry():
    A, B, bias = wl.make_inputs(520, 333, 264, seed=900, bias=True)
    c_host = binding.gemm_host(A.pin_memory(), B.pin_memory(), bias.pin_memory(), epilogue=GELU)
    c_dev = run_gpu(A, B, bias, GELU)
    assert torch.equal(c_host, c_dev)


@pytest.mark.parametrize("M,N,K", [(5000, 300, 200), (4099, 129, 201), (16384, 64, 64)])
def test_host_entry_in_row_panels(M, N, K):
    """Problems of more than 1024 rows go through the host entry in row panels
    (uploads, panel GEMMs and downloads overlapped on three streams); every
    panel boundary and an unaligned K (repacked per panel) against the oracle,
    twice in a row on the same workspace."""
    A, B, bias = wl.make_inputs(M, N, K, seed=901 + K, dist="uniform", bias=True)
    ref = run_oracle(A, B, bias, GELU)
    ws = torch.empty(binding.tg_gemm_host_workspace_size(M, N, K, True), dtype=torch.uint8,
                     device="cuda:0")
    for _ in range(2):
        c_host = binding.gemm_host(A.pin_memory(), B.pin_memory(), bias.pin_memory(),
                                   epilogue=GELU, workspace=ws)
        assert binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream) == 0
        assert_close(c_host, ref, f"host entry {M}x{N}x{K}")


@pytest.mark.parametrize("config_id", [0, 3, 9])
def test_bounded_wait_reports_timeout_and_context_survives(config_id):
    """A skipped operand load makes the consumer's bounded wait expire: the
    kernel exits cleanly, the host reads TG_ERR_TIMEOUT, and the next call
    works (config 0: CTA pair, config 3: single CTA)."""
    dev = torch.device("cuda:0")
    A, B, bias = wl.make_inputs(256, 512, 512, seed=1000, bias=True)
    a, b, bb = A.to(dev), B.to(dev), bias.to(dev)
    c = torch.empty(256, 512, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    assert binding.tg_gemm_check_error(stream) == binding.TG_OK
    st = binding.tg_gemm_ex(a.data_ptr(), b.data_ptr(), bb.data_ptr(), c.data_ptr(), 256, 512, 512,
                            GELU, config_id=config_id, wait_limit_ns=50_000_000,
                            inject=binding.TG_INJECT_SKIP_FIRST_LOAD, stream=stream)
    assert st == binding.TG_OK
    assert binding.tg_gemm_check_error(stream) == binding.TG_ERR_TIMEOUT
    assert binding.tg_gemm_check_error(stream) == binding.TG_OK      # cleared
    C = run_gpu(A, B, bias, GELU)
    assert_close(C, run_oracle(A, B, bias, GELU), "after timeout")


def test_invalid_arguments_on_device():
    dev = torch.device("cuda:0")
    a = torch.zeros(64, 64, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    # C overlapping A
    st = binding.tg_gemm(a.data_ptr(), a.data_ptr(), None, a.data_ptr(), 64, 64, 64, NONE, stream)
    assert st == binding.TG_ERR_INVALID_ARG
    with pytest.raises(binding.TgError):
        binding.gemm(a, a, epilogue=NONE, config_id=999)


# ---------------------------------------------------------------- tanh GELU and row softmax

TANH, SOFTMAX = binding.TG_EPILOGUE_BIAS_GELU_TANH, binding.TG_EPILOGUE_BIAS_SOFTMAX


def _ulp_distance(got_bits, exp_bits):
    g = got_bits.astype(np.int32)
    e = exp_bits.astype(np.int32)
    same = (e & 0x8000) == (g & 0x8000)
    return np.where(same, np.abs(e - g), (e & 0x7FFF) + (g & 0x7FFF))


def test_gelu_tanh_epilogue_within_one_ulp():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    keep = np.isfinite(vals) & (np.abs(vals.astype(np.float64)) <= 16)
    bias = torch.from_numpy(vals[keep].copy())
    M, N, K = 128, bias.numel(), 64
    A = torch.zeros(M, K, dtype=torch.float16)
    B = torch.zeros(K, N, dtype=torch.float16)
    C = run_gpu(A, B, bias, TANH)
    ref = run_oracle(A, B, bias, oracle.EPI_BIAS_GELU_TANH)
    dist = _ulp_distance(wl.to_bits(C), oracle.double_to_half_rne(ref))
    assert dist.max() <= 1, f"max ulp distance {dist.max()}"


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (129, 257, 300), (300, 520, 64)])
def test_gelu_tanh_epilogue_shapes(M, N, K):
    A, B, bias = wl.make_inputs(M, N, K, seed=M + N + K, bias=True)
    assert_close(run_gpu(A, B, bias, TANH), run_oracle(A, B, bias, TANH), f"tanh {M}x{N}x{K}")


def _check_softmax(C, ref, what):
    assert_close(C, ref, what)
    c = C.to(torch.float64).numpy()
    # tighter: fp16 rounding of a probability plus fp32 arithmetic
    err = np.abs(c - ref)
    assert np.all(err <= 1e-3 * ref + 2e-7), f"{what}: max rel err {np.max(err / (ref + 1e-30)):.2e}"
    assert np.allclose(c.sum(axis=1), 1.0, atol=2e-2), what


SOFTMAX_SHAPES = [(1, 1, 1), (7, 5, 13), (130, 64, 100), (300, 100, 257), (1000, 256, 512),
                  (257, 200, 64), (64, 33, 2050)]


@pytest.mark.parametrize("M,N,K", SOFTMAX_SHAPES)
def test_softmax_epilogue(M, N, K):
    A, B, bias = wl.make_inputs(M, N, K, seed=3 * M + N + 7 * K, bias=True)
    _check_softmax(run_gpu(A, B, bias, SOFTMAX), run_oracle(A, B, bias, SOFTMAX),
                   f"softmax {M}x{N}x{K}")


@pytest.mark.parametrize("config_id", [5, 6, 7, 8])
def test_softmax_every_capable_config(config_id):
    info = binding.tg_config_info(config_id)
    N = min(info["block_n"], 200)
    A, B, bias = wl.make_inputs(517, N, 333, seed=900 + config_id, dist="uniform", bias=True)
    _check_softmax(run_gpu(A, B, bias, SOFTMAX, config_id=config_id),
                   run_oracle(A, B, bias, SOFTMAX), f"softmax cfg{config_id}")


def test_softmax_without_bias_and_with_k0():
    A, B, _ = wl.make_inputs(100, 77, 90, seed=950)
    _check_softmax(run_gpu(A, B, None, SOFTMAX), run_oracle(A, B, None, SOFTMAX), "no bias")
    bias = torch.linspace(-3, 3, 50).to(torch.float16)
    A0 = torch.zeros(9, 0, dtype=torch.float16)
    B0 = torch.zeros(0, 50, dtype=torch.float16)
    _check_softmax(run_gpu(A0, B0, bias, SOFTMAX), run_oracle(A0, B0, bias, SOFTMAX), "K=0")


def test_softmax_rejects_wide_rows_and_incapable_configs():
    dev = torch.device("cuda:0")
    a = torch.zeros(64, 64, dtype=torch.float16, device=dev)
    b = torch.zeros(64, 300, dtype=torch.float16, device=dev)
    with pytest.raises(binding.TgError):
        binding.gemm(a, b, epilogue=SOFTMAX)            # N > 256
    b2 = torch.zeros(64, 128, dtype=torch.float16, device=dev)
    with pytest.raises(binding.TgError):
        binding.gemm(a, b2, epilogue=SOFTMAX, config_id=0)   # 8 epilogue warps
