"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle,
compare under the acceptance rule.

Acceptance (fp16 output vs the fp64 oracle), from the problem statement:
  * relative Frobenius error ||C - ref||_F / ||ref||_F <= 2e-3,
  * every element |C - ref| <= 1e-2 * max(1, |ref|),
  * no NaN / Inf in C.
Where the exact result is representable (identity, permutation and
integer-valued inputs) the comparison is bit-exact instead.
"""
import numpy as np
import torch

import oracle
from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import workloads as wl

REL_FROB_TOL = 2e-3
ELEM_TOL = 1e-2


def run_gpu(A, B, bias, epilogue, config_id=-1, **kw):
    """CPU fp16 tensors in, CPU fp16 C out, through tg_gemm_ex."""
    dev = torch.device("cuda:0")
    a = A.to(dev)
    b = B.to(dev)
    bb = bias.to(dev) if bias is not None else None
    c = binding.gemm(a, b, bb, epilogue=epilogue, config_id=config_id, **kw)
    torch.cuda.synchronize()
    st = binding.tg_gemm_check_error(torch.cuda.current_stream().cuda_stream)
    assert st == binding.TG_OK, binding.tg_status_string(st)
    return c.cpu()


def run_oracle(A, B, bias, epilogue, rows=None):
    return oracle.gemm(wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias), epilogue, rows=rows)


def assert_close(C, ref, what=""):
    c = C.to(torch.float64).numpy() if isinstance(C, torch.Tensor) else np.asarray(C, np.float64)
    assert c.shape == ref.shape, (c.shape, ref.shape)
    assert np.all(np.isfinite(c)), f"{what}: non-finite output"
    err = np.abs(c - ref)
    bound = ELEM_TOL * np.maximum(1.0, np.abs(ref))
    bad = err > bound
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements over tolerance; first at ({i},{j}): "
                             f"got {c[i, j]!r} want {ref[i, j]!r}")
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(c - ref) / nref if nref > 0 else np.linalg.norm(c)
    assert rel <= REL_FROB_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FROB_TOL}"
    return rel


def assert_close_blocked(C, ref, what="", block_rows=512):
    """assert_close over the whole output, taken in row blocks so that a
    full 8192 x 8192 comparison needs no (M, N) temporaries beyond the two
    operands: the per-element rule and the finiteness check per block, the
    relative Frobenius error from sums accumulated over every block."""
    c_all = C if isinstance(C, torch.Tensor) else torch.from_numpy(np.asarray(C))
    assert tuple(c_all.shape) == ref.shape, (tuple(c_all.shape), ref.shape)
    err2 = 0.0
    ref2 = 0.0
    for r0 in range(0, ref.shape[0], block_rows):
        r1 = min(ref.shape[0], r0 + block_rows)
        c = c_all[r0:r1].to(torch.float64).numpy()
        rb = ref[r0:r1]
        assert np.all(np.isfinite(c)), f"{what}: non-finite output in rows {r0}..{r1}"
        err = np.abs(c - rb)
        bad = err > ELEM_TOL * np.maximum(1.0, np.abs(rb))
        if bad.any():
            i, j = np.argwhere(bad)[0]
            raise AssertionError(f"{what}: {bad.sum()} elements over tolerance in rows "
                                 f"{r0}..{r1}; first at ({r0 + i},{j}): got {c[i, j]!r} "
                                 f"want {rb[i, j]!r}")
        err2 += float(np.sum(err * err))
        ref2 += float(np.sum(rb * rb))
    rel = np.sqrt(err2 / ref2) if ref2 > 0 else np.sqrt(err2)
    assert rel <= REL_FROB_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FROB_TOL}"
    return rel


def assert_bits_equal(C, expected_bits, what=""):
    got = wl.to_bits(C.contiguous())
    exp = np.asarray(expected_bits, dtype=np.uint16)
    assert got.shape == exp.shape
    diff = got != exp
    if diff.any():
        i, j = np.argwhere(diff)[0]
        raise AssertionError(f"{what}: {diff.sum()} elements differ; first at ({i},{j}): "
                             f"got {got[i, j]:#06x} want {exp[i, j]:#06x}")
