"""CPU reference (oracle) for the fused fp16 GEMM C = g(A.B + bias).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never imports it, and it imports
nothing from the product package.

The arithmetic lives in ``tg_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only builds that file with gcc, loads it with ctypes and passes
numpy arrays.  Every function cites the passage it follows in the C file:

* the GEMM itself -- "Designing High-Performance GPU Kernels with TileLang"
  (thecryptopost.io), the make_matmul kernel (fp16 A[M,K], B[K,N], C[M,N],
  fp32 accumulator);
* the bias + GELU epilogue -- the same tutorial (ainovat.com), fused-epilogue
  section (bias add and GELU on the accumulator before the one output write);
* the tanh approximation of GELU -- Hendrycks & Gimpel, "Gaussian Error
  Linear Units", section 2;
* the row softmax epilogue -- the same tutorial (ainovat.com), row-wise
  softmax section (per-row max and sum, then normalisation);
* attention forward -- the same tutorial (ainovat.com), FlashAttention
  section (softmax(scale Q K^T) V, causal and non-causal), as its plain
  definition.

Pins (tests/test_oracle_pins.py) hold it to closed forms, exact rational
arithmetic, exhaustive codec checks against numpy, and scipy's normal CDF.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

EPI_NONE = 0
EPI_BIAS = 1
EPI_BIAS_GELU = 2
EPI_BIAS_GELU_TANH = 3
EPI_BIAS_SOFTMAX = 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tg_oracle.c")
_LIB = os.path.join(_HERE, "libtg_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile tg_oracle.c into oracle/libtg_oracle.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O3", "-std=c11", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
               "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.tgo_gemm_rows.argtypes = [u16p, u16p, u16p, i64, i64, i64, ctypes.c_int, i64p, i64, f64p]
        lib.tgo_gemm_rows.restype = ctypes.c_int
        lib.tgo_gemm.argtypes = [u16p, u16p, u16p, i64, i64, i64, ctypes.c_int, f64p]
        lib.tgo_gemm.restype = ctypes.c_int
        lib.tgo_gemm_int_exact.argtypes = [u16p, u16p, u16p, i64, i64, i64, ctypes.c_int, u16p]
        lib.tgo_gemm_int_exact.restype = ctypes.c_int
        lib.tgo_half_to_double_n.argtypes = [u16p, i64, f64p]
        lib.tgo_double_to_half_rne_n.argtypes = [f64p, i64, u16p]
        lib.tgo_gelu_n.argtypes = [f64p, i64, f64p]
        lib.tgo_gelu_tanh_n.argtypes = [f64p, i64, f64p]
        lib.tgo_num_threads.restype = ctypes.c_int
        lib.tgo_set_num_threads.argtypes = [ctypes.c_int]
        lib.tgo_set_num_threads.restype = ctypes.c_int
        lib.tgo_attention.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_int,
                                      ctypes.c_double, i64p, i64, f64p]
        lib.tgo_attention.restype = ctypes.c_int
        _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """fp16 data (numpy float16 or uint16 bits) -> contiguous uint16 bits."""
    if x is None:
        return None
    x = np.asarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    if x.dtype != np.uint16:
        raise TypeError(f"expected float16 or uint16 bits, got {x.dtype}")
    return np.ascontiguousarray(x)


def _ptr(a, ctype):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleError(RuntimeError):
    pass


def gemm(A, B, bias=None, epilogue: int = EPI_NONE, rows=None) -> np.ndarray:
    """Reference g(A.B + bias) in float64.

    A: (M, K) fp16, B: (K, N) fp16, bias: (N,) fp16 or None.  With ``rows``
    (a sequence of row indices) only those rows are computed and the result
    is (len(rows), N); otherwise it is (M, N).
    """
    A, B, bias = _bits(A), _bits(B), _bits(bias)
    M, K = A.shape
    K2, N = B.shape
    if K2 != K:
        raise ValueError("inner dimensions differ")
    if bias is not None and bias.shape != (N,):
        raise ValueError("bias must have shape (N,)")
    lib = _load()
    if rows is None:
        out = np.empty((M, N), dtype=np.float64)
        st = lib.tgo_gemm(_ptr(A, ctypes.c_uint16), _ptr(B, ctypes.c_uint16),
                          _ptr(bias, ctypes.c_uint16), M, N, K, epilogue,
                          _ptr(out, ctypes.c_double))
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((r.size, N), dtype=np.float64)
        st = lib.tgo_gemm_rows(_ptr(A, ctypes.c_uint16), _ptr(B, ctypes.c_uint16),
                               _ptr(bias, ctypes.c_uint16), M, N, K, epilogue,
                               _ptr(r, ctypes.c_int64), r.size, _ptr(out, ctypes.c_double))
    if st != 0:
        raise OracleError(f"oracle gemm failed with status {st}")
    return out


def gemm_int_exact(A, B, bias=None, epilogue: int = EPI_NONE) -> np.ndarray:
    """Exact result for integer-valued inputs, correctly rounded to fp16.

    Returns the (M, N) uint16 fp16 bit patterns.  Raises OracleError if any
    input is not an integer below 2048 in magnitude, or for an epilogue other
    than NONE and BIAS.
    """
    A, B, bias = _bits(A), _bits(B), _bits(bias)
    M, K = A.shape
    _, N = B.shape
    out = np.empty((M, N), dtype=np.uint16)
    st = _load().tgo_gemm_int_exact(_ptr(A, ctypes.c_uint16), _ptr(B, ctypes.c_uint16),
                                    _ptr(bias, ctypes.c_uint16), M, N, K, epilogue,
                                    _ptr(out, ctypes.c_uint16))
    if st != 0:
        raise OracleError(f"oracle int-exact gemm failed with status {st}")
    return out


def attention(Q, K, V, causal: bool = False, scale=None, rows=None) -> np.ndarray:
    """Reference attention forward in float64.

    Q: (B, H, Sq, D), K and V: (B, H, Sk, D), fp16 (or uint16 bits).  ``scale``
    defaults to 1/sqrt(D).  Returns (B, H, Sq, D); with ``rows`` (flat query
    indices (b * H + h) * Sq + i) only those rows, as (len(rows), D).
    """
    Q, K, V = _bits(Q), _bits(K), _bits(V)
    if Q.ndim != 4 or K.ndim != 4 or V.ndim != 4:
        raise ValueError("Q, K, V must be (B, H, S, D)")
    B, H, Sq, D = Q.shape
    if K.shape[:2] != (B, H) or K.shape[3] != D or V.shape != K.shape:
        raise ValueError("K and V must be (B, H, Sk, D) matching Q")
    Sk = K.shape[2]
    sc = 1.0 / np.sqrt(D) if scale is None else float(scale)
    if rows is None:
        r = None
        out = np.empty((B, H, Sq, D), dtype=np.float64)
        n = B * H * Sq
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((r.size, D), dtype=np.float64)
        n = r.size
    st = _load().tgo_attention(_ptr(Q, ctypes.c_uint16), _ptr(K, ctypes.c_uint16),
                               _ptr(V, ctypes.c_uint16), B, H, Sq, Sk, D, 1 if causal else 0, sc,
                               _ptr(r, ctypes.c_int64), n, _ptr(out, ctypes.c_double))
    if st != 0:
        raise OracleError(f"oracle attention failed with status {st}")
    return out


def half_to_double(bits) -> np.ndarray:
    """The oracle's own fp16 decoder, elementwise."""
    b = _bits(np.asarray(bits, dtype=np.uint16))
    out = np.empty(b.shape, dtype=np.float64)
    _load().tgo_half_to_double_n(_ptr(b, ctypes.c_uint16), b.size, _ptr(out, ctypes.c_double))
    return out


def double_to_half_rne(x) -> np.ndarray:
    """The oracle's own double -> fp16 encoder (nearest, ties to even); bit patterns."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    _load().tgo_double_to_half_rne_n(_ptr(x, ctypes.c_double), x.size, _ptr(out, ctypes.c_uint16))
    return out


def gelu(x) -> np.ndarray:
    """The oracle's erf-form GELU in double, elementwise."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.float64)
    _load().tgo_gelu_n(_ptr(x, ctypes.c_double), x.size, _ptr(out, ctypes.c_double))
    return out


def gelu_tanh(x) -> np.ndarray:
    """The oracle's tanh-approximation GELU in double, elementwise."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.float64)
    _load().tgo_gelu_tanh_n(_ptr(x, ctypes.c_double), x.size, _ptr(out, ctypes.c_double))
    return out


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().tgo_num_threads())


def set_num_threads(n: int) -> int:
    """Threads for the oracle's later calls from this thread (timing only: the
    results do not depend on it); returns the previous count."""
    return int(_load().tgo_set_num_threads(int(n)))
