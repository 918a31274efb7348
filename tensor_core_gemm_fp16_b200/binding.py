"""ctypes binding of libtg_gemm.so (include/tg_gemm.h, include/tg_attention.h),
argument marshalling only.

The raw entry points keep the C names (``tg_gemm``, ``tg_gemm_ex``, ...) and
take integers for pointers and the stream.  ``gemm`` / ``gemm_host`` are the
torch-tensor conveniences: they check dtype, shape, contiguity and device,
pass ``data_ptr()`` and the current stream, and raise on a non-OK status.
Every step of the computation runs in the library's CUDA kernels; there is
no fallback of any kind, and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtg_gemm.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "tg_gemm.h")
HEADERS = [HEADER, os.path.join(os.path.dirname(HERE), "include", "tg_attention.h")]

TG_EPILOGUE_NONE = 0
TG_EPILOGUE_BIAS = 1
TG_EPILOGUE_BIAS_GELU = 2
TG_EPILOGUE_BIAS_GELU_TANH = 3
TG_EPILOGUE_BIAS_SOFTMAX = 4

TG_OK = 0
TG_ERR_INVALID_ARG = 1
TG_ERR_MISALIGNED = 2
TG_ERR_UNSUPPORTED_DEVICE = 3
TG_ERR_LAUNCH = 4
TG_ERR_TIMEOUT = 5
TG_ERR_OOM = 6
TG_ERR_CUDA = 7
TG_ERR_SCRATCH_LIMIT = 8

TG_INJECT_SKIP_FIRST_LOAD = 1
TG_ATTN_SPLIT_AUTO, TG_ATTN_SPLIT_NEVER, TG_ATTN_SPLIT_ALL = 0, 1, 2
TG_INJECT_SKIP_STREAMK_FLAGS = 2
TG_SPLIT_AUTO = 0
TG_SPLIT_TILES = 1
TG_SPLIT_STREAM_K = 2

EPILOGUES = {"none": TG_EPILOGUE_NONE, "bias": TG_EPILOGUE_BIAS, "bias_gelu": TG_EPILOGUE_BIAS_GELU,
             "bias_gelu_tanh": TG_EPILOGUE_BIAS_GELU_TANH, "bias_softmax": TG_EPILOGUE_BIAS_SOFTMAX}


class TgError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {tg_status_string(status)}" if what else tg_status_string(status))


class tg_config_t(ctypes.Structure):
    _fields_ = [("id", ctypes.c_int), ("block_m", ctypes.c_int), ("block_n", ctypes.c_int),
                ("block_k", ctypes.c_int), ("stages", ctypes.c_int), ("cta_pair", ctypes.c_int),
                ("group_m", ctypes.c_int), ("epi_warps", ctypes.c_int), ("split", ctypes.c_int),
                ("loader", ctypes.c_int)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class tg_attention_options_t(ctypes.Structure):
    _fields_ = [("wait_limit_ns", ctypes.c_uint64), ("inject", ctypes.c_int),
                ("kv_split", ctypes.c_int)]


class tg_options_t(ctypes.Structure):
    _fields_ = [("config_id", ctypes.c_int), ("wait_limit_ns", ctypes.c_uint64),
                ("inject", ctypes.c_int), ("group_m", ctypes.c_int), ("split", ctypes.c_int)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libtg_gemm.so not found at {path}; build it with "
                          "`python -m tensor_core_gemm_fp16_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, c_int, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.tg_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int, vp]
    lib.tg_gemm.restype = c_int
    lib.tg_gemm_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int,
                               ctypes.POINTER(tg_options_t), vp]
    lib.tg_gemm_ex.restype = c_int
    lib.tg_gemm_host.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int, vp, sz, vp]
    lib.tg_gemm_host.restype = c_int
    lib.tg_gemm_host_workspace_size.argtypes = [i64, i64, i64, c_int]
    lib.tg_gemm_host_workspace_size.restype = sz
    lib.tg_gemm_check_error.argtypes = [vp]
    lib.tg_gemm_check_error.restype = c_int
    lib.tg_status_string.argtypes = [c_int]
    lib.tg_status_string.restype = ctypes.c_char_p
    lib.tg_num_configs.argtypes = []
    lib.tg_num_configs.restype = c_int
    lib.tg_config_info.argtypes = [c_int, ctypes.POINTER(tg_config_t)]
    lib.tg_config_info.restype = c_int
    lib.tg_gemm_select_config.argtypes = [i64, i64, i64, c_int, c_int, ctypes.POINTER(tg_config_t)]
    lib.tg_gemm_select_config.restype = c_int
    lib.tg_gemm_launch_count.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int]
    lib.tg_gemm_launch_count.restype = c_int
    lib.tg_gemm_noalloc.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int, vp]
    lib.tg_gemm_noalloc.restype = c_int
    lib.tg_version.argtypes = []
    lib.tg_version.restype = c_int
    lib.tg_attention_fwd.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int,
                                     ctypes.c_float, vp]
    lib.tg_attention_fwd.restype = c_int
    lib.tg_attention_fwd_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int,
                                        ctypes.c_float, ctypes.POINTER(tg_attention_options_t), vp]
    lib.tg_attention_fwd_ex.restype = c_int
    i64p = ctypes.POINTER(i64)
    lib.tg_attention_plan.argtypes = [i64, i64, i64, i64, i64, c_int, c_int, c_int, i64p, i64p,
                                      i64p]
    lib.tg_attention_plan.restype = c_int
    _lib = lib
    return lib


def header_symbols(headers=None):
    """Function names declared in the library's headers (include/*.h)."""
    names = set()
    for header in ([headers] if isinstance(headers, str) else (headers or HEADERS)):
        with open(header) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(tg_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


# ---------------------------------------------------------------- raw entry points

def tg_gemm(A: int, B: int, bias: int | None, C: int, M: int, N: int, K: int, epilogue: int,
            stream: int | None = None) -> int:
    return load().tg_gemm(A, B, bias, C, M, N, K, epilogue, stream)


def tg_gemm_noalloc(A: int, B: int, bias: int | None, C: int, M: int, N: int, K: int,
                    epilogue: int, stream: int | None = None) -> int:
    """tg_gemm without any allocation: repacking scratch comes from the
    library's fixed device array (see tg_gemm.h)."""
    return load().tg_gemm_noalloc(A, B, bias, C, M, N, K, epilogue, stream)


def noalloc_scratch_bytes(header: str = HEADER) -> int:
    """TG_NOALLOC_SCRATCH_BYTES as declared in include/tg_gemm.h."""
    m = re.search(r"#define\s+TG_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)",
                  open(header).read())
    return int(m.group(1)) << int(m.group(2))


def tg_gemm_ex(A, B, bias, C, M, N, K, epilogue, config_id=-1, wait_limit_ns=0, inject=0,
               stream=None, group_m=0, split=0) -> int:
    opts = tg_options_t(config_id, wait_limit_ns, inject, group_m, split)
    return load().tg_gemm_ex(A, B, bias, C, M, N, K, epilogue, ctypes.byref(opts), stream)


def tg_gemm_host(A_host, B_host, bias_host, C_host, M, N, K, epilogue, workspace,
                 workspace_bytes, stream=None) -> int:
    return load().tg_gemm_host(A_host, B_host, bias_host, C_host, M, N, K, epilogue, workspace,
                               workspace_bytes, stream)


def tg_gemm_host_workspace_size(M, N, K, has_bias) -> int:
    return load().tg_gemm_host_workspace_size(M, N, K, 1 if has_bias else 0)


def tg_gemm_check_error(stream=None) -> int:
    return load().tg_gemm_check_error(stream)


def tg_status_string(status: int) -> str:
    return load().tg_status_string(status).decode()


def tg_num_configs() -> int:
    return load().tg_num_configs()


def tg_config_info(config_id: int) -> dict:
    c = tg_config_t()
    st = load().tg_config_info(config_id, ctypes.byref(c))
    if st != TG_OK:
        raise TgError(st, "tg_config_info")
    return c.as_dict()


def tg_gemm_select_config(M, N, K, epilogue, num_sms=148) -> dict:
    c = tg_config_t()
    st = load().tg_gemm_select_config(M, N, K, epilogue, num_sms, ctypes.byref(c))
    if st != TG_OK:
        raise TgError(st, "tg_gemm_select_config")
    return c.as_dict()


def tg_gemm_launch_count(A, B, bias, C, M, N, K, epilogue) -> int:
    return load().tg_gemm_launch_count(A, B, bias, C, M, N, K, epilogue)


def tg_version() -> int:
    return load().tg_version()


# ---------------------------------------------------------------- torch conveniences

def _epi(epilogue):
    if isinstance(epilogue, str):
        return EPILOGUES[epilogue]
    return int(epilogue)


def _stream_handle(torch, device):
    return torch.cuda.current_stream(device).cuda_stream


def gemm(a, b, bias=None, epilogue=None, out=None, *, config_id=-1, wait_limit_ns=0, inject=0,
         group_m=0, split=0):
    """C = g(a @ b + bias) on the GPU through tg_gemm_ex.

    a: (M, K) fp16 CUDA, b: (K, N) fp16 CUDA, bias: (N,) fp16 CUDA or None,
    both row-major contiguous.  epilogue defaults to "bias_gelu" when a
    bias is given, else "none".  Returns ``out`` (allocated if None).
    """
    import torch
    if epilogue is None:
        epilogue = TG_EPILOGUE_BIAS_GELU if bias is not None else TG_EPILOGUE_NONE
    epi = _epi(epilogue)
    for name, t in (("a", a), ("b", b), ("bias", bias), ("out", out)):
        if t is None:
            continue
        if t.dtype != torch.float16:
            raise TypeError(f"{name} must be float16, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous (row-major)")
    if a.dim() != 2 or b.dim() != 2 or a.shape[1] != b.shape[0]:
        raise ValueError(f"shape mismatch: a {tuple(a.shape)} @ b {tuple(b.shape)}")
    M, K = a.shape
    N = b.shape[1]
    if bias is not None and tuple(bias.shape) != (N,):
        raise ValueError(f"bias must have shape ({N},)")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    elif tuple(out.shape) != (M, N):
        raise ValueError(f"out must have shape ({M}, {N})")
    with torch.cuda.device(a.device):
        st = tg_gemm_ex(a.data_ptr(), b.data_ptr(), bias.data_ptr() if bias is not None else None,
                        out.data_ptr(), M, N, K, epi, config_id=config_id,
                        wait_limit_ns=wait_limit_ns, inject=inject,
                        stream=_stream_handle(torch, a.device), group_m=group_m, split=split)
    if st != TG_OK:
        raise TgError(st, "tg_gemm")
    return out


def tg_attention_fwd(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim, causal, scale,
                     stream=None) -> int:
    return load().tg_attention_fwd(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim, int(causal),
                                   float(scale), stream)


def tg_attention_plan(batch, heads, seq_q, seq_k, head_dim, causal, kv_split=0,
                      num_sms=148) -> dict:
    """Host-only: units, split units and grid of the launch tg_attention_fwd_ex
    would make (no device needed)."""
    units, split, grid = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    st = load().tg_attention_plan(batch, heads, seq_q, seq_k, head_dim, int(causal), kv_split,
                                  num_sms, ctypes.byref(units), ctypes.byref(split),
                                  ctypes.byref(grid))
    if st != TG_OK:
        raise TgError(st, "tg_attention_plan")
    return {"units": units.value, "split": split.value, "grid": grid.value}


def tg_attention_fwd_ex(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim, causal, scale,
                        wait_limit_ns=0, inject=0, stream=None, kv_split=0) -> int:
    opts = tg_attention_options_t(wait_limit_ns, inject, kv_split)
    return load().tg_attention_fwd_ex(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim,
                                      int(causal), float(scale), ctypes.byref(opts), stream)


def attention(q, k, v, causal=False, scale=0.0, out=None, *, wait_limit_ns=0, inject=0,
              kv_split=0):
    """O = softmax(scale q k^T) v on the GPU through tg_attention_fwd_ex.

    q: (B, H, Sq, D), k and v: (B, H, Sk, D), fp16 contiguous CUDA tensors,
    D in {64, 128}; scale 0 means 1/sqrt(D).  kv_split: TG_ATTN_SPLIT_*.
    Returns ``out`` (allocated if None).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if t is None:
            continue
        if t.dtype != torch.float16:
            raise TypeError(f"{name} must be float16, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or k.shape[:2] != q.shape[:2] \
            or k.shape[3] != q.shape[3]:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, "
                         f"v {tuple(v.shape)}")
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape:
        raise ValueError(f"out must have shape {tuple(q.shape)}")
    with torch.cuda.device(q.device):
        st = tg_attention_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H,
                                 Sq, Sk, D, causal, scale, wait_limit_ns=wait_limit_ns,
                                 inject=inject, stream=_stream_handle(torch, q.device),
                                 kv_split=kv_split)
    if st != TG_OK:
        raise TgError(st, "tg_attention_fwd")
    return out


def gemm_host(a, b, bias=None, epilogue=None, out=None, workspace=None, device=None):
    """End-to-end GEMM on HOST tensors through tg_gemm_host.

    a, b, bias, out are CPU fp16 tensors (pinned for async copies).  The
    device workspace (uint8 CUDA tensor) is allocated when not given.
    Enqueues copies + GEMM + copy-back on the current stream and waits for
    them; returns ``out``.
    """
    import torch
    if epilogue is None:
        epilogue = TG_EPILOGUE_BIAS_GELU if bias is not None else TG_EPILOGUE_NONE
    epi = _epi(epilogue)
    M, K = a.shape
    N = b.shape[1]
    device = torch.device(device or "cuda")
    has_bias = bias is not None and epi != TG_EPILOGUE_NONE
    need = tg_gemm_host_workspace_size(M, N, K, has_bias)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, pin_memory=True)
    with torch.cuda.device(device):
        stream = torch.cuda.current_stream(device)
        st = tg_gemm_host(a.data_ptr(), b.data_ptr(), bias.data_ptr() if has_bias else None,
                          out.data_ptr(), M, N, K, epi, workspace.data_ptr(),
                          workspace.numel(), stream.cuda_stream)
        if st != TG_OK:
            raise TgError(st, "tg_gemm_host")
        stream.synchronize()
    return out
