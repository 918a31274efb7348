"""Seeded synthetic inputs for the fp16 GEMM workloads.

This module only draws random numbers and packs them as fp16; it holds none
of the GEMM or epilogue arithmetic.  Both the CUDA path and the CPU oracle
are fed from it, so they always see the same fp16 bytes.

Recipe (the tutorial seeds nothing and draws with ``torch.randn`` on the
device; here the draws are on the host so that they are reproducible):

* ``g = torch.Generator().manual_seed(seed)``; then A, then B, then bias are
  drawn in that order as float32 and rounded to fp16 (round to nearest even).
* ``normal``: i.i.d. N(0, 1).  ``uniform``: i.i.d. U(-1, 1) = 2 * rand - 1.
* ``b_scale``/``a_scale`` multiply the float32 draw before rounding (the
  8192^3 workload keeps the GEMM output O(1) by scaling B by 1/sqrt(K)).

Shapes follow the tutorial: the square 2048^3 tensor-core GEMM of its
memory-hierarchy and schedule-sweep sections, plus a small, a ragged and a
large fused case.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

EPI_NONE = 0
EPI_BIAS = 1
EPI_BIAS_GELU = 2
EPI_BIAS_GELU_TANH = 3
EPI_BIAS_SOFTMAX = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    epilogue: int
    dist: str          # "normal" or "uniform"
    seed: int
    a_scale: float = 1.0
    b_scale: float = 1.0
    has_bias: bool = False

    @property
    def flops(self) -> int:
        """2*M*N*K: the tutorial's GEMM flop count (epilogue flops not counted)."""
        return 2 * self.M * self.N * self.K

    @property
    def algorithmic_bytes(self) -> int:
        """Bytes a perfect kernel moves: read A, B (and bias) once, write C once."""
        b = 2 * (self.M * self.K + self.K * self.N + self.M * self.N)
        return b + (2 * self.N if self.has_bias else 0)


WORKLOADS = {
    "gemm_256": Workload("gemm_256", 256, 256, 256, EPI_NONE, "normal", 0),
    "gemm_2048": Workload("gemm_2048", 2048, 2048, 2048, EPI_NONE, "normal", 1),
    "fused_2048": Workload("fused_2048", 2048, 2048, 2048, EPI_BIAS_GELU, "normal", 2,
                           has_bias=True),
    "ragged_fused": Workload("ragged_fused", 3000, 1537, 2050, EPI_BIAS_GELU, "uniform", 3,
                             has_bias=True),
    "fused_8192": Workload("fused_8192", 8192, 8192, 8192, EPI_BIAS_GELU, "normal", 4,
                           b_scale=1.0 / math.sqrt(8192), has_bias=True),
    # The epilogue variants: the tanh form of GELU on the square shape, and a
    # row softmax over 256 columns (scores of 8192 queries against 256 keys
    # with a 4096-wide contraction, B scaled by 1/sqrt(K)).
    "fused_tanh_2048": Workload("fused_tanh_2048", 2048, 2048, 2048, EPI_BIAS_GELU_TANH, "normal",
                                5, has_bias=True),
    "softmax_8192x256x4096": Workload("softmax_8192x256x4096", 8192, 256, 4096, EPI_BIAS_SOFTMAX,
                                      "normal", 6, b_scale=1.0 / math.sqrt(4096), has_bias=True),
    # Deep contractions with few output tiles: fewer tiles than SMs, so the
    # work is divided along K as well (stream-K).  B scaled by 1/sqrt(K).
    "deepk_fused_1024x1024x8192": Workload("deepk_fused_1024x1024x8192", 1024, 1024, 8192,
                                           EPI_BIAS_GELU, "normal", 7,
                                           b_scale=1.0 / math.sqrt(8192), has_bias=True),
    "deepk_512x512x16384": Workload("deepk_512x512x16384", 512, 512, 16384, EPI_NONE, "normal", 8,
                                    b_scale=1.0 / math.sqrt(16384)),
    # The same shape with both operands scaled by 1/sqrt(K) (the literal wording
    # of the large-workload description); parity only.
    "fused_8192_literal": Workload("fused_8192_literal", 8192, 8192, 8192, EPI_BIAS_GELU,
                                   "normal", 4, a_scale=1.0 / math.sqrt(8192),
                                   b_scale=1.0 / math.sqrt(8192), has_bias=True),
}


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """Attention forward: Q [B, H, Sq, D], K and V [B, H, Sk, D], fp16, row-major."""
    name: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    causal: bool
    seed: int

    @property
    def visible_pairs(self) -> int:
        """(query, key) pairs the softmax sees: Sq*Sk, or the lower triangle."""
        if not self.causal:
            return self.Sq * self.Sk
        return sum(min(i + 1, self.Sk) for i in range(self.Sq))

    @property
    def flops(self) -> int:
        """4*D per visible (query, key) pair and head: Q.K^T and P.V, 2 flops per MAC."""
        return 4 * self.D * self.B * self.H * self.visible_pairs

    @property
    def algorithmic_bytes(self) -> int:
        """Read Q, K, V once and write O once (fp16)."""
        return 2 * self.B * self.H * self.D * (2 * self.Sq + 2 * self.Sk)


# Attention shapes: head width 64 and 128, a sequence of 2048 with 16 heads
# and batch 4 (the common forward-pass benchmark size), causal and not, and
# small ragged cases for parity.
ATTN_WORKLOADS = {
    "attn_4x16x2048x128": AttnWorkload("attn_4x16x2048x128", 4, 16, 2048, 2048, 128, False, 20),
    "attn_causal_4x16x2048x128": AttnWorkload("attn_causal_4x16x2048x128", 4, 16, 2048, 2048,
                                              128, True, 21),
    "attn_4x16x2048x64": AttnWorkload("attn_4x16x2048x64", 4, 16, 2048, 2048, 64, False, 22),
    "attn_ragged_2x3x333x64": AttnWorkload("attn_ragged_2x3x333x64", 2, 3, 333, 333, 64, True, 23),
}


def attention_inputs(B: int, H: int, Sq: int, Sk: int, D: int, seed: int, dist: str = "normal"):
    """Return (Q, K, V) as CPU fp16 tensors, drawn in that order from one generator."""
    g = torch.Generator().manual_seed(seed)
    Q = _draw(g, (B, H, Sq, D), dist, 1.0)
    K = _draw(g, (B, H, Sk, D), dist, 1.0)
    V = _draw(g, (B, H, Sk, D), dist, 1.0)
    return Q, K, V


def attn_workload_inputs(w: AttnWorkload):
    return attention_inputs(w.B, w.H, w.Sq, w.Sk, w.D, w.seed)


def _draw(g: torch.Generator, shape, dist: str, scale: float) -> torch.Tensor:
    if dist == "normal":
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
    elif dist == "uniform":
        x = torch.rand(*shape, generator=g, dtype=torch.float32) * 2.0 - 1.0
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    if scale != 1.0:
        x = x * scale
    return x.to(torch.float16)


def make_inputs(M: int, N: int, K: int, seed: int, dist: str = "normal", *,
                bias: bool = False, a_scale: float = 1.0, b_scale: float = 1.0):
    """Return (A[M,K], B[K,N], bias[N] or None) as CPU fp16 torch tensors."""
    g = torch.Generator().manual_seed(seed)
    A = _draw(g, (M, K), dist, a_scale)
    B = _draw(g, (K, N), dist, b_scale)
    b = _draw(g, (N,), dist, 1.0) if bias else None
    return A, B, b


def workload_inputs(w: Workload):
    """Inputs of a named workload, in the recipe's draw order."""
    return make_inputs(w.M, w.N, w.K, w.seed, w.dist, bias=w.has_bias,
                       a_scale=w.a_scale, b_scale=w.b_scale)


def integer_inputs(M: int, N: int, K: int, seed: int, lo: int = -1, hi: int = 1,
                   bias: bool = False):
    """Integer-valued fp16 inputs drawn uniformly from {lo, ..., hi}."""
    g = torch.Generator().manual_seed(seed)
    A = torch.randint(lo, hi + 1, (M, K), generator=g).to(torch.float16)
    B = torch.randint(lo, hi + 1, (K, N), generator=g).to(torch.float16)
    b = torch.randint(lo, hi + 1, (N,), generator=g).to(torch.float16) if bias else None
    return A, B, b


def permutation(n: int, seed: int) -> np.ndarray:
    """A seeded random permutation of range(n)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(n, generator=g).numpy()


def to_bits(t: torch.Tensor | None) -> np.ndarray | None:
    """CPU fp16 tensor -> numpy uint16 bit patterns (no copy of the values' meaning)."""
    if t is None:
        return None
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
