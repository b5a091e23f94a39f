"""Seeded synthetic operands for the fp16 GEMM (+bias+ReLU) workloads.

This module only draws inputs. It holds none of the GEMM arithmetic, so both
sides of a parity check (the CUDA library and the CPU oracle) can take their
operands from here without sharing any of the computation.

The operands follow the shapes and value distributions of the five workloads
the pages' GEMM is exercised on (page 1 "4.2" runs an fp16-in / fp32-accumulate
GEMM on random fp16 inputs; page 3 "3.3" times a 1024x1024 matmul; page 4
"4.2" adds a per-column bias and a ReLU):

* ``A`` and ``B`` are drawn with a torch CPU generator seeded with ``seed``,
  A first, then B, then the bias, and every draw is cast to fp16.
* uniform workloads: ``rand * 2 - 1`` (entries in [-1, 1]);
  the ragged workload: ``randn * 0.25``; the bias: ``rand - 0.5``.
* sampled output positions (for shapes whose full CPU reference is too slow)
  come from a second generator seeded with ``seed + 1``.
* the residual of the general fused epilogue (page 4 "4.1": activation and
  residual connection fused into the GEMM) comes from a third generator seeded
  with ``seed + 2``: ``rand * 2 - 1`` cast to the output's type.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    dist: str  # "uniform" (U[-1,1]) or "normal025" (N(0,1)*0.25)
    out: str  # "f32" or "f16"
    bias_relu: bool
    sample: Optional[int] = None  # number of sampled output positions checked, None = all
    # General fused epilogue C = act(A.B + bias) + R: the activation ("none",
    # "relu" or "gelu"; None = not this epilogue), always with a bias, and
    # whether a residual R in C's type is added.
    act: Optional[str] = None
    residual: bool = False

    @property
    def has_bias(self) -> bool:
        return self.bias_relu or self.act is not None

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def out_bytes(self) -> int:
        return 4 if self.out == "f32" else 2

    @property
    def algorithmic_bytes(self) -> int:
        """Compulsory HBM bytes: A and B read once, C written once, bias and residual read once."""
        b = 2 * self.M * self.K + 2 * self.K * self.N + self.out_bytes * self.M * self.N
        if self.has_bias:
            b += 2 * self.N
        if self.residual:
            b += self.out_bytes * self.M * self.N
        return b


# The five workloads, in the order they are listed for this path.
WORKLOADS = {
    w.name: w
    for w in (
        Workload("gemm_256_f32", 256, 256, 256, "uniform", "f32", False),
        Workload("gemm_1024_f32", 1024, 1024, 1024, "uniform", "f32", False),
        Workload("gemm_bias_relu_4096_f16", 4096, 4096, 4096, "uniform", "f16", True),
        Workload("gemm_ragged_4000x3000x1000_f32", 4000, 3000, 1000, "normal025", "f32", False),
        Workload("gemm_8192_f16", 8192, 8192, 8192, "uniform", "f16", False, sample=4096),
    )
}
WORKLOAD_ORDER = list(WORKLOADS)

# Fused-epilogue workloads beyond the five: bias + GELU + residual connection
# at the bias+ReLU workload's size (a separate fp16 residual R, read once).
EPILOGUE_WORKLOADS = {
    w.name: w
    for w in (
        Workload("gemm_bias_gelu_residual_4096_f16", 4096, 4096, 4096, "uniform", "f16", False,
                 sample=4096, act="gelu", residual=True),
    )
}


def _draw(shape, dist: str, g: torch.Generator) -> torch.Tensor:
    if dist == "uniform":
        x = torch.rand(shape, generator=g, dtype=torch.float32) * 2.0 - 1.0
    elif dist == "normal025":
        x = torch.randn(shape, generator=g, dtype=torch.float32) * 0.25
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return x.to(torch.float16)


def make_operands(M: int, N: int, K: int, dist: str = "uniform", bias: bool = False, seed: int = 0):
    """Return CPU fp16 tensors ``(A[M,K], B[K,N], bias[N] or None)``, row-major and contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    A = _draw((M, K), dist, g)
    B = _draw((K, N), dist, g)
    b = None
    if bias:
        b = (torch.rand((N,), generator=g, dtype=torch.float32) - 0.5).to(torch.float16)
    return A, B, b


def workload_operands(w: Workload, seed: int = 0):
    return make_operands(w.M, w.N, w.K, w.dist, w.has_bias, seed)


def make_residual(M: int, N: int, out: str = "f16", seed: int = 0) -> torch.Tensor:
    """A CPU residual ``R[M,N]`` in the output's type (``out`` "f16" or "f32"), entries in [-1, 1]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 2)
    x = torch.rand((M, N), generator=g, dtype=torch.float32) * 2.0 - 1.0
    return x.to(torch.float16 if out == "f16" else torch.float32)


def sample_positions(M: int, N: int, count: int, seed: int = 1):
    """``count`` output positions (row, col), drawn with replacement over the M*N grid."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    flat = torch.randint(0, M * N, (count,), generator=g, dtype=torch.int64)
    return flat // N, flat % N


def integer_operands(M: int, N: int, K: int, lo: int = -2, hi: int = 2, seed: int = 0, bias: bool = False):
    """Small-integer fp16 operands (entries in [lo, hi]); every partial sum is exact in fp32
    as long as K * max|a| * max|b| stays below 2**24."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    A = torch.randint(lo, hi + 1, (M, K), generator=g).to(torch.float16)
    B = torch.randint(lo, hi + 1, (K, N), generator=g).to(torch.float16)
    b = torch.randint(lo, hi + 1, (N,), generator=g).to(torch.float16) if bias else None
    return A, B, b
