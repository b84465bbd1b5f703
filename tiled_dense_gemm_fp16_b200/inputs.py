"""Seeded synthetic inputs for C = ReLU(A . B).

This module holds no arithmetic of the method: it only draws operands.  Both
the CUDA path's tests and the oracle's tests take their A and B from here, so
the two sides always see identical fp16 bits.

Recipe (numpy ``default_rng(seed)``; A is drawn first, then B, both in float64
and rounded to fp16 with numpy's ``astype(float16)``, which rounds to nearest
even):
  * ``uniform``  : U[-1, 1]
  * ``normal01`` : N(0, 1) * 0.1
  * ``int``      : integers uniform in {-2, ..., 2}
Shapes of one config that has several problems draw them in order from one
generator, each shape's A then B.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

DISTRIBUTIONS = ("uniform", "normal01", "int")


def draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    """One fp16 operand of ``shape`` from distribution ``dist``."""
    if dist == "uniform":
        return rng.uniform(-1.0, 1.0, size=shape).astype(np.float16)
    if dist == "normal01":
        return (rng.standard_normal(size=shape) * 0.1).astype(np.float16)
    if dist == "int":
        return rng.integers(-2, 3, size=shape).astype(np.float16)
    raise ValueError(f"unknown distribution {dist!r}")


def operands(M: int, N: int, K: int, dist: str = "uniform", seed: int = 0,
             rng: np.random.Generator | None = None):
    """Row-major fp16 A (M x K) and B (K x N)."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    A = draw(rng, (M, K), dist)
    B = draw(rng, (K, N), dist)
    return A, B


def linear_operands(M: int, N: int, K: int, seed: int = 5, dist: str = "uniform"):
    """A linear layer's operands: x (M x K), the weight W stored N x K, and a bias of N values.

    Drawn in that order from ``default_rng(seed)``.
    """
    rng = np.random.default_rng(seed)
    x = draw(rng, (M, K), dist)
    W = draw(rng, (N, K), dist)
    b = draw(rng, (N,), dist)
    return x, W, b


@dataclass(frozen=True)
class Workload:
    name: str
    shapes: tuple          # ((M, N, K), ...)
    dist: str
    seed: int
    note: str = ""

    def problems(self, dist: str | None = None):
        """Yield (shape, A, B) for every shape, drawing in order from one generator."""
        rng = np.random.default_rng(self.seed)
        for (M, N, K) in self.shapes:
            A, B = operands(M, N, K, dist or self.dist, rng=rng)
            yield (M, N, K), A, B


# The five workloads the method is measured on: sizes, value distributions and
# seeds.  "square256" also has an integer-valued variant for bit-exact checks.
WORKLOADS = {
    "square256": Workload("square256", ((256, 256, 256),), "uniform", 0,
                          "small square; integer variant draws {-2..2} from the same seed"),
    "square4096": Workload("square4096", ((4096, 4096, 4096),), "normal01", 1,
                           "large square, N(0,1)*0.1"),
    "square8192": Workload("square8192", ((8192, 8192, 8192),), "uniform", 2,
                           "large square, compute-bound"),
    "skinny": Workload("skinny", ((1, 8192, 8192), (16, 8192, 8192), (64, 8192, 8192)),
                       "uniform", 3, "decode-like small M, bandwidth-bound"),
    "ragged": Workload("ragged", ((3001, 5003, 1021), (777, 12289, 4095), (8191, 129, 8193)),
                       "uniform", 4, "non-tile-multiple shapes with unaligned row strides"),
    # Beyond the five: a linear layer relu(x W^T + b) with the weight stored N x K.
    "linear8192": Workload("linear8192", ((8192, 8192, 8192),), "uniform", 5,
                           "x (M x K), weight stored N x K, fp16 bias; drawn by linear_operands"),
}


def flops(M: int, N: int, K: int) -> int:
    """Algorithmic flop count of one GEMM: one multiply and one add per (i, j, k)."""
    return 2 * M * N * K


def min_bytes(M: int, N: int, K: int) -> int:
    """Compulsory HBM bytes of one GEMM: read A and B once, write C once (fp16)."""
    return 2 * (M * K + K * N + M * N)
