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


# E4M3 codes of the integers -2..2 (values exact in every fp8 format step used here).
_E4M3_INT_CODES = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)
_E5M2_INT_CODES = np.array([0xC0, 0xBC, 0x00, 0x3C, 0x40], np.uint8)


def mx_group_offsets(m_sizes):
    """First stacked row of each group: groups start on multiples of 128 rows."""
    offs, r = [], 0
    for m in m_sizes:
        offs.append(r)
        r += (int(m) + 127) // 128 * 128
    return np.array(offs, np.int64), r


def _fp8_codes(values: np.ndarray, fmt: int) -> np.ndarray:
    import torch
    dt = torch.float8_e4m3fn if fmt == 0 else torch.float8_e5m2
    return torch.from_numpy(np.ascontiguousarray(values, np.float32)).to(dt).view(torch.uint8).numpy()


def mx_operands(m_sizes, N: int, K: int, seed: int, dist: str = "normal", a_format: int = 0, b_format: int = 0,
                scale_lo: int = 124, scale_hi: int = 131):
    """Grouped MXFP8 operands: A codes (stacked rows x K, padding rows drawn too), plain row-major
    scales SFA (rows x K/32), B codes (G x N x K) and SFB (G x N x K/32), in that order from
    ``default_rng(seed)``.

    ``dist``: "int" draws the integers -2..2 with unit scales (code 127); "normal" draws N(0,1)
    values rounded to the format by torch (nearest even, saturating formats clamp) and scales
    uniform in [scale_lo, scale_hi).
    """
    rng = np.random.default_rng(seed)
    G = len(m_sizes)
    _, rows = mx_group_offsets(m_sizes)
    S = K // 32
    if dist == "int":
        ta = _E4M3_INT_CODES if a_format == 0 else _E5M2_INT_CODES
        tb = _E4M3_INT_CODES if b_format == 0 else _E5M2_INT_CODES
        A = ta[rng.integers(0, 5, size=(rows, K))]
        SFA = np.full((rows, S), 127, np.uint8)
        B = tb[rng.integers(0, 5, size=(G, N, K))]
        SFB = np.full((G, N, S), 127, np.uint8)
        return A, SFA, B, SFB
    if dist != "normal":
        raise ValueError(f"unknown distribution {dist!r}")
    A = _fp8_codes(rng.standard_normal(size=(rows, K)), a_format)
    SFA = rng.integers(scale_lo, scale_hi, size=(rows, S)).astype(np.uint8)
    B = _fp8_codes(rng.standard_normal(size=(G, N, K)), b_format)
    SFB = rng.integers(scale_lo, scale_hi, size=(G, N, S)).astype(np.uint8)
    return A, SFA, B, SFB


# E2M1 codes of the integers -4..4 that the format holds (0, +-1, +-2, +-3, +-4).
_E2M1_INT_CODES = np.array([0xE, 0xD, 0xC, 0xA, 0x0, 0x2, 0x4, 0x5, 0x6], np.uint8)


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """4-bit codes (..., K) -> bytes (..., K/2), element 2i in the low nibble."""
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def nvf4_operands(m_sizes, N: int, K: int, seed: int, dist: str = "codes", scale_lo: int = 0x28,
                  scale_hi: int = 0x49):
    """Grouped NVF4 operands: packed A (stacked rows x K/2), plain scales SFA (rows x K/16), packed B
    (G x N x K/2) and SFB (G x N x K/16), drawn in that order from ``default_rng(seed)``.

    ``dist``: "int" draws the E2M1 integers -4..4 with unit scales (UE4M3 code 0x38 = 1.0);
    "codes" draws every E2M1 code uniformly and scale codes uniform in [scale_lo, scale_hi)
    (0x28..0x48: 2^-2 .. 2^2 with all mantissas).
    """
    rng = np.random.default_rng(seed)
    G = len(m_sizes)
    _, rows = mx_group_offsets(m_sizes)
    S = K // 16
    if dist == "int":
        A = _E2M1_INT_CODES[rng.integers(0, 9, size=(rows, K))]
        SFA = np.full((rows, S), 0x38, np.uint8)
        B = _E2M1_INT_CODES[rng.integers(0, 9, size=(G, N, K))]
        SFB = np.full((G, N, S), 0x38, np.uint8)
    elif dist == "codes":
        A = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
        SFA = rng.integers(scale_lo, scale_hi, size=(rows, S)).astype(np.uint8)
        B = rng.integers(0, 16, size=(G, N, K)).astype(np.uint8)
        SFB = rng.integers(scale_lo, scale_hi, size=(G, N, S)).astype(np.uint8)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return pack_fp4(A), SFA, pack_fp4(B), SFB


def w4_operands(M: int, N: int, K: int, group: int, seed: int, dist: str = "uniform"):
    """4-bit weight-only operands, drawn in this order from ``default_rng(seed)``: A (M x K fp16),
    the weight's codes (N x K, 0..15) packed two per byte (N x K/2), and fp16 scales (N x K/group).

    ``dist``: "int" draws A from the integers -2..2 and scales from {0.5, 1, 2} (every product
    and sum exact); "uniform" draws A from U[-1,1] and scales from U[0.002, 0.02] (the magnitude of
    a trained layer's weight step).
    """
    rng = np.random.default_rng(seed)
    if dist == "int":
        A = rng.integers(-2, 3, size=(M, K)).astype(np.float16)
    elif dist == "uniform":
        A = rng.uniform(-1.0, 1.0, size=(M, K)).astype(np.float16)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    if dist == "int":
        S = np.array([0.5, 1.0, 2.0], np.float16)[rng.integers(0, 3, size=(N, K // group))]
    else:
        S = rng.uniform(0.002, 0.02, size=(N, K // group)).astype(np.float16)
    return A, pack_fp4(codes), S


def mx_scales_blocked(sf: np.ndarray) -> np.ndarray:
    """Plain row-major scales (R x S) rearranged into the C ABI's 128 x 4 blocked byte layout:
    scale (r, s) goes to ((r//128)*(S'/4) + s//4)*512 + (r%32)*16 + ((r//32)%4)*4 + s%4, with
    S' = roundup(S, 4); padding bytes are 0.  A G x N x S array gives G blocked arrays back to back."""
    if sf.ndim == 3:
        parts = [mx_scales_blocked(sf[g]) for g in range(sf.shape[0])]
        return np.concatenate(parts) if parts else np.zeros(0, np.uint8)
    R, S = sf.shape
    Rp, Sp = (R + 127) // 128 * 128, (S + 3) // 4 * 4
    out = np.zeros(Rp * Sp, np.uint8)
    r = np.arange(R)[:, None]
    s = np.arange(S)[None, :]
    out[((r // 128) * (Sp // 4) + s // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + s % 4] = sf
    return out


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

# MXFP8 grouped workloads: (group sizes, N, K, seed).  "mxf8_moe" is a mixture-of-experts
# layer shape: 8 experts with ragged token counts (16384 tokens in all), N = 4096, K = 7168.
MX_WORKLOADS = {
    "mxf8_moe": ((2304, 1792, 2048, 2560, 1536, 2048, 2176, 1920), 4096, 7168, 6),
    "mxf8_8192": ((8192,), 8192, 8192, 7),
}

# 4-bit weight-only workloads: (M, N, K, group, seed).  "w4a16_decode" is a decode step of a
# 8192-wide layer (16 tokens), bound by streaming the packed weight; "w4a16_8192" is the
# large-M case (dequantize, then the fp16 tensor-core GEMM).
W4_WORKLOADS = {
    "w4a16_decode": (16, 8192, 8192, 128, 10),
    "w4a16_8192": (8192, 8192, 8192, 128, 11),
}

# NVF4 workloads: the 8192^3 problem the NVF4 path is quoted on, and the MoE layer shape.
NVF4_WORKLOADS = {
    "nvf4_8192": ((8192,), 8192, 8192, 8),
    "nvf4_moe": ((2304, 1792, 2048, 2560, 1536, 2048, 2176, 1920), 4096, 7168, 9),
}


def flops(M: int, N: int, K: int) -> int:
    """Algorithmic flop count of one GEMM: one multiply and one add per (i, j, k)."""
    return 2 * M * N * K


def min_bytes(M: int, N: int, K: int) -> int:
    """Compulsory HBM bytes of one GEMM: read A and B once, write C once (fp16)."""
    return 2 * (M * K + K * N + M * N)
