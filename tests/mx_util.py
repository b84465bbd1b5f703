"""Helpers for the MXFP8 grouped GEMM tests: the 128 x 4 blocked scale layout
of the C ABI, and the oracle on a sample of rows."""
import numpy as np

import oracle
from tiled_dense_gemm_fp16_b200.inputs import mx_scales_blocked

to_blocked = mx_scales_blocked
to_blocked_groups = mx_scales_blocked


def oracle_rows(A, SFA, B, SFB, g, rows, N, K, a_format, b_format, relu):
    """Oracle output (bf16 bits) of stacked rows ``rows`` of group g."""
    rows = np.asarray(rows, np.int64)
    return oracle.gemm_mxf8_grouped(np.ascontiguousarray(A[rows]), np.ascontiguousarray(SFA[rows]), B[g:g + 1],
                                    SFB[g:g + 1], [len(rows)], [0], N, K, a_format, b_format, relu=relu)


def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def abs_dot(A, SFA, B, SFB, g, rows, N, K, a_format, b_format):
    """sum_k |a(r,k) sa| |b_g(j,k) sb| for the given rows, from the oracle's own decoders
    (a bound for the accumulation error, not a reference value)."""
    dec_a = oracle.fp8_to_f64(np.arange(256, dtype=np.uint8), a_format)
    dec_b = oracle.fp8_to_f64(np.arange(256, dtype=np.uint8), b_format)
    sc = oracle.ue8m0_to_f64(np.arange(256, dtype=np.uint8))
    rows = np.asarray(rows, np.int64)
    av = np.abs(dec_a[A[rows]] * np.repeat(sc[SFA[rows]], 32, axis=1))
    bv = np.abs(dec_b[B[g]] * np.repeat(sc[SFB[g]], 32, axis=1))
    return av @ bv.T


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """Bytes (..., K/2) -> 4-bit codes (..., K), element 2i from the low nibble."""
    packed = np.asarray(packed, np.uint8)
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def nvf4_oracle_rows(A, SFA, B, SFB, g, rows, N, K, alpha, relu):
    rows = np.asarray(rows, np.int64)
    return oracle.gemm_nvf4_grouped(np.ascontiguousarray(A[rows]), np.ascontiguousarray(SFA[rows]), B[g:g + 1],
                                    SFB[g:g + 1], [len(rows)], [0], N, K, alpha=alpha, relu=relu)


def nvf4_abs_dot(A, SFA, B, SFB, g, rows, N, K):
    dec = oracle.e2m1_to_f64(np.arange(16, dtype=np.uint8))
    sc = oracle.ue4m3_to_f64(np.arange(128, dtype=np.uint8))
    rows = np.asarray(rows, np.int64)
    av = np.abs(dec[unpack_fp4(A[rows])] * np.repeat(sc[SFA[rows]], 16, axis=1))
    bv = np.abs(dec[unpack_fp4(B[g])] * np.repeat(sc[SFB[g]], 16, axis=1))
    return av @ bv.T
