"""CPU oracle for C = ReLU(A . B) (fp16 in, fp32 accumulate, fp16 out).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg import this package.  The product library never loads it and
has no fallback to it.  It shares no code with the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, compiled with gcc at -O2 and
no fast-math, fp contraction off).  This module only builds that file and
marshals numpy arrays through ctypes.

What it follows: the quick-start ``matmul_relu`` kernel on the "TileLang"
wiki page, section "Programming model": fp16 A (M x K) and B (K x N), an fp32
accumulator cleared to zero, a K loop of tile products, ``max(C_local, 0)`` on
the fp32 values and a copy into the fp16 output C (M x N).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

_lib = None
_lock = threading.Lock()

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
          "-shared", "-std=c11", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``_build/liboracle.so`` (if stale) and return its path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile an alternative oracle source (used by the pin-strength tests)."""
    src_path = out_path + ".c"
    with open(src_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *CFLAGS, src_path, "-o", out_path, "-lm"], check=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(lib):
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f32p = ctypes.POINTER(ctypes.c_float)
    i64 = ctypes.c_int64
    lib.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_f16_rne.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_f16_rne.restype = ctypes.c_uint16
    lib.oracle_f16_to_f32_array.argtypes = [u16p, f32p, i64]
    lib.oracle_f16_to_f32_array.restype = None
    lib.oracle_f32_to_f16_rne_array.argtypes = [f32p, u16p, i64]
    lib.oracle_f32_to_f16_rne_array.restype = None
    lib.oracle_gemm_relu_f16.argtypes = [u16p, u16p, u16p, i64, i64, i64, ctypes.c_int]
    lib.oracle_gemm_relu_f16.restype = ctypes.c_int
    lib.oracle_gemm_relu_f16_ex.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, i64, ctypes.c_int,
                                            ctypes.c_int, u16p, ctypes.c_int]
    lib.oracle_gemm_relu_f16_ex.restype = ctypes.c_int
    u8p = ctypes.POINTER(ctypes.c_uint8)
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_fp8_to_f64.argtypes = [ctypes.c_uint8, ctypes.c_int]
    lib.oracle_fp8_to_f64.restype = ctypes.c_double
    lib.oracle_ue8m0_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_ue8m0_to_f64.restype = ctypes.c_double
    lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
    lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
    lib.oracle_gemm_mxf8_grouped.argtypes = [u8p, u8p, u8p, u8p, u16p, i64p, i64p, ctypes.c_int, i64, i64,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.oracle_gemm_mxf8_grouped.restype = ctypes.c_int
    lib.oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_to_f64.restype = ctypes.c_double
    lib.oracle_ue4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_ue4m3_to_f64.restype = ctypes.c_double
    lib.oracle_gemm_nvf4_grouped.argtypes = [u8p, u8p, u8p, u8p, u16p, i64p, i64p, ctypes.c_int, i64, i64,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_int]
    lib.oracle_gemm_nvf4_grouped.restype = ctypes.c_int
    lib.oracle_dequant_w4_f16.argtypes = [u8p, u16p, u16p, i64, i64, i64]
    lib.oracle_dequant_w4_f16.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def load_library(path: str | None = None):
    """Load (building first if needed) the oracle library; ``path`` loads a variant."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _u16(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16 or uint16 bit patterns, got {a.dtype}")
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def f16_bits_to_f32(h: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load_library()
    h = _u16(np.asarray(h))
    out = np.empty(h.shape, dtype=np.float32)
    lib.oracle_f16_to_f32_array(_ptr(h, ctypes.c_uint16), _ptr(out, ctypes.c_float), h.size)
    return out


def f32_to_f16_bits(x: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load_library()
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint16)
    lib.oracle_f32_to_f16_rne_array(_ptr(x, ctypes.c_float), _ptr(out, ctypes.c_uint16), x.size)
    return out


def gemm_relu_f16(A: np.ndarray, B: np.ndarray, nthreads: int = 0, lib=None) -> np.ndarray:
    """C = f16_rne(relu(A . B)) with sequential fp32 accumulation; returns float16 (M, N)."""
    lib = lib or load_library()
    A = _u16(np.asarray(A))
    B = _u16(np.asarray(B))
    if A.ndim != 2 or B.ndim != 2 or A.shape[1] != B.shape[0]:
        raise ValueError(f"shape mismatch: A{A.shape} B{B.shape}")
    M, K = A.shape
    N = B.shape[1]
    C = np.empty((M, N), dtype=np.uint16)
    rc = lib.oracle_gemm_relu_f16(_ptr(A, ctypes.c_uint16), _ptr(B, ctypes.c_uint16),
                                  _ptr(C, ctypes.c_uint16), M, N, K, int(nthreads))
    if rc != 0:
        raise MemoryError("oracle could not allocate its work buffers")
    return C.view(np.float16)


def gemm_relu_f16_ex(A: np.ndarray, B: np.ndarray, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
                     b_nk: bool = False, bias: np.ndarray | None = None, C: np.ndarray | None = None,
                     nthreads: int = 0, lib=None, a_km: bool = False) -> np.ndarray:
    """General-layout form: A, B and C are flat fp16 buffers read/written with the given row strides.

    A holds M x K (a_km False) or K x M (a_km True) with row stride lda; B holds K x N (b_nk False)
    or N x K (b_nk True) with row stride ldb; ``bias`` is an fp16 vector of N or None.  Returns C (a
    fresh zero buffer of M*ldc elements unless one is given; only the M x N block is written).
    """
    lib = lib or load_library()
    A = _u16(np.asarray(A).reshape(-1))
    B = _u16(np.asarray(B).reshape(-1))
    if C is None:
        C = np.zeros(max(M * ldc, 1), dtype=np.uint16)
    else:
        C = _u16(np.asarray(C).reshape(-1)).copy()
    bias_p = None
    if bias is not None:
        bias = _u16(np.asarray(bias).reshape(-1))
        if bias.size < N:
            raise ValueError("bias must have N elements")
        bias_p = _ptr(bias, ctypes.c_uint16)
    need_a = ((K - 1) * lda + M if a_km else (M - 1) * lda + K) if M > 0 and K > 0 else 0
    need_b = ((K - 1) * ldb + N if not b_nk else (N - 1) * ldb + K) if K > 0 and N > 0 else 0
    if A.size < need_a or B.size < need_b or C.size < (M - 1) * ldc + N:
        raise ValueError("buffer too small for the given shape and strides")
    rc = lib.oracle_gemm_relu_f16_ex(_ptr(A, ctypes.c_uint16), _ptr(B, ctypes.c_uint16), _ptr(C, ctypes.c_uint16),
                                     M, N, K, lda, ldb, ldc, 1 if a_km else 0, 1 if b_nk else 0, bias_p,
                                     int(nthreads))
    if rc != 0:
        raise MemoryError("oracle could not allocate its work buffers")
    return C.view(np.float16)


def gemm_relu_f16_rows(A: np.ndarray, B: np.ndarray, rows, nthreads: int = 0, lib=None) -> np.ndarray:
    """Rows ``rows`` of the oracle result: the same definition applied to A[rows, :]."""
    rows = np.asarray(rows, dtype=np.int64)
    return gemm_relu_f16(np.ascontiguousarray(A[rows, :]), B, nthreads=nthreads, lib=lib)


E4M3, E5M2 = 0, 1


def fp8_to_f64(codes, fmt: int, lib=None) -> np.ndarray:
    """Values of FP8 codes (format E4M3 = 0 or E5M2 = 1)."""
    lib = lib or load_library()
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    return np.array([lib.oracle_fp8_to_f64(int(c), fmt) for c in codes], dtype=np.float64)


def ue8m0_to_f64(codes, lib=None) -> np.ndarray:
    lib = lib or load_library()
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    return np.array([lib.oracle_ue8m0_to_f64(int(c)) for c in codes], dtype=np.float64)


def f64_to_bf16_bits(x, lib=None) -> np.ndarray:
    lib = lib or load_library()
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    return np.array([lib.oracle_f64_to_bf16_rne(float(v)) for v in x], dtype=np.uint16)


def gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, row_offsets, N: int, K: int, a_format: int = E4M3,
                      b_format: int = E4M3, relu: bool = False, C=None, nthreads: int = 0, lib=None) -> np.ndarray:
    """Grouped MXFP8 GEMM: A (rows x K codes), SFA (rows x K/32 UE8M0), B (G x N x K codes),
    SFB (G x N x K/32); group g covers rows row_offsets[g] .. + m_sizes[g].  Returns bf16 bit patterns
    (rows x N, uint16); rows outside every group keep C's initial contents (zero by default)."""
    lib = lib or load_library()
    A = np.ascontiguousarray(np.asarray(A, dtype=np.uint8))
    SFA = np.ascontiguousarray(np.asarray(SFA, dtype=np.uint8))
    B = np.ascontiguousarray(np.asarray(B, dtype=np.uint8))
    SFB = np.ascontiguousarray(np.asarray(SFB, dtype=np.uint8))
    m_sizes = np.ascontiguousarray(np.asarray(m_sizes, dtype=np.int64))
    row_offsets = np.ascontiguousarray(np.asarray(row_offsets, dtype=np.int64))
    G = int(m_sizes.size)
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    rows = A.size // K if K else 0
    if row_offsets.size != G or (G and int((row_offsets + m_sizes).max()) > rows):
        raise ValueError("groups do not fit in A")
    if B.size < G * N * K or SFB.size < G * N * (K // 32) or SFA.size < rows * (K // 32):
        raise ValueError("operand too small")
    C = np.zeros(rows * N, np.uint16) if C is None else np.ascontiguousarray(np.asarray(C, np.uint16)).reshape(-1).copy()
    rc = lib.oracle_gemm_mxf8_grouped(_ptr(A, ctypes.c_uint8), _ptr(SFA, ctypes.c_uint8), _ptr(B, ctypes.c_uint8),
                                      _ptr(SFB, ctypes.c_uint8), _ptr(C, ctypes.c_uint16), _ptr(row_offsets, ctypes.c_int64),
                                      _ptr(m_sizes, ctypes.c_int64), G, N, K, int(a_format), int(b_format),
                                      1 if relu else 0, int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return C.reshape(rows, N) if N else C


def e2m1_to_f64(codes, lib=None) -> np.ndarray:
    lib = lib or load_library()
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    return np.array([lib.oracle_e2m1_to_f64(int(c)) for c in codes], dtype=np.float64)


def ue4m3_to_f64(codes, lib=None) -> np.ndarray:
    lib = lib or load_library()
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    return np.array([lib.oracle_ue4m3_to_f64(int(c)) for c in codes], dtype=np.float64)


def gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, row_offsets, N: int, K: int, alpha: float = 1.0, relu: bool = False,
                      C=None, nthreads: int = 0, lib=None) -> np.ndarray:
    """Grouped NVF4 GEMM: A (rows x K/2 packed E2M1 bytes), SFA (rows x K/16 UE4M3), B (G x N x K/2),
    SFB (G x N x K/16); returns bf16 bit patterns (rows x N); rows outside every group keep C's
    initial contents (zero by default)."""
    lib = lib or load_library()
    A = np.ascontiguousarray(np.asarray(A, dtype=np.uint8))
    SFA = np.ascontiguousarray(np.asarray(SFA, dtype=np.uint8))
    B = np.ascontiguousarray(np.asarray(B, dtype=np.uint8))
    SFB = np.ascontiguousarray(np.asarray(SFB, dtype=np.uint8))
    m_sizes = np.ascontiguousarray(np.asarray(m_sizes, dtype=np.int64))
    row_offsets = np.ascontiguousarray(np.asarray(row_offsets, dtype=np.int64))
    G = int(m_sizes.size)
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    rows = A.size // (K // 2) if K else 0
    if row_offsets.size != G or (G and int((row_offsets + m_sizes).max()) > rows):
        raise ValueError("groups do not fit in A")
    if B.size < G * N * (K // 2) or SFB.size < G * N * (K // 16) or SFA.size < rows * (K // 16):
        raise ValueError("operand too small")
    C = np.zeros(rows * N, np.uint16) if C is None else np.ascontiguousarray(np.asarray(C, np.uint16)).reshape(-1).copy()
    rc = lib.oracle_gemm_nvf4_grouped(_ptr(A, ctypes.c_uint8), _ptr(SFA, ctypes.c_uint8), _ptr(B, ctypes.c_uint8),
                                      _ptr(SFB, ctypes.c_uint8), _ptr(C, ctypes.c_uint16), _ptr(row_offsets, ctypes.c_int64),
                                      _ptr(m_sizes, ctypes.c_int64), G, N, K, float(alpha), 1 if relu else 0,
                                      int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return C.reshape(rows, N) if N else C


def dequant_w4_f16(Wq, S, N: int, K: int, group: int, lib=None) -> np.ndarray:
    """The N x K fp16 weight (float16 array) of 4-bit codes Wq (N x K/2 bytes) and fp16 scales
    S (N x K/group): f16_rne((q - 8) * s)."""
    lib = lib or load_library()
    Wq = np.ascontiguousarray(np.asarray(Wq, dtype=np.uint8))
    S = _u16(np.asarray(S))
    if Wq.size < N * (K // 2) or S.size < N * (K // group if group else 0):
        raise ValueError("operand too small")
    W = np.empty(N * K, np.uint16)
    if lib.oracle_dequant_w4_f16(_ptr(Wq, ctypes.c_uint8), _ptr(S, ctypes.c_uint16), _ptr(W, ctypes.c_uint16),
                                 N, K, group) != 0:
        raise ValueError("oracle rejected the arguments")
    return W.view(np.float16).reshape(N, K)


def gemm_relu_w4a16(A, Wq, S, group: int, nthreads: int = 0, lib=None) -> np.ndarray:
    """C = f16_rne(relu(A . dequant(W)^T)) for fp16 A (M x K): the dequantized weight, then the
    general-layout oracle with the weight stored N x K."""
    A = np.asarray(A)
    M, K = A.shape
    N = np.asarray(Wq).shape[0]
    W = dequant_w4_f16(Wq, S, N, K, group, lib=lib)
    return gemm_relu_f16_ex(A, W, M, N, K, K, K, N, b_nk=True, nthreads=nthreads, lib=lib).reshape(M, N)


def max_threads(lib=None) -> int:
    lib = lib or load_library()
    return int(lib.oracle_max_threads())
