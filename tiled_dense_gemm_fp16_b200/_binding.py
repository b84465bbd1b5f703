"""ctypes binding of ``libtg_gemm.so`` (the C ABI in ``include/tg_gemm.h``).

Argument marshalling only: every step of C = ReLU(A . B) runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or cannot be loaded,
every call raises.
"""
from __future__ import annotations

import ctypes
import enum
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtg_gemm.so")


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED_DEVICE = 2
    LAUNCH = 3
    TIMEOUT = 4
    INTERNAL = 5
    TOO_LARGE = 6


class Path(enum.IntEnum):
    INVALID = -2
    NONE = -1
    AUTO = 0
    TC = 1
    TC_EDGE = 2
    SKINNY = 3
    ZERO = 5
    TC_PAIR = 6
    TC_PAIR512 = 7
    REPACK = 8
    RC = 9


class TGError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = Status(status) if status in Status._value2member_map_ else status
        super().__init__(f"{what}: {status_string(status)} ({int(status)})" if what else status_string(status))


A_MK, A_KM = 0, 1
B_KN, B_NK = 0, 1
FP8_E4M3, FP8_E5M2 = 0, 1


class GemmOptions(ctypes.Structure):
    """Mirror of tg_gemm_options (include/tg_gemm.h)."""
    _fields_ = [
        ("lda", ctypes.c_int64),
        ("ldb", ctypes.c_int64),
        ("ldc", ctypes.c_int64),
        ("a_layout", ctypes.c_int32),
        ("b_layout", ctypes.c_int32),
        ("path", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("bias", ctypes.c_void_p),
        ("batch", ctypes.c_int64),
        ("stride_a", ctypes.c_int64),
        ("stride_b", ctypes.c_int64),
        ("stride_c", ctypes.c_int64),
    ]


EXPORTS = (
    "tg_gemm_relu_f16_ex",
    "tg_workspace_size_ex",
    "tg_select_path_ex",
    "tg_gemm_relu_f16",
    "tg_gemm_relu_f16_path",
    "tg_gemm_relu_f16_ws",
    "tg_workspace_size",
    "tg_select_path_ws",
    "tg_gemm_relu_f16_static_ws",
    "tg_select_path",
    "tg_path_supports",
    "tg_device_status",
    "tg_wait_timeout_selftest",
    "tg_status_string",
    "tg_path_name",
    "tg_version",
    "tg_gemm_mxf8_grouped",
    "tg_mx_grouped_rows",
    "tg_mx_scale_bytes",
    "tg_gemm_nvf4_grouped",
    "tg_nvf4_scale_bytes",
    "tg_gemm_relu_w4a16",
    "tg_w4a16_workspace_size",
    "tg_w4a16_kernel",
    "tg_dequant_w4_f16",
)

_lib = None
_lock = threading.Lock()


def _bind(lib):
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.tg_gemm_relu_f16.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    lib.tg_gemm_relu_f16.restype = i32
    lib.tg_gemm_relu_f16_path.argtypes = [vp, vp, vp, i64, i64, i64, vp, i32]
    lib.tg_gemm_relu_f16_path.restype = i32
    lib.tg_select_path.argtypes = [vp, vp, vp, i64, i64, i64]
    lib.tg_select_path.restype = i32
    lib.tg_gemm_relu_f16_ws.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp, i64]
    lib.tg_gemm_relu_f16_ws.restype = i32
    lib.tg_workspace_size.argtypes = [vp, vp, vp, i64, i64, i64]
    lib.tg_workspace_size.restype = i64
    lib.tg_select_path_ws.argtypes = [vp, vp, vp, i64, i64, i64, i64]
    lib.tg_select_path_ws.restype = i32
    lib.tg_gemm_relu_f16_static_ws.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    lib.tg_gemm_relu_f16_static_ws.restype = i32
    optp = ctypes.POINTER(GemmOptions)
    lib.tg_gemm_relu_f16_ex.argtypes = [vp, vp, vp, i64, i64, i64, optp, vp, vp, i64]
    lib.tg_gemm_relu_f16_ex.restype = i32
    lib.tg_workspace_size_ex.argtypes = [vp, vp, vp, i64, i64, i64, optp]
    lib.tg_workspace_size_ex.restype = i64
    lib.tg_select_path_ex.argtypes = [vp, vp, vp, i64, i64, i64, optp, i64]
    lib.tg_select_path_ex.restype = i32
    lib.tg_path_supports.argtypes = [i32, vp, vp, vp, i64, i64, i64]
    lib.tg_path_supports.restype = i32
    lib.tg_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.tg_device_status.restype = i32
    lib.tg_wait_timeout_selftest.argtypes = [i64, vp]
    lib.tg_wait_timeout_selftest.restype = i32
    lib.tg_status_string.argtypes = [i32]
    lib.tg_status_string.restype = ctypes.c_char_p
    lib.tg_path_name.argtypes = [i32]
    lib.tg_path_name.restype = ctypes.c_char_p
    lib.tg_version.argtypes = []
    lib.tg_version.restype = i32
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.tg_gemm_mxf8_grouped.argtypes = [vp, vp, vp, vp, vp, i64p, ctypes.c_int32, i64, i64, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, vp]
    lib.tg_gemm_mxf8_grouped.restype = i32
    lib.tg_mx_grouped_rows.argtypes = [i64p, ctypes.c_int32]
    lib.tg_mx_grouped_rows.restype = i64
    lib.tg_mx_scale_bytes.argtypes = [i64, i64]
    lib.tg_mx_scale_bytes.restype = i64
    lib.tg_gemm_nvf4_grouped.argtypes = [vp, vp, vp, vp, vp, i64p, ctypes.c_int32, i64, i64, ctypes.c_float,
                                         ctypes.c_int32, vp]
    lib.tg_gemm_nvf4_grouped.restype = i32
    lib.tg_nvf4_scale_bytes.argtypes = [i64, i64]
    lib.tg_nvf4_scale_bytes.restype = i64
    lib.tg_gemm_relu_w4a16.argtypes = [vp, vp, vp, vp, i64, i64, i64, ctypes.c_int32, vp, vp, i64]
    lib.tg_gemm_relu_w4a16.restype = i32
    lib.tg_w4a16_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int32]
    lib.tg_w4a16_workspace_size.restype = i64
    lib.tg_w4a16_kernel.argtypes = [i64, i64, i64, ctypes.c_int32]
    lib.tg_w4a16_kernel.restype = ctypes.c_int
    lib.tg_dequant_w4_f16.argtypes = [vp, vp, vp, i64, i64, ctypes.c_int32, vp]
    lib.tg_dequant_w4_f16.restype = i32
    return lib


def lib():
    """The loaded C library; raises if ``libtg_gemm.so`` is missing."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"{LIB_PATH} is not built; run `python -m tiled_dense_gemm_fp16_b200.build` "
                        "(there is no fallback implementation)")
                _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(status: int) -> str:
    return lib().tg_status_string(int(status)).decode()


def path_name(path: int) -> str:
    return lib().tg_path_name(int(path)).decode()


def version() -> int:
    return int(lib().tg_version())


def _check(st, what):
    if st != Status.OK:
        raise TGError(st, what)


# ---------------------------------------------------------------------------
# Raw pointer API (mirrors the C ABI one to one)
# ---------------------------------------------------------------------------

def gemm_relu_f16_raw(A: int, B: int, C: int, M: int, N: int, K: int, stream: int = 0, path: int = Path.AUTO) -> int:
    """Call the C ABI on raw device pointers; returns the tg_status value."""
    if int(path) == Path.AUTO:
        return int(lib().tg_gemm_relu_f16(A, B, C, M, N, K, stream))
    return int(lib().tg_gemm_relu_f16_path(A, B, C, M, N, K, stream, int(path)))


def gemm_relu_f16_ws_raw(A: int, B: int, C: int, M: int, N: int, K: int, stream: int, ws: int, ws_bytes: int) -> int:
    """tg_gemm_relu_f16_ws on raw device pointers; returns the tg_status value."""
    return int(lib().tg_gemm_relu_f16_ws(A, B, C, M, N, K, stream, ws, ws_bytes))


def gemm_relu_f16_static_ws_raw(A: int, B: int, C: int, M: int, N: int, K: int, stream: int = 0) -> int:
    """tg_gemm_relu_f16_static_ws on raw device pointers (no allocation anywhere); returns the tg_status."""
    return int(lib().tg_gemm_relu_f16_static_ws(A, B, C, M, N, K, stream))


STATIC_WORKSPACE_BYTES = 16 * 1024 * 1024


def workspace_size(A: int, B: int, C: int, M: int, N: int, K: int) -> int:
    return int(lib().tg_workspace_size(A, B, C, M, N, K))


def options(lda=0, ldb=0, ldc=0, b_layout=B_KN, bias=0, batch=0, stride_a=0, stride_b=0, stride_c=0,
            path=Path.AUTO, a_layout=A_MK, reserved=0) -> GemmOptions:
    """A tg_gemm_options value (zeros mean the dense defaults)."""
    return GemmOptions(lda, ldb, ldc, int(a_layout), int(b_layout), int(path), int(reserved), bias or None, batch,
                       stride_a, stride_b, stride_c)


def gemm_relu_f16_ex_raw(A: int, B: int, C: int, M: int, N: int, K: int, opts: GemmOptions | None = None,
                         stream: int = 0, ws: int = 0, ws_bytes: int = 0) -> int:
    """tg_gemm_relu_f16_ex on raw device pointers; returns the tg_status value."""
    return int(lib().tg_gemm_relu_f16_ex(A, B, C, M, N, K, ctypes.byref(opts) if opts is not None else None,
                                         stream, ws, ws_bytes))


def workspace_size_ex(A: int, B: int, C: int, M: int, N: int, K: int, opts: GemmOptions | None = None) -> int:
    return int(lib().tg_workspace_size_ex(A, B, C, M, N, K, ctypes.byref(opts) if opts is not None else None))


def select_path_ex(A: int, B: int, C: int, M: int, N: int, K: int, opts: GemmOptions | None = None,
                   ws_bytes: int = 0) -> int:
    return int(lib().tg_select_path_ex(A, B, C, M, N, K, ctypes.byref(opts) if opts is not None else None, ws_bytes))


def select_path(A: int, B: int, C: int, M: int, N: int, K: int) -> int:
    return int(lib().tg_select_path(A, B, C, M, N, K))


def select_path_ws(A: int, B: int, C: int, M: int, N: int, K: int, ws_bytes: int) -> int:
    return int(lib().tg_select_path_ws(A, B, C, M, N, K, ws_bytes))


def path_supports(path: int, A: int, B: int, C: int, M: int, N: int, K: int) -> bool:
    return bool(lib().tg_path_supports(int(path), A, B, C, M, N, K))


def device_status():
    """(Status, raw error word) after synchronizing the current device."""
    word = ctypes.c_uint32(0)
    st = int(lib().tg_device_status(ctypes.byref(word)))
    return Status(st), int(word.value)


def wait_timeout_selftest(budget_ns: int, stream: int = 0) -> int:
    return int(lib().tg_wait_timeout_selftest(int(budget_ns), stream))


# ---------------------------------------------------------------------------
# torch tensor API
# ---------------------------------------------------------------------------

def _stream_handle(device):
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def gemm_relu(A, B, out=None, path: int = Path.AUTO, stream=None, workspace="auto"):
    """C = ReLU(A @ B) for row-major fp16 CUDA tensors A (M, K) and B (K, N).

    ``out`` (M, N) fp16 on the same device is written in place if given.
    Runs on ``stream`` (a torch.cuda.Stream) or on the current stream.
    ``workspace``: "auto" lets torch allocate the scratch bytes the repack path
    needs when TMA cannot describe A or B (odd row lengths, unaligned bases);
    None never uses a workspace (edge mode instead); a uint8 CUDA tensor is
    used as given.  The library itself allocates nothing at run time.
    """
    import torch
    if A.dtype != torch.float16 or B.dtype != torch.float16:
        raise TypeError("A and B must be torch.float16")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise ValueError(f"shape mismatch: A{tuple(A.shape)} B{tuple(B.shape)}")
    if not (A.is_cuda and B.is_cuda) or A.device != B.device:
        raise ValueError("A and B must be CUDA tensors on the same device")
    if not (A.is_contiguous() and B.is_contiguous()):
        raise ValueError("A and B must be contiguous row-major tensors")
    M, K = A.shape
    N = B.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=A.device)
    elif (out.dtype != torch.float16 or tuple(out.shape) != (M, N) or not out.is_contiguous()
          or out.device != A.device):
        raise ValueError("out must be a contiguous (M, N) float16 tensor on A's device")
    handle = stream.cuda_stream if stream is not None else _stream_handle(A.device)
    a, b, c = A.data_ptr(), B.data_ptr(), out.data_ptr()
    with torch.cuda.device(A.device):
        if int(path) == Path.AUTO and workspace is not None:
            need = workspace_size(a, b, c, M, N, K)
            if need > 0:
                if isinstance(workspace, str):
                    workspace = torch.empty(need, dtype=torch.uint8, device=A.device)
                st = gemm_relu_f16_ws_raw(a, b, c, M, N, K, handle, workspace.data_ptr(), workspace.numel())
                _check(st, "tg_gemm_relu_f16_ws")
                return out
        st = gemm_relu_f16_raw(a, b, c, M, N, K, handle, path)
    _check(st, "tg_gemm_relu_f16")
    return out


def _call_ex(a, b, c, M, N, K, opts, device, stream, workspace):
    import torch
    handle = stream.cuda_stream if stream is not None else _stream_handle(device)
    with torch.cuda.device(device):
        need = workspace_size_ex(a, b, c, M, N, K, opts)
        if need < 0:
            raise TGError(Status.INVALID_ARG, "tg_workspace_size_ex")
        ws_ptr, ws_bytes = 0, 0
        if need > 0 and workspace is not None:
            if isinstance(workspace, str):
                workspace = torch.empty(need, dtype=torch.uint8, device=device)
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        st = gemm_relu_f16_ex_raw(a, b, c, M, N, K, opts, handle, ws_ptr, ws_bytes)
    _check(st, "tg_gemm_relu_f16_ex")


def linear_relu(x, weight, bias=None, out=None, stream=None, workspace="auto"):
    """ReLU(x @ weight^T + bias) for fp16 CUDA tensors: x (..., K), weight (N, K) as a
    linear layer stores it, bias (N,) or None.  Leading dimensions of x are flattened
    into M rows (x must be contiguous)."""
    import torch
    if x.dtype != torch.float16 or weight.dtype != torch.float16:
        raise TypeError("x and weight must be torch.float16")
    if weight.dim() != 2 or x.shape[-1] != weight.shape[1]:
        raise ValueError(f"shape mismatch: x{tuple(x.shape)} weight{tuple(weight.shape)}")
    if not (x.is_contiguous() and weight.is_contiguous()):
        raise ValueError("x and weight must be contiguous")
    K = x.shape[-1]
    N = weight.shape[0]
    lead = tuple(x.shape[:-1])
    M = 1
    for d in lead:
        M *= d
    if bias is not None and (bias.dtype != torch.float16 or bias.numel() != N or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous float16 tensor of N elements")
    if out is None:
        out = torch.empty(lead + (N,), dtype=torch.float16, device=x.device)
    opts = options(b_layout=B_NK, bias=bias.data_ptr() if bias is not None else 0)
    _call_ex(x.data_ptr(), weight.data_ptr(), out.data_ptr(), M, N, K, opts, x.device, stream, workspace)
    return out


def bmm_relu(A, B, bias=None, out=None, stream=None, workspace="auto"):
    """ReLU(A[e] @ B[e] + bias) for fp16 CUDA tensors A (b, M, K) and B (b, K, N)."""
    import torch
    if A.dim() != 3 or B.dim() != 3 or A.shape[0] != B.shape[0] or A.shape[2] != B.shape[1]:
        raise ValueError(f"shape mismatch: A{tuple(A.shape)} B{tuple(B.shape)}")
    if A.dtype != torch.float16 or B.dtype != torch.float16 or not (A.is_contiguous() and B.is_contiguous()):
        raise ValueError("A and B must be contiguous float16 tensors")
    nb, M, K = A.shape
    N = B.shape[2]
    if out is None:
        out = torch.empty((nb, M, N), dtype=torch.float16, device=A.device)
    opts = options(bias=bias.data_ptr() if bias is not None else 0, batch=nb, stride_a=M * K, stride_b=K * N,
                   stride_c=M * N)
    _call_ex(A.data_ptr(), B.data_ptr(), out.data_ptr(), M, N, K, opts, A.device, stream, workspace)
    return out


# ---------------------------------------------------------------------------
# MXFP8 grouped GEMM
# ---------------------------------------------------------------------------

def _i64_array(values):
    values = [int(v) for v in values]
    return (ctypes.c_int64 * max(1, len(values)))(*values), len(values)


def mx_grouped_rows(m_sizes) -> int:
    """Stacked rows of A / C for these group sizes (each group padded to 128 rows); -1 if invalid."""
    arr, n = _i64_array(m_sizes)
    return int(lib().tg_mx_grouped_rows(arr, n))


def mx_scale_bytes(rows: int, K: int) -> int:
    """Bytes of one blocked UE8M0 scale array for ``rows`` rows and K elements."""
    return int(lib().tg_mx_scale_bytes(rows, K))


def gemm_mxf8_grouped_raw(A: int, SFA: int, B: int, SFB: int, C: int, m_sizes, N: int, K: int,
                          a_format: int = FP8_E4M3, b_format: int = FP8_E4M3, relu: bool = False,
                          stream: int = 0) -> int:
    arr, n = _i64_array(m_sizes)
    return int(lib().tg_gemm_mxf8_grouped(A, SFA, B, SFB, C, arr, n, N, K, int(a_format), int(b_format),
                                          1 if relu else 0, stream))


def mxf8_grouped(A, SFA, B, SFB, m_sizes, relu=False, a_format=FP8_E4M3, b_format=FP8_E4M3, out=None,
                 stream=None):
    """Grouped MXFP8 GEMM on CUDA tensors (uint8 codes): A (rows, K), B (G, N, K), SFA / SFB in the
    blocked scale layout; returns C (rows, N) bfloat16 (rows outside the groups untouched)."""
    import torch
    if A.dim() != 2 or B.dim() != 3 or A.shape[1] != B.shape[2] or B.shape[0] != len(m_sizes):
        raise ValueError(f"shape mismatch: A{tuple(A.shape)} B{tuple(B.shape)} groups={len(m_sizes)}")
    rows, K = A.shape
    N = B.shape[1]
    if rows != mx_grouped_rows(m_sizes):
        raise ValueError("A must have tg_mx_grouped_rows(m_sizes) rows")
    for t in (A, B, SFA, SFB):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise TypeError("operands and scales must be contiguous uint8 tensors")
    if out is None:
        out = torch.empty((rows, N), dtype=torch.bfloat16, device=A.device)
    handle = stream.cuda_stream if stream is not None else _stream_handle(A.device)
    with torch.cuda.device(A.device):
        st = gemm_mxf8_grouped_raw(A.data_ptr(), SFA.data_ptr(), B.data_ptr(), SFB.data_ptr(), out.data_ptr(),
                                   m_sizes, N, K, a_format, b_format, relu, handle)
    _check(st, "tg_gemm_mxf8_grouped")
    return out


# ---------------------------------------------------------------------------
# NVF4 grouped GEMM
# ---------------------------------------------------------------------------

def nvf4_scale_bytes(rows: int, K: int) -> int:
    """Bytes of one blocked UE4M3 scale array for ``rows`` rows and K elements."""
    return int(lib().tg_nvf4_scale_bytes(rows, K))


def gemm_nvf4_grouped_raw(A: int, SFA: int, B: int, SFB: int, C: int, m_sizes, N: int, K: int, alpha: float = 1.0,
                          relu: bool = False, stream: int = 0) -> int:
    arr, n = _i64_array(m_sizes)
    return int(lib().tg_gemm_nvf4_grouped(A, SFA, B, SFB, C, arr, n, N, K, float(alpha), 1 if relu else 0, stream))


def nvf4_grouped(A, SFA, B, SFB, m_sizes, alpha=1.0, relu=False, out=None, stream=None):
    """Grouped NVF4 GEMM on CUDA uint8 tensors: A (rows, K/2) and B (G, N, K/2) packed E2M1, SFA / SFB
    blocked UE4M3 scales; returns C (rows, N) bfloat16 (rows outside the groups untouched)."""
    import torch
    if A.dim() != 2 or B.dim() != 3 or A.shape[1] != B.shape[2] or B.shape[0] != len(m_sizes):
        raise ValueError(f"shape mismatch: A{tuple(A.shape)} B{tuple(B.shape)} groups={len(m_sizes)}")
    rows, K = A.shape[0], 2 * A.shape[1]
    N = B.shape[1]
    if rows != mx_grouped_rows(m_sizes):
        raise ValueError("A must have tg_mx_grouped_rows(m_sizes) rows")
    for t in (A, B, SFA, SFB):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise TypeError("operands and scales must be contiguous uint8 tensors")
    if out is None:
        out = torch.empty((rows, N), dtype=torch.bfloat16, device=A.device)
    handle = stream.cuda_stream if stream is not None else _stream_handle(A.device)
    with torch.cuda.device(A.device):
        st = gemm_nvf4_grouped_raw(A.data_ptr(), SFA.data_ptr(), B.data_ptr(), SFB.data_ptr(), out.data_ptr(),
                                   m_sizes, N, K, alpha, relu, handle)
    _check(st, "tg_gemm_nvf4_grouped")
    return out


# ---------------------------------------------------------------------------
# 4-bit weight-only GEMM (W4A16)
# ---------------------------------------------------------------------------

def w4a16_workspace_size(M: int, N: int, K: int, group: int) -> int:
    return int(lib().tg_w4a16_workspace_size(M, N, K, group))


class W4Kernel(enum.IntEnum):
    INVALID = -1
    NONE = 0
    DECODE = 1
    FUSED = 2
    DEQUANT_GEMM = 3


def w4a16_kernel(M: int, N: int, K: int, group: int) -> "W4Kernel":
    """The kernels tg_gemm_relu_w4a16 runs for these sizes (host logic only)."""
    return W4Kernel(int(lib().tg_w4a16_kernel(M, N, K, group)))


def gemm_relu_w4a16_raw(A: int, Wq: int, S: int, C: int, M: int, N: int, K: int, group: int, stream: int = 0,
                        workspace: int = 0, workspace_bytes: int = 0) -> int:
    return int(lib().tg_gemm_relu_w4a16(A, Wq, S, C, M, N, K, group, stream, workspace, workspace_bytes))


def dequant_w4_f16_raw(Wq: int, S: int, W: int, N: int, K: int, group: int, stream: int = 0) -> int:
    return int(lib().tg_dequant_w4_f16(Wq, S, W, N, K, group, stream))


def gemm_relu_w4a16(A, Wq, S, group, out=None, stream=None, workspace="auto"):
    """ReLU(A @ dequant(W)^T) for CUDA tensors: A (M, K) float16, Wq (N, K/2) uint8 packed codes,
    S (N, K/group) float16 scales; returns C (M, N) float16."""
    import torch
    if A.dim() != 2 or Wq.dim() != 2 or S.dim() != 2 or Wq.shape[1] * 2 != A.shape[1] or S.shape[0] != Wq.shape[0]:
        raise ValueError(f"shape mismatch: A{tuple(A.shape)} Wq{tuple(Wq.shape)} S{tuple(S.shape)}")
    if A.dtype != torch.float16 or S.dtype != torch.float16 or Wq.dtype != torch.uint8:
        raise TypeError("A and S must be float16, Wq uint8")
    if not (A.is_contiguous() and Wq.is_contiguous() and S.is_contiguous()):
        raise ValueError("A, Wq and S must be contiguous")
    M, K = A.shape
    N = Wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=A.device)
    handle = stream.cuda_stream if stream is not None else _stream_handle(A.device)
    with torch.cuda.device(A.device):
        need = w4a16_workspace_size(M, N, K, group)
        if need < 0:
            raise TGError(Status.INVALID_ARG, "tg_w4a16_workspace_size")
        ws_ptr, ws_bytes = 0, 0
        if need > 0 and workspace is not None:
            if isinstance(workspace, str):
                workspace = torch.empty(need, dtype=torch.uint8, device=A.device)
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        st = gemm_relu_w4a16_raw(A.data_ptr(), Wq.data_ptr(), S.data_ptr(), out.data_ptr(), M, N, K, group, handle,
                                 ws_ptr, ws_bytes)
    _check(st, "tg_gemm_relu_w4a16")
    return out
