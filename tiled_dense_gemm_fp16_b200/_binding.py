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
    GEMV = 4
    ZERO = 5
    TC_PAIR = 6
    TC_PAIR512 = 7
    REPACK = 8


class TGError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = Status(status) if status in Status._value2member_map_ else status
        super().__init__(f"{what}: {status_string(status)} ({int(status)})" if what else status_string(status))


EXPORTS = (
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
    used as given.  The library itself never allocates.
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
