"""B200 (sm_100a) tiled fp16 GEMM with fused ReLU: C = ReLU(A . B).

The compute path is the C-ABI library ``libtg_gemm.so`` (hand-written CUDA
kernels: TMA, tcgen05.mma into tensor memory, fused ReLU + fp16 epilogue).
This package only marshals arguments to it; the library is loaded on first
use and every call raises if it is missing.
"""
from ._binding import (  # noqa: F401
    A_KM,
    A_MK,
    B_KN,
    B_NK,
    EXPORTS,
    FP8_E4M3,
    FP8_E5M2,
    GemmOptions,
    LIB_PATH,
    STATIC_WORKSPACE_BYTES,
    Path,
    Status,
    TGError,
    bmm_relu,
    device_status,
    gemm_relu,
    gemm_relu_f16_ex_raw,
    gemm_relu_f16_raw,
    gemm_relu_f16_static_ws_raw,
    gemm_relu_f16_ws_raw,
    gemm_mxf8_grouped_raw,
    gemm_nvf4_grouped_raw,
    linear_relu,
    lib,
    mx_grouped_rows,
    mx_scale_bytes,
    mxf8_grouped,
    nvf4_grouped,
    nvf4_scale_bytes,
    options,
    path_name,
    path_supports,
    select_path,
    select_path_ex,
    select_path_ws,
    status_string,
    version,
    wait_timeout_selftest,
    workspace_size,
    workspace_size_ex,
)
