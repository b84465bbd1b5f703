"""Helpers shared by the GPU parity tests: run the C-ABI path with guard bands
around C, and compare against the oracle."""
from __future__ import annotations

import numpy as np

GUARD = 64                 # fp16 elements (128 bytes) on each side of C
GUARD_BITS = 0x7E55        # a NaN pattern the kernels never write
ATOL, RTOL = 1e-3, 4e-3    # |gpu - ref| <= ATOL + RTOL * |ref|


def run_gpu(A: np.ndarray, B: np.ndarray, path=None, stream=None, offset_elems: int = 0, offsets=None,
            workspace: bool = False):
    """C = ReLU(A . B) through the C ABI; returns (C as float16 numpy, guards intact?).

    ``offset_elems`` shifts A, B and C by that many fp16 elements from a
    16-byte boundary (``offsets`` = (a, b, c) shifts them separately), to
    exercise base-pointer alignment handling.  ``workspace`` calls
    tg_gemm_relu_f16_ws with exactly tg_workspace_size bytes of workspace.
    """
    import torch
    import tiled_dense_gemm_fp16_b200 as tg

    M, K = A.shape
    N = B.shape[1]
    dev = torch.device("cuda", 0)
    oa, ob, oc = offsets if offsets is not None else (offset_elems,) * 3

    def put(x, off):
        buf = torch.empty(x.size + 8, dtype=torch.float16, device=dev)
        view = buf[off:off + x.size].view(x.shape)
        view.copy_(torch.from_numpy(np.ascontiguousarray(x)).to(dev))
        return buf, view

    _, Ad = put(A, oa)
    _, Bd = put(B, ob)
    cbuf = torch.full((M * N + 2 * GUARD + 8,), GUARD_BITS, dtype=torch.int16, device=dev)
    cbuf = cbuf.view(torch.float16)
    C = cbuf[GUARD + oc:GUARD + oc + M * N].view(M, N)
    sh = (stream or torch.cuda.current_stream(dev)).cuda_stream
    if workspace:
        need = tg.workspace_size(Ad.data_ptr(), Bd.data_ptr(), C.data_ptr(), M, N, K)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        st = tg.gemm_relu_f16_ws_raw(Ad.data_ptr(), Bd.data_ptr(), C.data_ptr(), M, N, K, sh, ws.data_ptr(), need)
    else:
        st = tg.gemm_relu_f16_raw(Ad.data_ptr(), Bd.data_ptr(), C.data_ptr(), M, N, K, sh,
                                  tg.Path.AUTO if path is None else path)
    if st != tg.Status.OK:
        raise tg.TGError(st, "tg_gemm_relu_f16")
    torch.cuda.synchronize(dev)
    dst, word = tg.device_status()
    assert dst == tg.Status.OK, f"device error word 0x{word:x}"
    host = cbuf.view(torch.int16).cpu().numpy().view(np.uint16)
    lo = host[:GUARD + oc]
    hi = host[GUARD + oc + M * N:]
    guards_ok = bool(np.all(lo == GUARD_BITS) and np.all(hi == GUARD_BITS))
    out = host[GUARD + oc:GUARD + oc + M * N].reshape(M, N).view(np.float16)
    return out, guards_ok


def assert_bitexact(got: np.ndarray, ref: np.ndarray, what=""):
    g, r = got.view(np.uint16), ref.view(np.uint16)
    bad = np.argwhere(g != r)
    assert bad.size == 0, (f"{what}: {len(bad)} mismatches, first at {tuple(bad[0])}: "
                           f"gpu 0x{int(g[tuple(bad[0])]):04x} oracle 0x{int(r[tuple(bad[0])]):04x}")


def assert_close(got: np.ndarray, ref: np.ndarray, what=""):
    g = got.astype(np.float64)
    r = ref.astype(np.float64)
    assert not np.any(got.view(np.uint16) & 0x8000), f"{what}: negative or -0 output"
    both_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    err = np.where(both_inf, 0.0, np.abs(g - r))
    tol = ATOL + RTOL * np.abs(r)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {len(bad)} elements out of tolerance, first at {tuple(bad[0])}: "
                           f"gpu {g[tuple(bad[0])]} oracle {r[tuple(bad[0])]}, max err {np.nanmax(err)}")
    return float(np.max(err)) if err.size else 0.0


def sample_rows(M: int, n: int = 48, seed: int = 0, tile: int = 128):
    """Rows to check at full size: tile boundaries, the last rows and random ones."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, M - 1, M - 2, min(tile - 1, M - 1), min(tile, M - 1)}
    rows |= {int(r) for r in rng.integers(0, M, size=n)}
    return sorted(r for r in rows if 0 <= r < M)
