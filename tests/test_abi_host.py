"""C-ABI library: it loads, exports every function the headers declare, and its
host-side argument logic (validation, path choice) behaves as documented.
No kernel is launched: these run without a GPU."""
import ctypes
import glob
import os
import re

import pytest

import tiled_dense_gemm_fp16_b200 as tg
from tiled_dense_gemm_fp16_b200 import Path, Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Well-separated fake device addresses (never dereferenced by host logic).
A0, B0, C0 = 0x10_0000_0000, 0x20_0000_0000, 0x30_0000_0000


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"TG_API\s+[^;(]*?\b(tg_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_loads_and_exports_every_declared_symbol():
    lib = tg.lib()
    names = declared_functions()
    assert "tg_gemm_relu_f16" in names and len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert isinstance(getattr(lib, n), ctypes._CFuncPtr)
    assert set(tg.EXPORTS) <= set(names)


def test_version_and_strings():
    assert tg.version() >= 100
    assert tg.status_string(Status.OK) == "ok"
    assert "invalid" in tg.status_string(Status.INVALID_ARG)
    assert tg.path_name(Path.TC) == "tc" and tg.path_name(Path.TC_EDGE) == "tc_edge"
    assert tg.path_name(Path.TC_PAIR) == "tc_pair" and tg.path_name(Path.SKINNY) == "skinny"
    assert tg.path_name(Path.TC_PAIR512) == "tc_pair512"
    assert tg.status_string(99) == "unknown status"


@pytest.mark.parametrize("M,N,K", [(-1, 4, 4), (4, -1, 4), (4, 4, -1), (2**31, 8, 8), (8, 2**31, 8), (8, 8, 2**31)])
def test_invalid_sizes(M, N, K):
    assert tg.select_path(A0, B0, C0, M, N, K) == Path.INVALID
    assert tg.gemm_relu_f16_raw(A0, B0, C0, M, N, K) == Status.INVALID_ARG


def test_null_pointers():
    assert tg.gemm_relu_f16_raw(0, B0, C0, 8, 8, 8) == Status.INVALID_ARG
    assert tg.gemm_relu_f16_raw(A0, 0, C0, 8, 8, 8) == Status.INVALID_ARG
    assert tg.gemm_relu_f16_raw(A0, B0, 0, 8, 8, 8) == Status.INVALID_ARG
    # Empty C: nothing to do, pointers may be NULL, no CUDA call is made.
    assert tg.gemm_relu_f16_raw(0, 0, 0, 0, 8, 8) == Status.OK
    assert tg.gemm_relu_f16_raw(0, 0, 0, 8, 0, 8) == Status.OK
    assert tg.select_path(0, 0, 0, 0, 0, 0) == Path.NONE


def test_odd_pointer_rejected():
    assert tg.gemm_relu_f16_raw(A0 + 1, B0, C0, 8, 8, 8) == Status.INVALID_ARG
    assert tg.gemm_relu_f16_raw(A0, B0, C0 + 1, 8, 8, 8) == Status.INVALID_ARG


def test_overlap_rejected():
    M, N, K = 64, 64, 64
    # C overlapping the last byte of A, or starting inside B.
    assert tg.gemm_relu_f16_raw(A0, B0, A0 + 2 * M * K - 2, M, N, K) == Status.INVALID_ARG
    assert tg.gemm_relu_f16_raw(A0, B0, B0 + 128, M, N, K) == Status.INVALID_ARG
    # Adjacent but not overlapping is fine for the host logic.
    assert tg.select_path(A0, B0, A0 + 2 * M * K, M, N, K) == Path.SKINNY


def test_path_selection():
    assert tg.select_path(A0, B0, C0, 128, 128, 0) == Path.ZERO
    # Large aligned shapes: the tensor-core kernel whose tile waves cost least.
    assert tg.select_path(A0, B0, C0, 4096, 4096, 4096) == Path.TC_PAIR512
    assert tg.select_path(A0, B0, C0, 8192, 8192, 8192) == Path.TC_PAIR512
    assert tg.select_path(A0, B0, C0, 300, 264, 64) == Path.TC_PAIR       # 4 pair tiles vs 2 wide ones
    assert tg.select_path(A0, B0, C0, 20000, 256, 64) == Path.TC_PAIR
    assert tg.select_path(A0, B0, C0, 384, 10240, 64) == Path.TC          # 120 CTA tiles fit one wave
    # Small M with aligned rows: the split-K small-M kernel; above M = 128 only for a large B.
    for M in (1, 16, 64, 256):
        assert tg.select_path(A0, B0, C0, M, 8192, 8192) == Path.SKINNY
    assert tg.select_path(A0, B0, C0, 128, 256, 256) == Path.SKINNY
    assert tg.select_path(A0, B0, C0, 256, 4096, 4096) == Path.SKINNY
    assert tg.select_path(A0, B0, C0, 256, 256, 256) == Path.TC_PAIR
    assert tg.select_path(A0, B0, C0, 256, 2048, 2048) == Path.TC_PAIR
    assert tg.select_path(A0, B0, C0, 257, 8192, 8192) == Path.TC_PAIR
    assert tg.select_path(A0, B0, C0, 64, 8191, 8192) == Path.RC
    # Row strides that are not 16-byte multiples, or misaligned bases, need the edge mode.
    assert tg.select_path(A0, B0, C0, 3001, 5003, 1021) == Path.RC
    assert tg.select_path(A0, B0, C0, 777, 12289, 4095) == Path.RC
    assert tg.select_path(A0, B0, C0, 8191, 129, 8193) == Path.RC
    assert tg.select_path(A0 + 2, B0, C0, 256, 256, 256) == Path.RC


def test_forced_path_requirements():
    assert tg.path_supports(Path.TC, A0, B0, C0, 256, 256, 256)
    assert tg.path_supports(Path.TC_PAIR, A0, B0, C0, 256, 256, 256)
    assert not tg.path_supports(Path.TC_PAIR, A0, B0, C0, 256, 250, 256)
    assert tg.path_supports(Path.TC_PAIR512, A0, B0, C0, 256, 256, 256)
    assert not tg.path_supports(Path.TC_PAIR512, A0, B0, C0, 256, 256, 252)
    assert not tg.path_supports(Path.TC, A0, B0, C0, 256, 250, 256)
    assert not tg.path_supports(Path.TC, A0, B0, C0, 256, 256, 250)
    assert tg.path_supports(Path.TC_EDGE, A0, B0, C0, 256, 250, 250)
    assert not tg.path_supports(Path.ZERO, A0, B0, C0, 256, 256, 256)
    assert tg.path_supports(Path.ZERO, A0, B0, C0, 256, 256, 0)
    assert not tg.path_supports(42, A0, B0, C0, 256, 256, 256)
    assert tg.path_supports(Path.SKINNY, A0, B0, C0, 256, 256, 256)
    assert not tg.path_supports(Path.SKINNY, A0, B0, C0, 257, 256, 256)
    assert not tg.path_supports(Path.SKINNY, A0, B0, C0, 16, 250, 256)
    assert tg.gemm_relu_f16_raw(A0, B0, C0, 256, 250, 256, 0, Path.TC) == Status.INVALID_ARG


def test_no_device_is_reported_not_faked():
    """Without a GPU a valid call reports the missing device; it never computes on the CPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert tg.gemm_relu_f16_raw(A0, B0, C0, 64, 64, 64) == Status.UNSUPPORTED_DEVICE
    st, _ = tg.device_status()
    assert st == Status.UNSUPPORTED_DEVICE


def test_workspace_size_and_repack_choice():
    up = lambda x: (x + 255) // 256 * 256
    # TMA-describable operands and 16-byte aligned rows of C need no workspace.
    assert tg.workspace_size(A0, B0, C0, 8192, 8192, 8192) == 0
    # C's rows not 16-byte aligned: the fastest path writes a padded C
    # (M x N rounded up to 8) in the workspace; without one it still runs.
    assert tg.workspace_size(A0, B0, C0 + 2, 512, 512, 512) == up(2 * 512 * 512)
    assert tg.select_path(A0, B0, C0 + 2, 512, 512, 512) == Path.TC_PAIR
    assert tg.select_path_ws(A0, B0, C0 + 2, 512, 512, 512, up(2 * 512 * 512)) == Path.REPACK
    assert tg.select_path_ws(A0, B0, C0 + 2, 512, 512, 512, up(2 * 512 * 512) - 1) == Path.TC_PAIR
    # Operands TMA cannot describe.  When 1/N + 1/K > 1/2400 the residue-class kernel takes
    # them, needing at most a padded copy of B (rows rounded up to 8 elements, 256-byte aligned).
    assert tg.workspace_size(A0, B0, C0, 512, 509, 512) == up(2 * 512 * 512)        # odd N: B copy only
    assert tg.select_path_ws(A0, B0, C0, 512, 509, 512, up(2 * 512 * 512)) == Path.RC
    assert tg.workspace_size(A0, B0, C0 + 2, 64, 512, 512) == 0                      # the small-M kernel
    M, N, K = 3001, 5003, 1021
    assert tg.workspace_size(A0, B0, C0, M, N, K) == up(2 * K * 5008)
    # One column of 144-wide tiles with 256 rows and 32+ k-blocks per CTA: B is realigned in
    # place with two k-blocks in flight, faster than copying it first, so no workspace.
    assert tg.workspace_size(A0, B0, C0, 8191, 129, 8193) == 0
    assert tg.select_path_ws(A0, B0, C0, 8191, 129, 8193, up(2 * 8193 * 136)) == Path.RC
    # Short K walks (17 k-blocks) keep the copy: (8191, 129, 1027).
    assert tg.workspace_size(A0, B0, C0, 8191, 129, 1027) == up(2 * 1027 * 136)
    assert tg.workspace_size(A0, B0, C0, 64, 64, 100) == 0                          # odd K: only A, read in place
    assert tg.workspace_size(A0 + 2, B0, C0, 64, 64, 64) == 0                       # misaligned A base
    assert tg.workspace_size(A0, B0, C0, -1, 4, 4) == -1
    for ws in (0, up(2 * K * 5008)):
        assert tg.select_path_ws(A0, B0, C0, M, N, K, ws) == Path.RC
    # Large N and K: the repack path (copies of A, B and C around the CTA-pair kernel) when the
    # workspace holds its copies, the residue-class kernel otherwise.
    M, N, K = 777, 12289, 4095
    ab = up(2 * M * 4096) + up(2 * K * 12296)
    need = tg.workspace_size(A0, B0, C0, M, N, K)
    assert need == ab + up(2 * M * 12296)
    assert tg.select_path_ws(A0, B0, C0, M, N, K, need) == Path.REPACK
    assert tg.select_path_ws(A0, B0, C0, M, N, K, ab) == Path.REPACK                # A and B copies only
    assert tg.select_path_ws(A0, B0, C0, M, N, K, ab - 1) == Path.RC
    assert tg.select_path_ws(A0, B0, C0, 4096, 4096, 4096, need) == Path.TC_PAIR512


def test_w4a16_kernel_choice():
    K4 = tg.W4Kernel
    assert tg.w4a16_kernel(16, 8192, 8192, 128) == K4.DECODE      # the decode workload
    assert tg.w4a16_kernel(1, 1, 256, 32) == K4.DECODE
    assert tg.w4a16_kernel(1, 1, 384, 32) == K4.FUSED               # K % 256 != 0
    assert tg.w4a16_kernel(16, 8192, 16384, 128) == K4.DECODE     # K / 8 = 2048: the longest slice
    assert tg.w4a16_kernel(16, 8192, 32768, 128) == K4.FUSED      # slices would be longer
    assert tg.w4a16_kernel(16, 8192, 8192 + 128, 128) == K4.FUSED  # K % 256 != 0
    assert tg.w4a16_kernel(17, 8192, 8192, 128) == K4.FUSED
    assert tg.w4a16_kernel(256, 8192, 8192, 128) == K4.FUSED
    assert tg.w4a16_kernel(257, 8192, 8192, 128) == K4.DEQUANT_GEMM
    assert tg.w4a16_kernel(0, 8192, 8192, 128) == K4.NONE
    assert tg.w4a16_kernel(4, 8, 0, 32) == K4.NONE
    assert tg.w4a16_kernel(4, 8, 128, 48) == K4.INVALID          # group not a power of two
    assert tg.w4a16_kernel(4, 8, 96, 32) == K4.INVALID           # K % 64 != 0
    assert tg.w4a16_kernel(-1, 8, 128, 32) == K4.INVALID


def test_environment_cannot_change_the_shipped_kernel_choice(monkeypatch):
    # Tuning knobs exist only in a -DTG_TUNING build; the shipped library ignores them.
    monkeypatch.setenv("TG_TUNE_W4_DECODE", "0")
    assert tg.w4a16_kernel(16, 8192, 8192, 128) == tg.W4Kernel.DECODE


def test_padded_c_with_general_layouts():
    up = lambda x: (x + 255) // 256 * 256
    M, N, K = 1000, 1001, 512      # A and B describable by TMA in every layout below; C rows of 2002 bytes
    # B K x N with rows of 1001: the residue-class kernel on a padded copy of B, writing C itself.
    need = tg.workspace_size_ex(A0, B0, C0, M, N, K, tg.options())
    assert need == up(2 * K * 1008)
    assert tg.select_path_ex(A0, B0, C0, M, N, K, tg.options(), need) == Path.RC
    for opts, b_copy in [(tg.options(b_layout=tg.B_NK), 0),                     # B N x K: rows of K, aligned
                         (tg.options(a_layout=tg.A_KM, ldb=1008), 0)]:          # A K x M (M % 8 == 0), B padded ld
        need = tg.workspace_size_ex(A0, B0, C0, M, N, K, opts)
        assert need == b_copy + up(2 * M * 1008), (opts.b_layout, opts.a_layout)
        assert tg.select_path_ex(A0, B0, C0, M, N, K, opts, need) == Path.REPACK
        # Without room for the padded C, describable operands keep the tensor-core kernels.
        if b_copy == 0:
            assert tg.select_path_ex(A0, B0, C0, M, N, K, opts, need - 1) in (Path.TC, Path.TC_PAIR, Path.TC_PAIR512)
    # 16-byte aligned rows of C (ldc a multiple of 8) need no copy of C.
    assert tg.workspace_size_ex(A0, B0, C0, M, N, K, tg.options(b_layout=tg.B_NK, ldc=1008)) == 0
    # Strided batches: one padded C serves every entry in turn.
    o = tg.options(b_layout=tg.B_NK, batch=3, stride_a=M * K, stride_b=N * K, stride_c=M * N + 3)
    assert tg.workspace_size_ex(A0, B0, C0, M, N, K, o) == up(2 * M * 1008)
    # Small M keeps the small-M kernel, which writes C element by element anyway; M = 200 with this
    # small B takes the tile kernels, which ask for the padded C.
    assert tg.workspace_size_ex(A0, B0, C0, 100, N, K, tg.options(b_layout=tg.B_NK)) == 0
    assert tg.workspace_size_ex(A0, B0, C0, 200, N, K, tg.options(b_layout=tg.B_NK)) == up(2 * 200 * 1008)


def test_workspace_argument_checks():
    M, N, K = 300, 301, 299
    need = tg.workspace_size(A0, B0, C0, M, N, K)
    W0 = 0x40_0000_0000
    assert tg.gemm_relu_f16_ws_raw(A0, B0, C0, M, N, K, 0, W0 + 16, need) == Status.INVALID_ARG   # not 256-aligned
    assert tg.gemm_relu_f16_ws_raw(A0, B0, C0, M, N, K, 0, A0, need) == Status.INVALID_ARG        # overlaps A
    assert tg.gemm_relu_f16_ws_raw(A0, B0, C0, M, N, K, 0, 0, 64) == Status.INVALID_ARG           # NULL with bytes
    assert tg.gemm_relu_f16_ws_raw(A0, B0, C0, M, N, K, 0, W0, -5) == Status.INVALID_ARG
    assert tg.gemm_relu_f16_raw(A0, B0, C0, M, N, K, 0, Path.REPACK) == Status.INVALID_ARG        # needs _ws


def test_extended_options_validation_and_paths():
    o = tg.options(b_layout=tg.B_NK)
    assert tg.select_path_ex(A0, B0, C0, 8192, 8192, 8192, o) == Path.TC_PAIR512
    assert tg.select_path_ex(A0, B0, C0, 64, 8192, 8192, o) == Path.SKINNY
    assert tg.select_path_ex(A0, B0, C0, 64, 8192, 8192, None) == Path.SKINNY
    # Strides below the row lengths, overlapping C entries, unknown layouts are refused.
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(ldc=100)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(lda=32)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(b_layout=tg.B_NK, ldb=32)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(b_layout=7)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(batch=2, stride_c=64 * 128 - 1)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(batch=2, stride_a=64 * 64, stride_b=64 * 128,
                                                                 stride_c=64 * 128)) == Path.SKINNY
    # Padded strides that are multiples of 8 keep TMA; others need the repack path.
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(lda=520, ldb=528, ldc=536)) == Path.TC_PAIR
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(lda=513)) == Path.RC
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(lda=513), 1 << 30) == Path.RC
    # B stored N x K with an odd K: only the repack path (the no-scratch kernels read B stored K x N).
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 511, tg.options(b_layout=tg.B_NK)) == Path.REPACK
    up = lambda x: (x + 255) // 256 * 256
    assert tg.workspace_size_ex(A0, B0, C0, 300, 200, 511, tg.options(b_layout=tg.B_NK)) == up(2 * 300 * 512) + up(2 * 200 * 512)
    assert tg.workspace_size_ex(A0, B0, C0, 300, 200, 512, tg.options(b_layout=tg.B_NK, ldb=515)) == up(2 * 200 * 512)
    # A forced path must be able to run the operands.
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(path=Path.TC_EDGE, b_layout=tg.B_NK)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(path=Path.TC)) == Path.TC
    # A stored K x M: the 128/256-row tensor-core kernels, never the small-M kernel or the edge mode.
    t = tg.options(a_layout=tg.A_KM)
    assert tg.select_path_ex(A0, B0, C0, 8192, 8192, 8192, t) == Path.TC_PAIR512
    assert tg.select_path_ex(A0, B0, C0, 64, 8192, 8192, t) in (Path.TC, Path.TC_PAIR)
    assert tg.select_path_ex(A0, B0, C0, 64, 8192, 8192, tg.options(a_layout=tg.A_KM, path=Path.SKINNY)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 512, 512, 512, tg.options(a_layout=tg.A_KM, path=Path.TC_EDGE)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 300, 128, 64, tg.options(a_layout=tg.A_KM, lda=299)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 300, 128, 64, tg.options(a_layout=2)) == Path.INVALID
    assert tg.select_path_ex(A0, B0, C0, 64, 128, 64, tg.options(reserved=1)) == Path.INVALID
    # An M that is not a multiple of 8 leaves K x M rows unaligned: repack into K x roundup(M, 8).
    assert tg.select_path_ex(A0, B0, C0, 300, 512, 512, t) == Path.REPACK     # the call then needs a workspace
    assert tg.gemm_relu_f16_ex_raw(A0, B0, C0, 300, 512, 512, t) == Status.INVALID_ARG
    assert tg.select_path_ex(A0, B0, C0, 304, 512, 512, t) in (Path.TC, Path.TC_PAIR)
    assert tg.workspace_size_ex(A0, B0, C0, 301, 512, 512, t) == up(2 * 512 * 304)
    assert tg.workspace_size_ex(A0, B0, C0, 304, 512, 512, t) == 0
    # A bias that overlaps C is refused.
    assert tg.gemm_relu_f16_ex_raw(A0, B0, C0, 64, 64, 64, tg.options(bias=C0 + 64)) == Status.INVALID_ARG


def test_mx_host_helpers_and_validation():
    assert tg.mx_grouped_rows([200, 0, 77, 128]) == 256 + 0 + 128 + 128
    assert tg.mx_grouped_rows([]) == 0
    assert tg.mx_grouped_rows([-1]) == -1
    assert tg.mx_grouped_rows([1] * 257) == -1
    assert tg.mx_scale_bytes(1, 32) == 128 * 4
    assert tg.mx_scale_bytes(300, 7168) == 384 * 224
    assert tg.mx_scale_bytes(300, 100) == -1
    P = 0x40_0000_0000
    ok = dict(A=P, SFA=P + (1 << 30), B=P + (2 << 30), SFB=P + (3 << 30), C=P + (4 << 30))

    def call(**kw):
        a = {**ok, **kw}
        return tg.gemm_mxf8_grouped_raw(a["A"], a["SFA"], a["B"], a["SFB"], a["C"], kw.get("m", [128]),
                                        kw.get("N", 256), kw.get("K", 256), kw.get("af", 0), kw.get("bf", 0))
    assert call(K=100) == Status.INVALID_ARG          # K not a multiple of 32
    assert call(N=100) == Status.INVALID_ARG          # N not a multiple of 8
    assert call(af=2) == Status.INVALID_ARG
    assert call(C=P + (4 << 30) + 8) == Status.INVALID_ARG   # C not 16-byte aligned
    assert call(SFA=0) == Status.INVALID_ARG
    assert call(C=P + 64) == Status.INVALID_ARG       # C overlaps A
    assert call(m=[-3]) == Status.INVALID_ARG
    assert call(m=[0, 0]) == Status.OK                # nothing to do: no launch
    assert call(N=0) == Status.OK


def test_mx_blocked_layout_formula():
    """The blocked scale layout is a permutation: every (row, block) lands on its own byte, and one
    128-row x 4-block atom fills 512 consecutive bytes (32 lines of 16)."""
    import numpy as np
    from tiled_dense_gemm_fp16_b200 import inputs
    R, S = 300, 10
    vals = (np.arange(R * S) % 251 + 1).astype(np.uint8).reshape(R, S)
    out = inputs.mx_scales_blocked(vals)
    assert out.size == tg.mx_scale_bytes(R, 32 * S) == 384 * 12
    assert np.count_nonzero(out) == R * S
    # Row 37 (line 5, quarter 1), block 6 (atom column 1, byte 2) of the first 128 rows.
    assert out[(0 * 3 + 1) * 512 + 5 * 16 + 1 * 4 + 2] == vals[37, 6]
    # Row 200 (second 128-row band): band 1, line 8, quarter 2, block 9 (atom column 2, byte 1).
    assert out[(1 * 3 + 2) * 512 + 8 * 16 + 2 * 4 + 1] == vals[200, 9]


def test_nvf4_host_validation():
    assert tg.nvf4_scale_bytes(300, 7168) == 384 * 448
    assert tg.nvf4_scale_bytes(1, 40) == -1
    P = 0x40_0000_0000

    def call(K=256, N=256, alpha=1.0, m=(128,), C=P + (4 << 30)):
        return tg.gemm_nvf4_grouped_raw(P, P + (1 << 30), P + (2 << 30), P + (3 << 30), C, list(m), N, K, alpha)
    assert call(K=96) == Status.INVALID_ARG           # K not a multiple of 64
    assert call(N=12) == Status.INVALID_ARG
    assert call(alpha=float("nan")) == Status.INVALID_ARG
    assert call(alpha=float("inf")) == Status.INVALID_ARG
    assert call(C=P + 32) == Status.INVALID_ARG       # C overlaps A
    assert call(m=(0,)) == Status.OK


def test_w4a16_host_validation():
    assert tg.w4a16_workspace_size(16, 8192, 8192, 128) == 0
    assert tg.w4a16_workspace_size(300, 256, 512, 128) == 2 * 256 * 512
    assert tg.w4a16_workspace_size(300, 256, 500, 128) == -1      # K % 64
    assert tg.w4a16_workspace_size(300, 256, 512, 48) == -1       # group not a multiple of 32
    assert tg.w4a16_workspace_size(300, 256, 768, 96) == -1       # group not a power of two
    assert tg.w4a16_workspace_size(300, 256, 512, 384) == -1      # group does not divide K
    P = 0x40_0000_0000

    def call(M=16, N=256, K=512, g=128, A=P, W=P + (1 << 30), S=P + (2 << 30), C=P + (3 << 30)):
        return tg.gemm_relu_w4a16_raw(A, W, S, C, M, N, K, g)
    assert call(K=96) == Status.INVALID_ARG
    assert call(g=16) == Status.INVALID_ARG
    assert call(A=P + 8) == Status.INVALID_ARG                    # A not 16-byte aligned
    assert call(S=P + (2 << 30) + 1) == Status.INVALID_ARG        # scales not 2-byte aligned
    assert call(C=P + 64) == Status.INVALID_ARG                   # C overlaps A
    assert call(M=0) == Status.OK
    assert tg.dequant_w4_f16_raw(P, P + (1 << 30), P + 32, 16, 256, 64) == Status.INVALID_ARG  # W overlaps Wq
