"""Parity of the residue-class path (TG_PATH_RC: no scratch, any 2-byte
alignment) with the CPU oracle, through the C ABI.

The kernel loads A's rows in classes r mod 8 (rows of a class share one
16-byte offset) and shifts B's k-rows to match; B is realigned in shared
memory when TMA cannot describe it; C is written with aligned 16-byte stores
plus partial blocks at the ends of each row piece.  Few-tile shapes split K
over a cluster.  Integer-valued inputs are compared bit for bit, float inputs
within |gpu - oracle| <= 1e-3 + 4e-3 * |oracle|; guard bands around C catch
stray writes.
"""
import numpy as np
import pytest

import oracle
from gpu_util import GUARD, GUARD_BITS, assert_bitexact, assert_close, run_gpu
from tiled_dense_gemm_fp16_b200 import inputs
from tiled_dense_gemm_fp16_b200._binding import Path

pytestmark = pytest.mark.gpu

RC = Path.RC

SHAPES = [
    (1, 1, 8), (1, 8, 1), (3, 9, 8), (7, 17, 9), (8, 8, 8), (9, 129, 63), (15, 240, 64), (16, 241, 65),
    (17, 256, 127), (63, 257, 128), (127, 513, 199), (128, 255, 8), (129, 16, 1021), (200, 136, 72),
    (257, 777, 300), (300, 301, 299), (640, 520, 75), (1000, 1001, 1003), (1025, 129, 2049),
    (2000, 3000, 300),  # enough tiles for a full wave: 176-wide tiles (the width is chosen per wave count)
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_rc_integer_bitexact(M, N, K):
    A, B = inputs.operands(M, N, K, "int", seed=M * 5 + N * 3 + K)
    got, guards = run_gpu(A, B, RC)
    assert guards, (M, N, K)
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc {(M, N, K)}")


@pytest.mark.parametrize("M,N,K", [(1, 16, 3), (5, 64, 1), (100, 8, 7), (33, 520, 5), (40, 9, 3), (300, 257, 1)])
def test_rc_short_k(M, N, K):
    """K < 8: fewer k-rows than row classes, with B describable by TMA or realigned."""
    A, B = inputs.operands(M, N, K, "int", seed=K + N)
    got, guards = run_gpu(A, B, RC)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc short K {(M, N, K)}")


@pytest.mark.parametrize("offsets", [(1, 0, 0), (0, 3, 0), (0, 0, 5), (7, 6, 1), (2, 4, 6), (3, 3, 3)])
@pytest.mark.parametrize("M,N,K", [(131, 264, 200), (300, 257, 129), (77, 136, 1000), (2000, 72, 2048)])
def test_rc_unaligned_bases(offsets, M, N, K):
    """Bases 2, 4, ..., 14 bytes past a 16-byte boundary, per operand: every class shift of A and B.
    (2000, 72, 2048) takes 256-row tiles with K split over a cluster."""
    A, B = inputs.operands(M, N, K, "int", seed=sum(offsets) + M)
    got, guards = run_gpu(A, B, RC, offsets=offsets)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc offsets {offsets} {(M, N, K)}")


@pytest.mark.parametrize("M,N,K", [(1000, 129, 4099), (8191, 129, 1027), (300, 16, 5000), (50, 240, 3001),
                                   (2000, 200, 777), (129, 72, 20000), (2000, 72, 3001), (3000, 16, 4000)])
def test_rc_split_k_cluster(M, N, K):
    """One column of tiles and few rows of tiles: K split over a cluster, partials summed over DSMEM.
    (8191, 129, 1027), (2000, 72, 3001) and (3000, 16, 4000) take 256-row tiles (two accumulators)."""
    A, B = inputs.operands(M, N, K, "int", seed=M + N + K)
    got, guards = run_gpu(A, B, RC)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc split {(M, N, K)}")


@pytest.mark.parametrize("M,N,K,offsets", [
    (2000, 129, 16385, (0, 0, 0)),  # 256-row tiles, K split over a cluster, 32+ k-blocks per CTA
    (2000, 129, 16385, (5, 1, 3)),
    (8000, 601, 2100, (0, 0, 0)),   # a wave of 160-column tiles, 33 k-blocks each
    (8000, 601, 2100, (0, 3, 0)),
    (8191, 129, 8193, (0, 0, 0)),   # the small-N workload at full size
])
def test_rc_realign_two_blocks_in_flight(M, N, K, offsets):
    """B realigned in place with two k-blocks in flight: tiles narrower than 256 columns and K walks
    of 32 or more k-blocks per CTA."""
    A, B = inputs.operands(M, N, K, "int", seed=M + N + K + sum(offsets))
    got, guards = run_gpu(A, B, RC, offsets=offsets)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc two-deep {(M, N, K)} {offsets}")


@pytest.mark.parametrize("M,N,K", [(129, 257, 65), (1000, 1001, 1003), (2000, 129, 4099)])
def test_rc_uniform(M, N, K):
    A, B = inputs.operands(M, N, K, "uniform", seed=7 + K)
    got, guards = run_gpu(A, B, RC)
    assert guards
    assert_close(got, oracle.gemm_relu_f16(A, B), f"rc uniform {(M, N, K)}")


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (300, 264, 136), (129, 64, 8000)])
def test_rc_on_aligned_operands(M, N, K):
    """Everything aligned: one class, B loaded by TMA as it is."""
    A, B = inputs.operands(M, N, K, "int", seed=3)
    got, guards = run_gpu(A, B, RC)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc aligned {(M, N, K)}")


@pytest.mark.parametrize("M,N,K,a_off", [(64, 136, 77, 3), (200, 129, 1021, 1), (1000, 16, 5003, 7), (2000, 129, 1021, 5)])
def test_rc_infinities_do_not_leak_into_the_next_row(M, N, K, a_off):
    """The first k-block of a class holds, before k = 0, the previous row's last values (or the bytes
    just before A).  Those sit next to infinities here and NaN patterns fill the bytes before A; the
    kernel must clear them, so every row matches the oracle bit for bit."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A, B = inputs.operands(M, N, K, "int", seed=K)
    A = A.copy()
    A[::3, K - 7:] = np.float16(np.inf)       # rows 0, 3, 6, ...: infinite tails
    A[1::3, K - 1] = np.float16(-np.inf)
    B = B.copy()
    B[K - 7:, :] = 0                            # their products are NaN (0 * inf): rows with infinite tails give +0
    dev = torch.device("cuda", 0)
    abuf = torch.full((A.size + 16,), 0x7E01, dtype=torch.int16, device=dev).view(torch.float16)
    Ad = abuf[a_off:a_off + A.size].view(M, K)
    Ad.copy_(torch.from_numpy(A).to(dev))
    Bd = torch.from_numpy(B).to(dev)
    cbuf = torch.full((M * N + 2 * GUARD,), GUARD_BITS, dtype=torch.int16, device=dev).view(torch.float16)
    C = cbuf[GUARD:GUARD + M * N].view(M, N)
    st = tg.gemm_relu_f16_raw(Ad.data_ptr(), Bd.data_ptr(), C.data_ptr(), M, N, K,
                              torch.cuda.current_stream().cuda_stream, RC)
    assert st == tg.Status.OK, tg.status_string(st)
    torch.cuda.synchronize()
    status, word = tg.device_status()
    assert status == tg.Status.OK, hex(word)
    host = cbuf.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(host[:GUARD] == GUARD_BITS) and np.all(host[GUARD + M * N:] == GUARD_BITS)
    got = host[GUARD:GUARD + M * N].reshape(M, N).view(np.float16)
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"rc infinities {(M, N, K)}")


@pytest.mark.parametrize("bias", [False, True], ids=["nobias", "bias"])
@pytest.mark.parametrize("strides", ["odd", "padded8"])
@pytest.mark.parametrize("M,N,K", [(300, 264, 136), (517, 1000, 333), (1000, 129, 2000), (2000, 136, 2000)])
def test_rc_strides_bias_batches(M, N, K, strides, bias):
    from test_gpu_layouts import STRIDES, run_ex
    lda, ldb, ldc = STRIDES[strides](M, N, K, False)
    got, ref, guards = run_ex(M, N, K, lda=lda, ldb=ldb, ldc=ldc, b_nk=False, bias=bias, batch=2, gap=40,
                              seed=M + K, path=RC, workspace=False)
    assert guards
    for e, (g, r) in enumerate(zip(got, ref)):
        assert_bitexact(g, r, f"rc entry {e} {(M, N, K)} {strides} bias={bias}")


def test_rc_is_the_no_workspace_route_for_unaligned_rows():
    import tiled_dense_gemm_fp16_b200 as tg
    A0, B0, C0 = 0x10_0000_0000, 0x20_0000_0000, 0x30_0000_0000   # never dereferenced
    for (M, N, K) in [(3001, 5003, 1021), (777, 12289, 4095), (8191, 129, 8193), (100, 8, 7), (100, 9, 7)]:
        assert tg.select_path(A0, B0, C0, M, N, K) == RC
