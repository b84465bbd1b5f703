"""Parity of the 4-bit weight-only GEMM (tg_gemm_relu_w4a16) and of the stand-alone
dequantization (tg_dequant_w4_f16) with the oracle.

The dequantized weight is compared bit for bit.  Integer activations with scales in
{0.5, 1, 2} give exact sums, compared bit for bit; other inputs within the fp16 GEMM
tolerance |gpu - oracle| <= 1e-3 + 4e-3 |oracle|."""
import numpy as np
import pytest

import oracle
from gpu_util import GUARD_BITS, assert_bitexact, assert_close, sample_rows
from tiled_dense_gemm_fp16_b200 import inputs

pytestmark = pytest.mark.gpu


def _dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("N,K", [(1, 128), (130, 512), (1024, 4096)])
def test_dequant_bitexact(N, K, group):
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    rng = np.random.default_rng(N + K + group)
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    # Scales over the whole fp16 range, subnormals and +-inf-producing ones included.
    S = rng.integers(0, 1 << 16, size=(N, K // group)).astype(np.uint16).view(np.float16)
    S[~np.isfinite(S)] = np.float16(1.0)
    Wq = inputs.pack_fp4(codes)
    W = torch.empty((N, K), dtype=torch.float16, device="cuda")
    Wq_d, S_d = _dev(Wq), _dev(S)  # held: the library call only sees raw pointers
    st = tg.dequant_w4_f16_raw(Wq_d.data_ptr(), S_d.data_ptr(), W.data_ptr(), N, K, group)
    assert st == tg.Status.OK
    torch.cuda.synchronize()
    want = oracle.dequant_w4_f16(Wq, S, N, K, group)
    assert np.array_equal(W.cpu().numpy().view(np.uint16), want.view(np.uint16))


def run_w4(M, N, K, group, dist, seed):
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A, Wq, S = inputs.w4_operands(M, N, K, group, seed, dist)
    G = 64
    cbuf = torch.full((M * N + 2 * G,), GUARD_BITS, dtype=torch.int16, device="cuda").view(torch.float16)
    C = cbuf[G:G + M * N].view(M, N)
    tg.gemm_relu_w4a16(_dev(A), _dev(Wq), _dev(S), group, out=C)
    torch.cuda.synchronize()
    status, word = tg.device_status()
    assert status == tg.Status.OK, hex(word)
    host = cbuf.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(host[:G] == GUARD_BITS) and np.all(host[G + M * N:] == GUARD_BITS)
    return host[G:G + M * N].view(np.float16).reshape(M, N), (A, Wq, S)


@pytest.mark.parametrize("M", [1, 5, 16, 64, 200, 256])
@pytest.mark.parametrize("N,K,group", [(128, 64, 64), (520, 1024, 32), (1000, 512, 128)])
def test_fused_integer_bitexact(M, N, K, group):
    got, (A, Wq, S) = run_w4(M, N, K, group, "int", seed=M + N + K)
    assert_bitexact(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 {(M, N, K, group)}")


@pytest.mark.parametrize("M,N,K,group", [(8, 4096, 4096, 128), (64, 1032, 2048, 64), (256, 384, 8192, 128)])
def test_fused_float(M, N, K, group):
    got, (A, Wq, S) = run_w4(M, N, K, group, "uniform", seed=M * 7 + K)
    assert_close(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 float {(M, N, K, group)}")


@pytest.mark.parametrize("M,N,K,group", [(257, 520, 512, 64), (1000, 264, 1024, 128)])
def test_large_m_dequantize_then_gemm(M, N, K, group):
    got, (A, Wq, S) = run_w4(M, N, K, group, "int", seed=M)
    assert_bitexact(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 large M {(M, N, K)}")


def test_large_m_needs_workspace():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M, N, K, g = 300, 256, 512, 128
    A = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    S = torch.ones((N, K // g), dtype=torch.float16, device="cuda")
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert tg.gemm_relu_w4a16_raw(A.data_ptr(), Wq.data_ptr(), S.data_ptr(), C.data_ptr(), M, N, K, g) == \
        tg.Status.INVALID_ARG
    assert tg.w4a16_workspace_size(M, N, K, g) == 2 * N * K


def test_k_zero_is_zero():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    C = torch.full((7, 24), 3.0, dtype=torch.float16, device="cuda")
    st = tg.gemm_relu_w4a16_raw(0, 0, 0, C.data_ptr(), 7, 24, 0, 32)
    assert st == tg.Status.OK
    torch.cuda.synchronize()
    assert np.all(C.cpu().numpy().view(np.uint16) == 0)


@pytest.mark.parametrize("name", list(inputs.W4_WORKLOADS))
def test_workloads_sampled_rows(name):
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M, N, K, group, seed = inputs.W4_WORKLOADS[name]
    A, Wq, S = inputs.w4_operands(M, N, K, group, seed, "uniform")
    C = tg.gemm_relu_w4a16(_dev(A), _dev(Wq), _dev(S), group)
    torch.cuda.synchronize()
    rows = sample_rows(M, n=16, seed=seed) if M > 16 else np.arange(M)
    want = oracle.gemm_relu_w4a16(np.ascontiguousarray(A[rows]), Wq, S, group)
    assert_close(C[torch.from_numpy(np.asarray(rows)).cuda()].cpu().numpy(), want, f"{name} rows")


# ---------------------------------------------------------------------------
# M <= 16 with K % 256 == 0 takes the decode kernel (register dequantization,
# warp-level MMAs, cluster split-K); the shapes below cover its splits of K
# (8 down to 1), ragged N, every scale group from 32 to K, and K that it does
# not take (K % 256 != 0, or slices longer than it holds), which falls back
# to the tcgen05 kernel.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 3, 16])
@pytest.mark.parametrize("N,K,group", [(130, 256, 32), (1000, 768, 128), (257, 3072, 1024), (640, 16384, 64),
                                       (520, 1280, 256), (130, 384, 128), (384, 32768, 256)])
def test_decode_integer_bitexact(M, N, K, group):
    import tiled_dense_gemm_fp16_b200 as tg
    want = tg.W4Kernel.DECODE if (K % 256 == 0 and K <= 16384) else tg.W4Kernel.FUSED
    assert tg.w4a16_kernel(M, N, K, group) == want
    got, (A, Wq, S) = run_w4(M, N, K, group, "int", seed=3 * M + N + K)
    assert_bitexact(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 decode {(M, N, K, group)}")


@pytest.mark.parametrize("M,N,K,group", [(16, 8192, 1024, 128), (7, 1536, 8192, 32)])
def test_decode_float(M, N, K, group):
    got, (A, Wq, S) = run_w4(M, N, K, group, "uniform", seed=M + 5 * K)
    assert_close(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 decode float {(M, N, K, group)}")


@pytest.mark.parametrize("M,N,K,group", [(1, 520, 1088, 64), (16, 1000, 576, 64), (9, 4096, 4160, 64),
                                         (4, 512, 16640, 128)])
def test_tcgen05_kernel_still_serves_small_m(M, N, K, group):
    # K not a multiple of 256, or K beyond the decode kernel's 16384: the tcgen05 fused kernel.
    import tiled_dense_gemm_fp16_b200 as tg
    assert tg.w4a16_kernel(M, N, K, group) == tg.W4Kernel.FUSED
    got, (A, Wq, S) = run_w4(M, N, K, group, "int", seed=M * 11 + K)
    assert_bitexact(got, oracle.gemm_relu_w4a16(A, Wq, S, group), f"W4A16 tcgen05 {(M, N, K, group)}")


def test_decode_deterministic():
    a, _ = run_w4(16, 2048, 8192, 128, "uniform", seed=77)
    b, _ = run_w4(16, 2048, 8192, 128, "uniform", seed=77)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
