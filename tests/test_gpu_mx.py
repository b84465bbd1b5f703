"""Parity of the MXFP8 block-scaled grouped GEMM (tg_gemm_mxf8_grouped) with the oracle.

Integer-valued operands with unit scales give exact sums, so those outputs are
compared bit for bit.  Other inputs are compared within
  |gpu - oracle| <= 2^-7 |oracle| + 2^-20 sum_k |a sa| |b sb|:
one bf16 rounding step on each side (the GPU rounds its fp32 sum, the oracle
the near-exact sum: at most one bf16 unit apart, 2^-7 relative) plus the fp32
accumulation error of the tensor core, bounded far above K * 2^-24 relative to
the sum of magnitudes."""
import numpy as np
import pytest

import oracle
from gpu_util import GUARD_BITS
from mx_util import abs_dot, bf16_to_f64, oracle_rows, to_blocked, to_blocked_groups
from tiled_dense_gemm_fp16_b200 import inputs

pytestmark = pytest.mark.gpu


def run_mx(m_sizes, N, K, *, dist="int", seed=0, a_format=0, b_format=0, relu=False, scale_lo=124, scale_hi=131):
    """Run the GPU kernel; returns (C bits (rows x N) with guard rows intact, inputs)."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A, SFA, B, SFB = inputs.mx_operands(m_sizes, N, K, seed, dist, a_format, b_format, scale_lo, scale_hi)
    rows = A.shape[0]
    assert rows == tg.mx_grouped_rows(m_sizes)
    dev = torch.device("cuda", 0)
    Ad = torch.from_numpy(A).to(dev)
    Bd = torch.from_numpy(B).to(dev)
    SFAd = torch.from_numpy(to_blocked(SFA)).to(dev)
    SFBd = torch.from_numpy(to_blocked_groups(SFB)).to(dev)
    assert SFAd.numel() == tg.mx_scale_bytes(rows, K)
    assert SFBd.numel() == len(m_sizes) * tg.mx_scale_bytes(N, K)
    C = torch.full((rows, N), GUARD_BITS, dtype=torch.int16, device=dev).view(torch.bfloat16)
    tg.mxf8_grouped(Ad, SFAd, Bd, SFBd, list(m_sizes), relu=relu, a_format=a_format, b_format=b_format, out=C)
    torch.cuda.synchronize()
    status, word = tg.device_status()
    assert status == tg.Status.OK, hex(word)
    got = C.view(torch.int16).cpu().numpy().view(np.uint16)
    return got, (A, SFA, B, SFB)


def check_rows(got, ops, m_sizes, N, K, *, a_format=0, b_format=0, relu=False, exact=False, sample=None):
    A, SFA, B, SFB = ops
    offs, rows = inputs.mx_group_offsets(m_sizes)
    covered = np.zeros(rows, bool)
    for g, (o, m) in enumerate(zip(offs, m_sizes)):
        covered[o:o + m] = True
        if m == 0:
            continue
        rr = np.arange(o, o + m) if sample is None else np.unique(
            np.concatenate([[o, o + m - 1], o + np.random.default_rng(g).integers(0, m, size=sample)]))
        want = oracle_rows(A, SFA, B, SFB, g, rr, N, K, a_format, b_format, relu)
        have = got[rr]
        if exact:
            assert np.array_equal(have, want), f"group {g}: {np.argwhere(have != want)[:5]}"
        else:
            w, h = bf16_to_f64(want), bf16_to_f64(have)
            assert np.array_equal(np.isnan(w), np.isnan(h)), f"group {g}: NaN positions differ"
            tol = 2.0 ** -7 * np.abs(w) + 2.0 ** -20 * abs_dot(A, SFA, B, SFB, g, rr, N, K, a_format, b_format)
            ok = np.isnan(w) | (np.abs(h - w) <= tol)
            assert ok.all(), f"group {g}: max excess {np.max(np.abs(h - w) - tol)} at {np.argwhere(~ok)[:3]}"
    assert np.all(got[~covered] == GUARD_BITS), "a row outside every group was written"


@pytest.mark.parametrize("relu", [False, True], ids=["plain", "relu"])
@pytest.mark.parametrize("m_sizes,N,K", [
    ((128,), 256, 128),
    ((200, 0, 77, 128), 512, 256),
    ((1, 129, 255), 264, 160),
    ((300,), 136, 96),
    ((64, 64, 64, 64, 64, 64, 64, 64, 64, 64, 64, 3), 384, 384),
], ids=["one_tile", "ragged_groups", "ragged_nk", "n136_k96", "twelve_groups"])
def test_integer_bitexact(m_sizes, N, K, relu):
    got, ops = run_mx(m_sizes, N, K, dist="int", seed=len(m_sizes) + N, relu=relu)
    check_rows(got, ops, m_sizes, N, K, relu=relu, exact=True)


@pytest.mark.parametrize("a_format,b_format", [(0, 0), (1, 1), (1, 0), (0, 1)],
                         ids=["e4m3", "e5m2", "e5m2_e4m3", "e4m3_e5m2"])
def test_formats_integer_bitexact(a_format, b_format):
    m_sizes, N, K = (150, 90), 256, 256
    got, ops = run_mx(m_sizes, N, K, dist="int", seed=3, a_format=a_format, b_format=b_format)
    check_rows(got, ops, m_sizes, N, K, a_format=a_format, b_format=b_format, exact=True)


@pytest.mark.parametrize("a_format,b_format", [(0, 0), (1, 1), (0, 1)], ids=["e4m3", "e5m2", "mixed"])
@pytest.mark.parametrize("relu", [False, True], ids=["plain", "relu"])
def test_normal_values_with_scales(a_format, b_format, relu):
    m_sizes, N, K = (333, 128, 45), 520, 1024
    got, ops = run_mx(m_sizes, N, K, dist="normal", seed=11 + a_format, a_format=a_format, b_format=b_format,
                      relu=relu)
    check_rows(got, ops, m_sizes, N, K, a_format=a_format, b_format=b_format, relu=relu)


def test_wide_scale_range():
    """Scales spread over 2^-20 .. 2^20: the block scaling, not the values, sets the magnitudes."""
    m_sizes, N, K = (256,), 256, 512
    got, ops = run_mx(m_sizes, N, K, dist="normal", seed=21, scale_lo=107, scale_hi=148)
    check_rows(got, ops, m_sizes, N, K)


def test_k_zero_writes_zero_rows():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    m_sizes, N = (5, 130), 64
    rows = tg.mx_grouped_rows(m_sizes)
    C = torch.full((rows, N), GUARD_BITS, dtype=torch.int16, device="cuda")
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = tg.gemm_mxf8_grouped_raw(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                  C.data_ptr(), m_sizes, N, 0)
    assert st == tg.Status.OK
    got = C.cpu().numpy().view(np.uint16)
    offs, _ = inputs.mx_group_offsets(m_sizes)
    mask = np.zeros(rows, bool)
    for o, m in zip(offs, m_sizes):
        mask[o:o + m] = True
    assert np.all(got[mask] == 0) and np.all(got[~mask] == GUARD_BITS)


def test_nan_scale_propagates():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    m_sizes, N, K = (128,), 256, 128
    A, SFA, B, SFB = inputs.mx_operands(m_sizes, N, K, 4, "int")
    SFA[7, 2] = 255
    C = tg.mxf8_grouped(torch.from_numpy(A).cuda(), torch.from_numpy(to_blocked(SFA)).cuda(), torch.from_numpy(B).cuda(),
                        torch.from_numpy(to_blocked_groups(SFB)).cuda(), list(m_sizes))
    got = C.view(torch.int16).cpu().numpy().view(np.uint16)
    want = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, [0], N, K)
    w, h = bf16_to_f64(want), bf16_to_f64(got)
    assert np.isnan(h[7]).all() and np.isnan(w[7]).all()
    assert np.array_equal(np.delete(got, 7, axis=0), np.delete(want, 7, axis=0))


@pytest.mark.parametrize("name", list(inputs.MX_WORKLOADS))
def test_workloads_sampled_rows(name):
    """The benchmark's MXFP8 workloads at full size, sampled rows of every group."""
    m_sizes, N, K, seed = inputs.MX_WORKLOADS[name]
    got, ops = run_mx(m_sizes, N, K, dist="normal", seed=seed)
    check_rows(got, ops, m_sizes, N, K, sample=6)


@pytest.mark.parametrize("m_sizes,N,K", [
    ((128,), 256, 128),
    ((200, 0, 77, 128), 512, 256),
    ((1, 129, 255, 384), 264, 160),
    ((64,) * 11 + (3,), 384, 384),
], ids=["one_tile", "ragged_groups", "odd_tile_counts", "twelve_groups"])
def test_kernel_integer_bitexact(m_sizes, N, K):
    """Groups with an odd number of 128-row tiles, an empty group, and a last group that ends the
    stacked rows."""
    got, ops = run_mx(m_sizes, N, K, dist="int", seed=len(m_sizes) + 2 * N, relu=True)
    check_rows(got, ops, m_sizes, N, K, relu=True, exact=True)


def test_kernel_normal_values():
    m_sizes, N, K = (333, 128, 45), 520, 1024
    got, ops = run_mx(m_sizes, N, K, dist="normal", seed=31, a_format=1, b_format=0)
    check_rows(got, ops, m_sizes, N, K, a_format=1, b_format=0)
