"""Parity of the NVF4 block-scaled grouped GEMM (tg_gemm_nvf4_grouped) with the oracle.

Integer-valued E2M1 operands with unit scales (and alpha a power of two) give
exact sums and are compared bit for bit.  Other inputs are compared within
  |gpu - oracle| <= 2^-7 |oracle| + 2^-20 |alpha| sum_k |a sa| |b sb|
(one bf16 step between the GPU's rounding of alpha * (fp32 sum) and the
oracle's single rounding, plus the fp32 accumulation error)."""
import numpy as np
import pytest

from gpu_util import GUARD_BITS
from mx_util import bf16_to_f64, nvf4_abs_dot, nvf4_oracle_rows
from tiled_dense_gemm_fp16_b200 import inputs

pytestmark = pytest.mark.gpu


def run_nvf4(m_sizes, N, K, *, dist="int", seed=0, alpha=1.0, relu=False):
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A, SFA, B, SFB = inputs.nvf4_operands(m_sizes, N, K, seed, dist)
    rows = A.shape[0]
    dev = torch.device("cuda", 0)
    sfa_b, sfb_b = inputs.mx_scales_blocked(SFA), inputs.mx_scales_blocked(SFB)
    assert sfa_b.size == tg.nvf4_scale_bytes(rows, K) and sfb_b.size == len(m_sizes) * tg.nvf4_scale_bytes(N, K)
    C = torch.full((rows, N), GUARD_BITS, dtype=torch.int16, device=dev).view(torch.bfloat16)
    tg.nvf4_grouped(torch.from_numpy(A).to(dev), torch.from_numpy(sfa_b).to(dev), torch.from_numpy(B).to(dev),
                    torch.from_numpy(sfb_b).to(dev), list(m_sizes), alpha=alpha, relu=relu, out=C)
    torch.cuda.synchronize()
    status, word = tg.device_status()
    assert status == tg.Status.OK, hex(word)
    return C.view(torch.int16).cpu().numpy().view(np.uint16), (A, SFA, B, SFB)


def check(got, ops, m_sizes, N, K, *, alpha=1.0, relu=False, exact=False, sample=None):
    A, SFA, B, SFB = ops
    offs, rows = inputs.mx_group_offsets(m_sizes)
    covered = np.zeros(rows, bool)
    for g, (o, m) in enumerate(zip(offs, m_sizes)):
        covered[o:o + m] = True
        if m == 0:
            continue
        rr = np.arange(o, o + m) if sample is None else np.unique(
            np.concatenate([[o, o + m - 1], o + np.random.default_rng(g).integers(0, m, size=sample)]))
        want = nvf4_oracle_rows(A, SFA, B, SFB, g, rr, N, K, alpha, relu)
        have = got[rr]
        if exact:
            assert np.array_equal(have, want), f"group {g}: {np.argwhere(have != want)[:5]}"
        else:
            w, h = bf16_to_f64(want), bf16_to_f64(have)
            tol = 2.0 ** -7 * np.abs(w) + 2.0 ** -20 * abs(alpha) * nvf4_abs_dot(A, SFA, B, SFB, g, rr, N, K)
            ok = np.abs(h - w) <= tol
            assert ok.all(), f"group {g}: max excess {np.max(np.abs(h - w) - tol)} at {np.argwhere(~ok)[:3]}"
    assert np.all(got[~covered] == GUARD_BITS), "a row outside every group was written"


@pytest.mark.parametrize("relu", [False, True], ids=["plain", "relu"])
@pytest.mark.parametrize("m_sizes,N,K", [
    ((128,), 256, 256),
    ((200, 0, 77, 128), 512, 512),
    ((1, 129, 255), 264, 192),
    ((300,), 136, 64),
    ((64,) * 11 + (3,), 384, 320),
], ids=["one_tile", "ragged_groups", "ragged_nk", "n136_k64", "twelve_groups"])
def test_integer_bitexact(m_sizes, N, K, relu):
    got, ops = run_nvf4(m_sizes, N, K, dist="int", seed=len(m_sizes) + N, relu=relu)
    check(got, ops, m_sizes, N, K, relu=relu, exact=True)


def test_alpha_power_of_two_bitexact():
    m_sizes, N, K = (150, 90), 256, 512
    got, ops = run_nvf4(m_sizes, N, K, dist="int", seed=3, alpha=0.25)
    check(got, ops, m_sizes, N, K, alpha=0.25, exact=True)


@pytest.mark.parametrize("alpha", [1.0, 0.37, -2.5], ids=["one", "fraction", "negative"])
@pytest.mark.parametrize("relu", [False, True], ids=["plain", "relu"])
def test_all_codes_with_scales(alpha, relu):
    m_sizes, N, K = (333, 128, 45), 520, 1024
    got, ops = run_nvf4(m_sizes, N, K, dist="codes", seed=11, alpha=alpha, relu=relu)
    check(got, ops, m_sizes, N, K, alpha=alpha, relu=relu)


def test_k_zero_writes_zero_rows():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    m_sizes, N = (5, 130), 64
    rows = tg.mx_grouped_rows(m_sizes)
    C = torch.full((rows, N), GUARD_BITS, dtype=torch.int16, device="cuda")
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = tg.gemm_nvf4_grouped_raw(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                  C.data_ptr(), m_sizes, N, 0)
    assert st == tg.Status.OK
    got = C.cpu().numpy().view(np.uint16)
    offs, _ = inputs.mx_group_offsets(m_sizes)
    mask = np.zeros(rows, bool)
    for o, m in zip(offs, m_sizes):
        mask[o:o + m] = True
    assert np.all(got[mask] == 0) and np.all(got[~mask] == GUARD_BITS)


@pytest.mark.parametrize("name", list(inputs.NVF4_WORKLOADS))
def test_workloads_sampled_rows(name):
    m_sizes, N, K, seed = inputs.NVF4_WORKLOADS[name]
    got, ops = run_nvf4(m_sizes, N, K, dist="codes", seed=seed)
    check(got, ops, m_sizes, N, K, sample=6)


@pytest.mark.parametrize("m_sizes,N,K", [
    ((128,), 256, 256),
    ((200, 0, 77, 128), 512, 512),
    ((1, 129, 255, 384), 264, 192),
    ((64,) * 11 + (3,), 384, 320),
], ids=["one_tile", "ragged_groups", "odd_tile_counts", "twelve_groups"])
def test_kernel_integer_bitexact(m_sizes, N, K):
    """Groups with an odd number of 128-row tiles, an empty group, and a last group that ends the
    stacked rows."""
    got, ops = run_nvf4(m_sizes, N, K, dist="int", seed=len(m_sizes) + 2 * N, relu=True)
    check(got, ops, m_sizes, N, K, relu=True, exact=True)


def test_kernel_all_codes():
    m_sizes, N, K = (333, 128, 45), 520, 1024
    got, ops = run_nvf4(m_sizes, N, K, dist="codes", seed=33, alpha=0.37)
    check(got, ops, m_sizes, N, K, alpha=0.37)
