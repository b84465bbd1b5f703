"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: bit-exact on integer-valued inputs (values in {-2..2}: every partial sum
is an integer below 2^24, so any summation order is exact), and
|gpu - oracle| <= 1e-3 + 4e-3 * |oracle| elementwise on float inputs.
Guard bands around C check that nothing outside C is written.
"""
import numpy as np
import pytest

import oracle
from gpu_util import assert_bitexact, assert_close, run_gpu, sample_rows
from tiled_dense_gemm_fp16_b200 import inputs
from tiled_dense_gemm_fp16_b200._binding import Path

pytestmark = pytest.mark.gpu

TC, EDGE, SKINNY, PAIR, WIDE = Path.TC, Path.TC_EDGE, Path.SKINNY, Path.TC_PAIR, Path.TC_PAIR512


def _paths_for(M, N, K):
    paths = [None, EDGE]
    if N % 8 == 0 and K % 8 == 0:
        paths += [TC, PAIR, WIDE]
        if M <= 256:
            paths.append(SKINNY)
    return paths


@pytest.mark.parametrize("path,N", [(PAIR, 256), (WIDE, 512)], ids=["pair256", "pair512"])
def test_pair_kernel_single_tile(path, N):
    """One tile on one SM pair, one 64-deep k-block: the smallest cta_group::2 case."""
    A, B = inputs.operands(256, N, 64, "int", seed=12)
    got, guards = run_gpu(A, B, path)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"pair 256x{N}x64")


# ---------------------------------------------------------------------------
# Small square workload (256^3): integer variant bit-exact, uniform within tolerance
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", [None, TC, EDGE, PAIR, WIDE], ids=["auto", "tc", "edge", "pair", "wide"])
def test_square256_integer_bitexact(path):
    A, B = inputs.operands(256, 256, 256, "int", seed=0)
    got, guards = run_gpu(A, B, path)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), "square256 int")


@pytest.mark.parametrize("path", [None, TC, EDGE, PAIR, WIDE], ids=["auto", "tc", "edge", "pair", "wide"])
def test_square256_uniform(path):
    (shape, A, B), = inputs.WORKLOADS["square256"].problems()
    got, guards = run_gpu(A, B, path)
    assert guards
    assert_close(got, oracle.gemm_relu_f16(A, B), "square256 uniform")


# ---------------------------------------------------------------------------
# Tile edges: sizes around the 128 x 256 x 64 tile, bit-exact on integer inputs
# ---------------------------------------------------------------------------

EDGE_SHAPES = [
    (1, 1, 1), (1, 8, 8), (15, 17, 9), (16, 16, 16), (17, 33, 65), (127, 255, 63),
    (128, 256, 64), (129, 257, 65), (255, 129, 127), (257, 513, 200), (300, 264, 136),
    (128, 8, 1000), (8, 1000, 24), (640, 520, 72), (1000, 1000, 1000),
]


@pytest.mark.parametrize("M,N,K", EDGE_SHAPES)
def test_tile_edges_integer_bitexact(M, N, K):
    A, B = inputs.operands(M, N, K, "int", seed=M * 7 + N * 3 + K)
    ref = oracle.gemm_relu_f16(A, B)
    for path in _paths_for(M, N, K):
        got, guards = run_gpu(A, B, path)
        assert guards, (M, N, K, path)
        assert_bitexact(got, ref, f"{(M, N, K)} path={path}")


@pytest.mark.parametrize("M,N,K", [(129, 257, 65), (300, 264, 136), (1000, 1000, 1000)])
def test_tile_edges_uniform(M, N, K):
    A, B = inputs.operands(M, N, K, "uniform", seed=5)
    ref = oracle.gemm_relu_f16(A, B)
    for path in _paths_for(M, N, K):
        got, guards = run_gpu(A, B, path)
        assert guards
        assert_close(got, ref, f"{(M, N, K)} path={path}")


SKINNY_SHAPES = [
    (1, 8, 8), (1, 136, 72), (2, 1024, 1000), (7, 520, 4096), (8, 128, 64), (15, 264, 136),
    (16, 8192, 512), (17, 1000, 200), (31, 128, 8), (64, 520, 1000), (100, 2048, 2048),
    (128, 136, 4104), (129, 256, 64), (200, 1024, 312), (255, 392, 1000), (256, 8192, 256),
]


@pytest.mark.parametrize("M,N,K", SKINNY_SHAPES)
def test_skinny_integer_bitexact(M, N, K):
    """Small M: panels of 128 columns, split K, cluster reduction; partial panels and short K."""
    A, B = inputs.operands(M, N, K, "int", seed=M + 11 * N + K)
    ref = oracle.gemm_relu_f16(A, B)
    got, guards = run_gpu(A, B, SKINNY)
    assert guards, (M, N, K)
    assert_bitexact(got, ref, f"skinny {(M, N, K)}")


@pytest.mark.parametrize("M,N,K", [(1, 8192, 8192), (16, 1024, 4096), (64, 8192, 1024), (256, 520, 2048)])
def test_skinny_uniform(M, N, K):
    A, B = inputs.operands(M, N, K, "uniform", seed=M + N + K)
    ref = oracle.gemm_relu_f16(A, B)
    got, guards = run_gpu(A, B, SKINNY)
    assert guards
    assert_close(got, ref, f"skinny {(M, N, K)}")


@pytest.mark.parametrize("offset", [1, 2, 3, 5, 7])
@pytest.mark.parametrize("M,N,K", [(200, 136, 72), (131, 257, 199)])
def test_misaligned_base_pointers_use_edge_mode(offset, M, N, K):
    """Bases 2*offset bytes off a 16-byte boundary: TMA cannot take them; the
    edge mode realigns rows from aligned 16-byte loads (every shift 2..14 B)."""
    A, B = inputs.operands(M, N, K, "int", seed=2 + offset)
    ref = oracle.gemm_relu_f16(A, B)
    got, guards = run_gpu(A, B, None, offset_elems=offset)
    assert guards
    assert_bitexact(got, ref, f"offset {offset}")


# ---------------------------------------------------------------------------
# Repack path (caller workspace) and unaligned C on the TMA kernels
# ---------------------------------------------------------------------------

REPACK_SHAPES = [(1, 9, 7), (15, 17, 9), (129, 257, 65), (255, 129, 127), (300, 301, 299),
                 (640, 520, 75), (1000, 1001, 1003), (16, 8191, 517), (257, 777, 1021),
                 (200, 6001, 6001), (300, 8191, 5003), (129, 4999, 8193)]


@pytest.mark.parametrize("M,N,K", REPACK_SHAPES)
def test_repack_integer_bitexact(M, N, K):
    """Odd row lengths with a workspace: the residue-class kernel on a padded copy of B, or, for large N
    and K (1/N + 1/K <= 1/2400), A and B copied into zero-padded rows around the CTA-pair kernel with a
    padded C copied back."""
    import tiled_dense_gemm_fp16_b200 as tg
    A, B = inputs.operands(M, N, K, "int", seed=M + 3 * N + 5 * K)
    want = Path.REPACK if 2400 * (N + K) <= N * K else Path.RC
    assert tg.select_path_ws(1 << 12, 1 << 40, 1 << 41, M, N, K, 1 << 40) == want
    got, guards = run_gpu(A, B, workspace=True)
    assert guards, (M, N, K)
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"workspace route {(M, N, K)}")


@pytest.mark.parametrize("offsets", [(1, 0, 0), (0, 3, 0), (0, 0, 5), (7, 2, 1), (0, 0, 4)])
def test_unaligned_bases(offsets):
    """Misaligned A or B go through the repack path; a misaligned C alone keeps the TMA kernels without a
    workspace and, with one, has the GEMM write a padded C that a realigning copy moves into place."""
    for (M, N, K) in [(300, 264, 136), (64, 520, 72)]:
        A, B = inputs.operands(M, N, K, "int", seed=sum(offsets) + M)
        ref = oracle.gemm_relu_f16(A, B)
        for ws in (False, True):
            got, guards = run_gpu(A, B, offsets=offsets, workspace=ws)
            assert guards, (offsets, M, N, K, ws)
            assert_bitexact(got, ref, f"offsets {offsets} {(M, N, K)} ws={ws}")


@pytest.mark.parametrize("c_off", [1, 2, 3, 7])
@pytest.mark.parametrize("M,N,K", [(520, 1032, 264), (777, 1001, 136), (300, 8, 64), (1100, 2053, 512)])
def test_padded_c_copy_back(M, N, K, c_off):
    """C's rows not 16-byte aligned, with a workspace: the GEMM writes a padded C and the realigning copy
    writes every element of C (interior 16-byte blocks and the ragged ends of each row) and nothing else."""
    import tiled_dense_gemm_fp16_b200 as tg
    A, B = inputs.operands(M, N, K, "int", seed=M + N + c_off)
    # K % 8 == 0 keeps A and B TMA-describable when N % 8 == 0, so only C is copied.
    if K % 8 == 0 and N % 8 == 0:
        assert tg.select_path_ws(16, 1 << 40, (1 << 41) + 2 * c_off, M, N, K, 1 << 40) == Path.REPACK
    got, guards = run_gpu(A, B, offsets=(0, 0, c_off), workspace=True)
    assert guards, (M, N, K, c_off)
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), f"padded C {(M, N, K)} offset {c_off}")


@pytest.mark.parametrize("M,N,K", [(300, 301, 299), (1000, 1001, 1003)])
def test_repack_uniform(M, N, K):
    A, B = inputs.operands(M, N, K, "uniform", seed=17)
    got, guards = run_gpu(A, B, workspace=True)
    assert guards
    assert_close(got, oracle.gemm_relu_f16(A, B), f"repack uniform {(M, N, K)}")


def test_torch_api_allocates_workspace_itself():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A, B = inputs.operands(257, 259, 261, "int", seed=4)
    Ad, Bd = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    C1 = tg.gemm_relu(Ad, Bd)                  # B copied into a torch-allocated workspace
    C2 = tg.gemm_relu(Ad, Bd, workspace=None)  # no workspace
    torch.cuda.synchronize()
    ref = oracle.gemm_relu_f16(A, B)
    assert_bitexact(C1.cpu().numpy(), ref, "torch api with workspace")
    assert_bitexact(C2.cpu().numpy(), ref, "torch api without workspace")


def test_random_shapes_fuzz():
    """Random sizes (aligned and not) through the default path and the workspace path, bit for bit."""
    rng = np.random.default_rng(2024)
    for i in range(40):
        M, N, K = (int(x) for x in rng.integers(1, 1200, size=3))
        if i % 4 == 0:  # every fourth shape with 16-byte row strides
            N, K = (N + 7) // 8 * 8, (K + 7) // 8 * 8
        A, B = inputs.operands(M, N, K, "int", seed=5000 + i)
        ref = oracle.gemm_relu_f16(A, B)
        for ws in (False, True):
            got, guards = run_gpu(A, B, workspace=ws)
            assert guards, (M, N, K, ws)
            assert_bitexact(got, ref, f"fuzz {(M, N, K)} ws={ws}")


def test_back_to_back_calls_on_one_stream():
    """Consecutive dependent launches (a call's output feeds the next) stay ordered."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M = 512
    A, B = inputs.operands(M, M, M, "int", seed=77)
    Ad, Bd = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    ones = torch.ones((M, M), dtype=torch.float16, device="cuda") / 64
    C1 = tg.gemm_relu(Ad, Bd)
    C2 = tg.gemm_relu(C1, ones)          # reads C1 right after the kernel that writes it
    C3 = tg.gemm_relu(C2, ones)
    torch.cuda.synchronize()
    r1 = oracle.gemm_relu_f16(A, B)
    r2 = oracle.gemm_relu_f16(r1, np.full((M, M), 1 / 64, np.float16))
    r3 = oracle.gemm_relu_f16(r2, np.full((M, M), 1 / 64, np.float16))
    assert_bitexact(C1.cpu().numpy(), r1, "first")
    assert_close(C2.cpu().numpy(), r2, "second")
    assert_close(C3.cpu().numpy(), r3, "third")


# ---------------------------------------------------------------------------
# Degenerate sizes
# ---------------------------------------------------------------------------

def test_k_zero_fills_positive_zero():
    A = np.zeros((37, 0), np.float16)
    B = np.zeros((0, 53), np.float16)
    got, guards = run_gpu(A, B)
    assert guards
    assert np.all(got.view(np.uint16) == 0)


def test_empty_outputs_are_noops():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    A = torch.zeros((0, 16), dtype=torch.float16, device="cuda")
    B = torch.zeros((16, 8), dtype=torch.float16, device="cuda")
    assert tg.gemm_relu(A, B).shape == (0, 8)
    A = torch.zeros((8, 16), dtype=torch.float16, device="cuda")
    B = torch.zeros((16, 0), dtype=torch.float16, device="cuda")
    assert tg.gemm_relu(A, B).shape == (8, 0)


def test_special_values():
    """Overflow to +inf past 65504, and ReLU of all-negative tiles to +0."""
    K = 16384
    A = np.full((130, K), 2.0, np.float16)
    B = np.full((K, 264), 2.0, np.float16)       # 4K = 65536 -> +inf
    B[:, 8:16] = -2.0                             # -65536 -> ReLU -> +0
    B[:4095, 16:24] = 0.0                         # 4 * 12289 = 49156 -> 49152 (nearest even half)
    ref = oracle.gemm_relu_f16(A, B)
    for path in (TC, EDGE, PAIR, WIDE):
        got, _ = run_gpu(A, B, path)
        assert_bitexact(got, ref, f"special path={path}")
    assert np.all(np.isinf(ref[:, :8].astype(np.float32))) and np.all(ref[:, 8:16].view(np.uint16) == 0)


def test_deterministic():
    A, B = inputs.operands(513, 777, 300, "uniform", seed=9)
    a, _ = run_gpu(A, B)
    b, _ = run_gpu(A, B)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_non_default_stream():
    import torch
    A, B = inputs.operands(256, 512, 128, "int", seed=3)
    s = torch.cuda.Stream()
    got, _ = run_gpu(A, B, stream=s)
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), "side stream")


# ---------------------------------------------------------------------------
# The five workloads at full size (sampled rows where the full oracle is slow)
# ---------------------------------------------------------------------------

def _check_workload(name, dist=None, exact=False, full_oracle_max_macs=5e9, paths=(None,)):
    for (M, N, K), A, B in inputs.WORKLOADS[name].problems(dist):
        full = M * N * K <= full_oracle_max_macs
        rows = list(range(M)) if full else sample_rows(M, seed=M + N + K)
        ref = oracle.gemm_relu_f16_rows(A, B, rows)
        for path in paths:
            if path == "ws":
                got, guards = run_gpu(A, B, workspace=True)
            else:
                got, guards = run_gpu(A, B, path)
            assert guards, (name, M, N, K, path)
            sub = got[rows]
            what = f"{name} {(M, N, K)} path={path} dist={dist or inputs.WORKLOADS[name].dist}"
            if exact:
                assert_bitexact(sub, ref, what)
            else:
                assert_close(sub, ref, what)


def test_workload_square4096():
    _check_workload("square4096", paths=(None, TC, PAIR, EDGE))


def test_workload_square4096_integer():
    _check_workload("square4096", dist="int", exact=True, paths=(None, TC, PAIR))


def test_workload_square8192():
    _check_workload("square8192", paths=(None, TC, PAIR))


def test_workload_square8192_integer():
    _check_workload("square8192", dist="int", exact=True, paths=(None, TC, PAIR))


def test_workload_skinny():
    _check_workload("skinny", paths=(None, SKINNY, TC, EDGE))


def test_workload_skinny_integer():
    _check_workload("skinny", dist="int", exact=True, paths=(None, SKINNY, TC, EDGE))


def test_workload_ragged():
    _check_workload("ragged", paths=(None, "ws"))


def test_workload_ragged_integer():
    _check_workload("ragged", dist="int", exact=True, paths=(None, "ws"))


# ---------------------------------------------------------------------------
# Large indices: more than 2^31 elements in A (64-bit address arithmetic)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K", [32776, 32775], ids=["aligned", "odd_K"])
def test_more_than_2_31_elements(K):
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M, N = 65544, 136
    assert M * K > 2**31
    rng = np.random.default_rng(K)
    dev = torch.device("cuda", 0)
    # Only the checked rows carry seeded random values; every other row of A
    # is all ones, and one of those rows is checked too.
    rows = [0, 1, 127, 128, M // 2, M - 129, M - 2, M - 1]
    A_rows = rng.integers(-2, 3, size=(len(rows), K)).astype(np.float16)
    B = rng.integers(-2, 3, size=(K, N)).astype(np.float16)
    Ad = torch.ones((M, K), dtype=torch.float16, device=dev)
    for r, a in zip(rows, A_rows):
        Ad[r].copy_(torch.from_numpy(a))
    Bd = torch.from_numpy(B).to(dev)
    C = tg.gemm_relu(Ad, Bd)
    torch.cuda.synchronize()
    got = C[rows].cpu().numpy()
    assert_bitexact(got, oracle.gemm_relu_f16(A_rows, B), f"M*K > 2^31, K={K}")
    # An all-ones row: C = ReLU(column sums of B).
    ones_row = C[2].cpu().numpy()
    ref_ones = oracle.gemm_relu_f16(np.ones((1, K), np.float16), B)[0]
    assert_bitexact(ones_row, ref_ones, "all-ones row")
    del Ad, Bd, C
    torch.cuda.empty_cache()
