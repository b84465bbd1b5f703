"""Parity of the general-layout entry point tg_gemm_relu_f16_ex with the oracle:
row strides, A stored K x M (C = A^T . B), B stored N x K (a linear layer's
weight), a fused bias, strided batches, and the torch helpers built on it.  Integer-valued inputs (and
integer bias) are compared bit for bit; float inputs within the tolerance."""
import numpy as np
import pytest

import oracle
from gpu_util import GUARD_BITS, assert_bitexact, assert_close, sample_rows
from tiled_dense_gemm_fp16_b200 import inputs
from tiled_dense_gemm_fp16_b200._binding import Path

pytestmark = pytest.mark.gpu


def _flat(rng, rows, cols, ld, dist):
    """rows x cols values (integers or U[-1,1]) inside a rows x ld buffer with junk padding."""
    buf = rng.uniform(-50, 50, size=(rows, ld)).astype(np.float16)  # padding must never be read
    vals = inputs.draw(rng, (rows, cols), dist)
    buf[:, :cols] = vals
    return buf.reshape(-1), vals


def run_ex(M, N, K, *, lda, ldb, ldc, b_nk, bias, batch=1, gap=0, dist="int", seed=0, path=Path.AUTO,
           workspace=True, offsets=(0, 0, 0), a_km=False):
    """Draw operands, run tg_gemm_relu_f16_ex, and return (gpu C entries, oracle C entries, guards ok)."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    rng = np.random.default_rng(seed)
    a_rows, a_cols = (K, M) if a_km else (M, K)
    b_rows, b_cols = (N, K) if b_nk else (K, N)
    sa = a_rows * lda + gap
    sb = b_rows * ldb + gap
    sc = (M - 1) * ldc + N + gap if M > 0 else gap
    A_all = np.zeros(max(1, (batch - 1) * sa + a_rows * lda), np.float16)
    B_all = np.zeros(max(1, (batch - 1) * sb + b_rows * ldb), np.float16)
    entries = []
    for e in range(batch):
        fa, _ = _flat(rng, a_rows, a_cols, lda, dist)
        fb, _ = _flat(rng, b_rows, b_cols, ldb, dist)
        A_all[e * sa:e * sa + fa.size] = fa
        B_all[e * sb:e * sb + fb.size] = fb
        entries.append((e * sa, e * sb, e * sc))
    bias_h = rng.integers(-8, 9, size=N).astype(np.float16) if (bias and dist == "int") else (
        rng.uniform(-0.5, 0.5, size=N).astype(np.float16) if bias else None)
    c_len = (batch - 1) * sc + (M - 1) * ldc + N
    G = 64
    dev = torch.device("cuda", 0)

    def put(x, off):
        buf = torch.empty(x.size + 8, dtype=torch.float16, device=dev)
        buf[off:off + x.size].copy_(torch.from_numpy(x).to(dev))
        return buf, buf[off:]

    _, Ad = put(A_all, offsets[0])
    _, Bd = put(B_all, offsets[1])
    cbuf = torch.full((c_len + 2 * G + 8,), GUARD_BITS, dtype=torch.int16, device=dev).view(torch.float16)
    Cd = cbuf[G + offsets[2]:]
    bias_d = torch.from_numpy(bias_h).to(dev) if bias_h is not None else None
    opts = tg.options(lda=lda, ldb=ldb, ldc=ldc, b_layout=tg.B_NK if b_nk else tg.B_KN,
                      a_layout=tg.A_KM if a_km else tg.A_MK,
                      bias=bias_d.data_ptr() if bias_d is not None else 0, batch=batch,
                      stride_a=sa, stride_b=sb, stride_c=sc, path=path)
    need = tg.workspace_size_ex(Ad.data_ptr(), Bd.data_ptr(), Cd.data_ptr(), M, N, K, opts)
    assert need >= 0
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = tg.gemm_relu_f16_ex_raw(Ad.data_ptr(), Bd.data_ptr(), Cd.data_ptr(), M, N, K, opts,
                                 torch.cuda.current_stream().cuda_stream,
                                 ws.data_ptr() if workspace else 0, need if workspace else 0)
    assert st == tg.Status.OK, tg.status_string(st)
    torch.cuda.synchronize()
    status, word = tg.device_status()
    assert status == tg.Status.OK, hex(word)
    host = cbuf.view(torch.int16).cpu().numpy().view(np.uint16)
    guards = bool(np.all(host[:G + offsets[2]] == GUARD_BITS) and np.all(host[G + offsets[2] + c_len:] == GUARD_BITS))
    cflat = host[G + offsets[2]:G + offsets[2] + c_len]
    got, ref = [], []
    for (oa, ob, oc) in entries:
        want = oracle.gemm_relu_f16_ex(A_all[oa:], B_all[ob:], M, N, K, lda, ldb, ldc, b_nk=b_nk, bias=bias_h,
                                       C=np.full(M * ldc, GUARD_BITS, np.uint16), a_km=a_km).view(np.uint16)
        g = cflat[oc:oc + M * ldc]
        # Padding columns of C between rows are never written.
        pad = np.ones(M * ldc, bool)
        pad[np.arange(M)[:, None] * ldc + np.arange(N)[None, :]] = False
        pad = pad[:g.size]
        assert np.all(g[pad] == GUARD_BITS), "a padding element of C was written"
        rows = np.arange(M)[:, None] * ldc + np.arange(N)[None, :]
        got.append(g[rows].view(np.float16))
        ref.append(want[rows].view(np.float16))
    return got, ref, guards


STRIDES = {
    "dense": lambda M, N, K, b_nk: (K, K if b_nk else N, N),
    "padded8": lambda M, N, K, b_nk: (K + 8, (K if b_nk else N) + 16, N + 24),
    "odd": lambda M, N, K, b_nk: (K + 1, (K if b_nk else N) + 3, N + 5),
}


@pytest.mark.parametrize("b_nk", [False, True], ids=["B_KN", "B_NK"])
@pytest.mark.parametrize("bias", [False, True], ids=["nobias", "bias"])
@pytest.mark.parametrize("strides", list(STRIDES))
@pytest.mark.parametrize("M,N,K", [(300, 264, 136), (64, 520, 72), (517, 1000, 333)])
def test_layouts_integer_bitexact(M, N, K, b_nk, bias, strides):
    lda, ldb, ldc = STRIDES[strides](M, N, K, b_nk)
    got, ref, guards = run_ex(M, N, K, lda=lda, ldb=ldb, ldc=ldc, b_nk=b_nk, bias=bias,
                              seed=M + N + K + int(b_nk) + 2 * int(bias))
    assert guards
    assert_bitexact(got[0], ref[0], f"{(M, N, K)} {strides} b_nk={b_nk} bias={bias}")


@pytest.mark.parametrize("path", [Path.TC, Path.TC_PAIR, Path.TC_PAIR512, Path.SKINNY],
                         ids=["tc", "pair", "pair512", "skinny"])
@pytest.mark.parametrize("b_nk", [False, True], ids=["B_KN", "B_NK"])
def test_forced_kernels_weight_layout_and_bias(path, b_nk):
    M, N, K = (200, 1032, 264) if path == Path.SKINNY else (520, 1032, 264)
    got, ref, guards = run_ex(M, N, K, lda=K, ldb=K if b_nk else N, ldc=N, b_nk=b_nk, bias=True, path=path,
                              seed=int(path) * 10 + int(b_nk))
    assert guards
    assert_bitexact(got[0], ref[0], f"path {path} b_nk={b_nk}")


@pytest.mark.parametrize("b_nk", [False, True], ids=["B_KN", "B_NK"])
@pytest.mark.parametrize("M,N,K", [(96, 136, 72), (300, 301, 299)])
def test_strided_batches(M, N, K, b_nk):
    lda, ldb, ldc = K + 8, (K if b_nk else N) + 8, N + 8
    got, ref, guards = run_ex(M, N, K, lda=lda, ldb=ldb, ldc=ldc, b_nk=b_nk, bias=True, batch=3, gap=40,
                              seed=7 + int(b_nk))
    assert guards
    for e in range(3):
        assert_bitexact(got[e], ref[e], f"batch entry {e}")


def test_unaligned_bases_with_weight_layout():
    got, ref, guards = run_ex(130, 264, 200, lda=200, ldb=200, ldc=264, b_nk=True, bias=True, offsets=(1, 3, 2),
                              seed=11)
    assert guards
    assert_bitexact(got[0], ref[0], "unaligned bases, B_NK")


def test_weight_layout_unaligned_needs_workspace():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M, N, K = 64, 64, 63
    A = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    W = torch.zeros((N, K), dtype=torch.float16, device="cuda")
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    st = tg.gemm_relu_f16_ex_raw(A.data_ptr(), W.data_ptr(), C.data_ptr(), M, N, K, tg.options(b_layout=tg.B_NK))
    assert st == tg.Status.INVALID_ARG                          # no workspace: refused, nothing launched
    assert tg.linear_relu(A, W).shape == (M, N)                 # torch helper supplies one


def test_k_zero_with_bias_is_relu_of_bias():
    got, ref, guards = run_ex(37, 53, 0, lda=8, ldb=53, ldc=60, b_nk=False, bias=True, seed=3)
    assert guards
    assert_bitexact(got[0], ref[0], "K = 0 with bias")


def test_float_inputs_with_bias():
    got, ref, guards = run_ex(1000, 1024, 768, lda=768, ldb=768, ldc=1024, b_nk=True, bias=True, dist="uniform",
                              seed=19)
    assert guards
    assert_close(got[0], ref[0], "float B_NK + bias")


@pytest.mark.parametrize("b_nk", [False, True], ids=["B_KN", "B_NK"])
@pytest.mark.parametrize("path", [Path.AUTO, Path.TC, Path.TC_PAIR, Path.TC_PAIR512],
                         ids=["auto", "tc", "pair", "pair512"])
@pytest.mark.parametrize("M,N,K", [(520, 1032, 264), (64, 520, 72), (301, 777, 333)])
def test_transposed_a(M, N, K, path, b_nk):
    """A stored K x M (C = A^T . B) with every tensor-core kernel; ragged M goes through the repack path."""
    if path != Path.AUTO and M % 8:
        pytest.skip("a K x M A with M not a multiple of 8 needs the repack path")
    got, ref, guards = run_ex(M, N, K, lda=M, ldb=K if b_nk else N, ldc=N, b_nk=b_nk, bias=True, path=path,
                              a_km=True, seed=M + int(path) + 3 * int(b_nk))
    assert guards
    assert_bitexact(got[0], ref[0], f"A_KM {(M, N, K)} path {path} b_nk={b_nk}")


@pytest.mark.parametrize("strides", ["padded8", "odd"])
def test_transposed_a_strides_and_batches(strides):
    M, N, K = 200, 264, 136
    lda, ldb, ldc = (M + 8, N + 16, N + 24) if strides == "padded8" else (M + 3, N + 1, N + 5)
    got, ref, guards = run_ex(M, N, K, lda=lda, ldb=ldb, ldc=ldc, b_nk=False, bias=True, batch=2, gap=24,
                              a_km=True, seed=31)
    assert guards
    for e in range(2):
        assert_bitexact(got[e], ref[e], f"A_KM {strides} entry {e}")


def test_transposed_a_float_full_tiles():
    got, ref, guards = run_ex(1024, 1024, 1024, lda=1024, ldb=1024, ldc=1024, b_nk=False, bias=False,
                              dist="uniform", a_km=True, seed=41)
    assert guards
    assert_close(got[0], ref[0], "A_KM float 1024")


def test_torch_helpers():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    rng = np.random.default_rng(5)
    x = inputs.draw(rng, (3, 70, 96), "int")
    W = inputs.draw(rng, (136, 96), "int")
    b = rng.integers(-8, 9, size=136).astype(np.float16)
    y = tg.linear_relu(torch.from_numpy(x).cuda(), torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda())
    want = oracle.gemm_relu_f16_ex(x.reshape(-1, 96), W, 210, 136, 96, 96, 96, 136, b_nk=True, bias=b)
    assert_bitexact(y.cpu().numpy().reshape(210, 136), want.reshape(210, 136), "linear_relu")
    A = inputs.draw(rng, (4, 33, 40), "int")
    B = inputs.draw(rng, (4, 40, 24), "int")
    C = tg.bmm_relu(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda())
    for e in range(4):
        assert_bitexact(C[e].cpu().numpy(), oracle.gemm_relu_f16(A[e], B[e]), f"bmm_relu {e}")


def test_linear_8192_weight_layout_full_size():
    """The linear-layer workload at full size: x (8192 x 8192), W (8192 x 8192) as N x K, fp16 bias."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    M = N = K = 8192
    x, W, b = inputs.linear_operands(M, N, K, seed=5)
    y = tg.linear_relu(torch.from_numpy(x).cuda(), torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda())
    torch.cuda.synchronize()
    rows = sample_rows(M, n=24, seed=5)
    want = oracle.gemm_relu_f16_ex(np.ascontiguousarray(x[rows]), W, len(rows), N, K, K, K, N, b_nk=True, bias=b)
    assert_close(y[rows].cpu().numpy(), want.reshape(len(rows), N), "linear 8192 rows")
