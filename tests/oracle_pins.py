"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Each ``check_*`` function takes a loaded oracle library (the real one, or a
deliberately broken variant in ``test_oracle_pin_strength.py``) and raises
AssertionError when the oracle disagrees with:
  * numpy's own float16 conversion (an independent implementation),
  * IEEE 754 binary16 values derived by hand (``tests/golden/``),
  * exact integer matrix products,
  * exact rational sums and the standard error bound of recursive fp32
    summation,
  * closed forms (identity, all-ones, zero operands, overflow),
  * the hand-worked examples of the matmul_relu quick-start kernel
    ("TileLang" wiki page, "Programming model"),
  * for the MXFP8 grouped GEMM: torch's own float8_e4m3fn / float8_e5m2 /
    float8_e8m0fnu decoders and float32 -> bfloat16 rounding (independent
    implementations), hand-derived bfloat16 edge values, exact rational
    sums rounded to bfloat16 by search over all bfloat16 values, and
    closed forms (identity A, scale invariance, group separation).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

import oracle
from tiled_dense_gemm_fp16_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits(a):
    return np.asarray(a).view(np.uint16)


# --------------------------------------------------------------------------
# fp16 <-> fp32 conversions
# --------------------------------------------------------------------------

def check_f16_to_f32_all_patterns(lib):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_bits_to_f32(h, lib=lib)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def load_f16_golden():
    rows = []
    with open(os.path.join(GOLDEN, "f16_rne_edges.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            x = float(tok[0]) if tok[0] in ("inf", "-inf") else float.fromhex(tok[0])
            rows.append((x, int(tok[1], 16), " ".join(tok[2:])))
    return rows


def check_f32_to_f16_golden(lib):
    rows = load_f16_golden()
    assert len(rows) >= 20
    x = np.array([r[0] for r in rows], dtype=np.float32)
    # Every golden input is exactly representable in fp32.
    assert all(float(xi) == r[0] for xi, r in zip(x, rows))
    got = oracle.f32_to_f16_bits(x, lib=lib)
    for g, (xv, want, why) in zip(got, rows):
        assert int(g) == want, f"{xv!r}: got 0x{int(g):04x}, want 0x{want:04x} ({why})"


def check_f32_to_f16_vs_numpy(lib, n=1 << 20, seed=123):
    rng = np.random.default_rng(seed)
    # Uniform random bit patterns: every exponent, NaNs and infinities.
    u = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    # Values concentrated on the fp16 range, subnormals included.
    e = rng.integers(-30, 18, size=n)
    v = (rng.uniform(1.0, 2.0, size=n) * np.exp2(e)) * rng.choice([-1.0, 1.0], size=n)
    x = np.concatenate([u.view(np.float32), v.astype(np.float32)])
    got = oracle.f32_to_f16_bits(x, lib=lib)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], ref[~nan])
    gh = got[nan]
    assert np.all((gh & 0x7C00) == 0x7C00) and np.all((gh & 0x03FF) != 0)


def check_f32_to_f16_ties(lib):
    """Midpoints of every pair of adjacent positive halves round to the even pattern.

    For positive finite halves the bit pattern order is the value order, so the
    two neighbours of the midpoint of patterns p and p+1 are p and p+1 and the
    even one is whichever has a clear low bit.  The midpoint above 65504 is
    65520 and ties to the even pattern 0x7c00, which is +inf.
    """
    p = np.arange(0, 0x7BFF, dtype=np.uint16)          # p and p+1 both finite
    lo = p.view(np.float16).astype(np.float64)
    hi = (p + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # exact in fp32
    want = np.where(p % 2 == 0, p, p + 1).astype(np.uint16)
    got = oracle.f32_to_f16_bits(mid, lib=lib)
    assert np.array_equal(got, want)
    got_neg = oracle.f32_to_f16_bits(-mid, lib=lib)
    assert np.array_equal(got_neg, want | 0x8000)
    assert int(oracle.f32_to_f16_bits(np.array([65520.0], np.float32), lib=lib)[0]) == 0x7C00


# --------------------------------------------------------------------------
# GEMM + ReLU
# --------------------------------------------------------------------------

def load_worked_examples():
    examples = []
    cur = None
    with open(os.path.join(GOLDEN, "gemm_worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] == "example":
                cur = {"id": int(tok[1])}
                examples.append(cur)
            elif tok[0] == "M":
                cur["M"], cur["N"], cur["K"] = (int(t) for t in tok[3:6])
            else:
                cur[tok[0]] = [float(t) for t in tok[1:]]
    return examples


def check_worked_examples(lib):
    ex = load_worked_examples()
    assert len(ex) == 3
    for e in ex:
        M, N, K = e["M"], e["N"], e["K"]
        A = np.array(e["A"], dtype=np.float16).reshape(M, K)
        B = np.array(e["B"], dtype=np.float16).reshape(K, N)
        want = np.array(e["C"], dtype=np.float16).reshape(M, N)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        assert np.array_equal(_bits(got), _bits(want)), f"example {e['id']}: {got} != {want}"


def _exact_int_reference(A, B):
    """ReLU of the exact integer product, rounded to fp16 by numpy."""
    S = A.astype(np.int64) @ B.astype(np.int64)
    R = np.maximum(S, 0).astype(np.float64)
    with np.errstate(over="ignore"):
        return R.astype(np.float16)


def check_integer_exact(lib):
    """Integer operands: every partial sum is an integer below 2^24, so fp32 is exact."""
    rng = np.random.default_rng(7)
    for (M, N, K) in [(7, 5, 13), (33, 17, 65), (64, 48, 300), (3, 129, 2500), (1, 1, 1)]:
        A = rng.integers(-2, 3, size=(M, K)).astype(np.float16)
        B = rng.integers(-2, 3, size=(K, N)).astype(np.float16)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        assert np.array_equal(_bits(got), _bits(_exact_int_reference(A, B))), (M, N, K)


def check_all_ones(lib):
    """All-ones operands: C = fp16(K); exactly K up to 2048, its nearest even half above."""
    for K in (1, 2, 17, 255, 2048, 2049, 2051, 4097, 6001):
        A = np.ones((3, K), np.float16)
        B = np.ones((K, 5), np.float16)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        if K <= 2048:
            want = float(K)
        else:
            # quantum 2 in [2048, 4096), 4 in [4096, 8192); ties to even patterns
            q = 2 if K < 4096 else 4
            lo = (K // q) * q
            r = K - lo
            up = r * 2 > q or (r * 2 == q and (lo // q) % 2 == 1)
            want = float(lo + q if up else lo)
        assert np.all(got.astype(np.float64) == want), (K, got[0, 0], want)


def check_overflow(lib):
    """Products of 2 * 2 summed K times: 4K; 65504 is finite, 65520 and above is +inf."""
    for K, want in [(16376, 0x7BFF), (16379, 0x7BFF), (16380, 0x7C00), (20000, 0x7C00)]:
        A = np.full((1, K), 2.0, np.float16)
        B = np.full((K, 2), 2.0, np.float16)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        assert np.all(_bits(got) == want), (K, hex(int(_bits(got)[0, 0])))


def check_identity(lib):
    """A = I gives ReLU(B) bit for bit, with +0 for every non-positive entry."""
    rng = np.random.default_rng(11)
    K, N = 96, 70
    B = rng.uniform(-3, 3, size=(K, N)).astype(np.float16)
    B[0, :8] = np.array([0.0, -0.0, 6e-8, -6e-8, 1e-5, 65504, -65504, 2.0**-24], np.float16)
    A = np.eye(K, dtype=np.float16)
    got = oracle.gemm_relu_f16(A, B, lib=lib)
    want = np.where(B.astype(np.float32) > 0, B, np.float16(0.0)).astype(np.float16)
    assert np.array_equal(_bits(got), _bits(want))
    # Transposed roles on a non-square right operand: B = I gives ReLU(A).
    A2 = rng.uniform(-3, 3, size=(40, K)).astype(np.float16)
    got2 = oracle.gemm_relu_f16(A2, np.eye(K, dtype=np.float16), lib=lib)
    want2 = np.where(A2.astype(np.float32) > 0, A2, np.float16(0.0)).astype(np.float16)
    assert np.array_equal(_bits(got2), _bits(want2))


def check_zero_operands(lib):
    rng = np.random.default_rng(5)
    A = rng.uniform(-1, 1, size=(9, 31)).astype(np.float16)
    B = rng.uniform(-1, 1, size=(31, 12)).astype(np.float16)
    for a, b in [(np.zeros_like(A), B), (A, np.zeros_like(B)), (-np.zeros_like(A), B)]:
        got = oracle.gemm_relu_f16(a, b, lib=lib)
        assert np.all(_bits(got) == 0)
    # K = 0: the empty sum is +0.
    got = oracle.gemm_relu_f16(np.zeros((4, 0), np.float16), np.zeros((0, 6), np.float16), lib=lib)
    assert got.shape == (4, 6) and np.all(_bits(got) == 0)


def check_nonnegative(lib):
    for dist in inputs.DISTRIBUTIONS:
        A, B = inputs.operands(37, 53, 211, dist, seed=3)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        assert np.all((_bits(got) & 0x8000) == 0)
        assert np.all(got.astype(np.float32) >= 0)


def _f16_of_real(x: float, toward: str) -> float:
    """fp16(x) of a real x, with x first pushed one double ulp outward."""
    y = float(x)
    y = math.nextafter(y, -math.inf) if toward == "down" else math.nextafter(y, math.inf)
    with np.errstate(over="ignore"):
        return float(np.float16(max(y, 0.0)))


def check_exact_rational_bound(lib):
    """|fp32 recursive sum - exact sum| <= gamma_{K-1} * sum |a_k b_k| (products exact).

    The oracle's fp16 output must then lie between fp16(relu(S - E)) and
    fp16(relu(S + E)), because ReLU and rounding to nearest are monotone.
    """
    u = Fraction(1, 1 << 24)
    for (M, N, K), dist, seed in [((8, 8, 8), "uniform", 0), ((5, 3, 17), "normal01", 1),
                                  ((4, 6, 257), "uniform", 2)]:
        A, B = inputs.operands(M, N, K, dist, seed=seed)
        got = oracle.gemm_relu_f16(A, B, lib=lib).astype(np.float64)
        Af = [[Fraction(float(v)) for v in row] for row in A.astype(np.float64)]
        Bf = [[Fraction(float(v)) for v in row] for row in B.astype(np.float64)]
        gamma = (K - 1) * u / (1 - (K - 1) * u)
        for i in range(M):
            for j in range(N):
                prods = [Af[i][k] * Bf[k][j] for k in range(K)]
                S = sum(prods, Fraction(0))
                E = gamma * sum(abs(p) for p in prods)
                lo = _f16_of_real(S - E, "down")
                hi = _f16_of_real(S + E, "up")
                assert lo <= got[i, j] <= hi, (i, j, float(S), got[i, j], lo, hi)


def check_sequential_fp32_tiny(lib):
    """An independent fp32 scalar loop (numpy.float32 arithmetic) in k order agrees bit for bit."""
    for (M, N, K), dist, seed in [((8, 8, 8), "uniform", 0), ((5, 3, 17), "normal01", 4),
                                  ((2, 7, 64), "uniform", 9)]:
        A, B = inputs.operands(M, N, K, dist, seed=seed)
        got = oracle.gemm_relu_f16(A, B, lib=lib)
        want = np.empty((M, N), np.float16)
        for i in range(M):
            for j in range(N):
                s = np.float32(0.0)
                for k in range(K):
                    s = np.float32(s + np.float32(A[i, k]) * np.float32(B[k, j]))
                want[i, j] = np.float16(s) if s > 0 else np.float16(0.0)
        assert np.array_equal(_bits(got), _bits(want)), (M, N, K)


def check_rows_and_threads(lib):
    A, B = inputs.operands(67, 45, 129, "uniform", seed=8)
    full = oracle.gemm_relu_f16(A, B, nthreads=1, lib=lib)
    par = oracle.gemm_relu_f16(A, B, nthreads=4, lib=lib)
    assert np.array_equal(_bits(full), _bits(par))
    rows = [0, 5, 66, 31]
    sub = oracle.gemm_relu_f16_rows(A, B, rows, lib=lib)
    assert np.array_equal(_bits(sub), _bits(full[rows]))


# --------------------------------------------------------------------------
# General layouts and bias (oracle_gemm_relu_f16_ex)
# --------------------------------------------------------------------------

def check_ex_dense_equals_base(lib):
    """Dense strides, B as K x N, no bias: the same bits as the base oracle."""
    for (M, N, K), dist in [((37, 53, 211), "uniform"), ((8, 8, 8), "normal01"), ((64, 17, 300), "int")]:
        A, B = inputs.operands(M, N, K, dist, seed=M + N)
        base = oracle.gemm_relu_f16(A, B, lib=lib)
        ex = oracle.gemm_relu_f16_ex(A, B, M, N, K, K, N, N, lib=lib).reshape(M, N)
        assert np.array_equal(_bits(ex), _bits(base)), (M, N, K)


def check_ex_weight_layout(lib):
    """B stored N x K (C = A . B^T) gives the base oracle's bits on the transposed copy."""
    for (M, N, K) in [(29, 41, 67), (5, 130, 9)]:
        A, B = inputs.operands(M, N, K, "uniform", seed=K)
        Bt = np.ascontiguousarray(B.T)                       # N x K storage of the same B
        ex = oracle.gemm_relu_f16_ex(A, Bt, M, N, K, K, K, N, b_nk=True, lib=lib).reshape(M, N)
        assert np.array_equal(_bits(ex), _bits(oracle.gemm_relu_f16(A, B, lib=lib))), (M, N, K)


def check_ex_transposed_a(lib):
    """A stored K x M (C = A^T . B) gives the base oracle's bits on the transposed copy, also with
    B stored N x K."""
    for (M, N, K) in [(29, 41, 67), (70, 9, 33)]:
        A, B = inputs.operands(M, N, K, "uniform", seed=M * K)
        At = np.ascontiguousarray(A.T)                       # K x M storage of the same A
        want = _bits(oracle.gemm_relu_f16(A, B, lib=lib))
        ex = oracle.gemm_relu_f16_ex(At, B, M, N, K, M, N, N, a_km=True, lib=lib).reshape(M, N)
        assert np.array_equal(_bits(ex), want), (M, N, K)
        Bt = np.ascontiguousarray(B.T)
        ex2 = oracle.gemm_relu_f16_ex(At, Bt, M, N, K, M, K, N, a_km=True, b_nk=True, lib=lib).reshape(M, N)
        assert np.array_equal(_bits(ex2), want), (M, N, K)


def check_ex_strides(lib):
    """Row strides wider than the rows read the same values; C's padding is left alone."""
    M, N, K = 23, 31, 45
    lda, ldb, ldc = K + 7, N + 3, N + 5
    A, B = inputs.operands(M, N, K, "int", seed=9)
    rng = np.random.default_rng(10)
    Ap = rng.uniform(-9, 9, size=(M, lda)).astype(np.float16)
    Bp = rng.uniform(-9, 9, size=(K, ldb)).astype(np.float16)
    Ap[:, :K] = A
    Bp[:, :N] = B
    Cinit = np.full(M * ldc, 0x7E55, dtype=np.uint16)
    got = oracle.gemm_relu_f16_ex(Ap, Bp, M, N, K, lda, ldb, ldc, C=Cinit, lib=lib).view(np.uint16).reshape(M, ldc)
    assert np.array_equal(got[:, :N], _bits(oracle.gemm_relu_f16(A, B, lib=lib)))
    assert np.all(got[:, N:] == 0x7E55)


def check_ex_bias_exact(lib):
    """Integer operands and bias: relu(A . B + bias) is exact, so fp16 of it is unique."""
    M, N, K = 19, 40, 133
    A, B = inputs.operands(M, N, K, "int", seed=21)
    bias = np.random.default_rng(22).integers(-40, 41, size=N).astype(np.float16)
    got = oracle.gemm_relu_f16_ex(A, B, M, N, K, K, N, N, bias=bias, lib=lib).reshape(M, N)
    S = A.astype(np.int64) @ B.astype(np.int64) + bias.astype(np.int64)[None, :]
    want = np.maximum(S, 0).astype(np.float64).astype(np.float16)
    assert np.array_equal(_bits(got), _bits(want))


def check_ex_bias_closed_form(lib):
    """A = 0: every row of C is ReLU(bias) (+0 for non-positive entries)."""
    M, N, K = 6, 33, 17
    bias = np.random.default_rng(3).uniform(-4, 4, size=N).astype(np.float16)
    bias[:4] = np.array([0.0, -0.0, 65504, -1e-7], np.float16)
    A = np.zeros((M, K), np.float16)
    B = np.random.default_rng(4).uniform(-1, 1, size=(N, K)).astype(np.float16)
    got = oracle.gemm_relu_f16_ex(A, B, M, N, K, K, K, N, b_nk=True, bias=bias, lib=lib).reshape(M, N)
    want = np.where(bias.astype(np.float32) > 0, bias, np.float16(0)).astype(np.float16)
    assert np.array_equal(_bits(got), np.tile(_bits(want), (M, 1)))


# --------------------------------------------------------------------------
# MXFP8 grouped GEMM
# --------------------------------------------------------------------------

def _torch_fp8(codes, fmt):
    import torch
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy())
    return t.view(torch.float8_e4m3fn if fmt == 0 else torch.float8_e5m2).to(torch.float64).numpy()


def _same_values(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    num = ~np.isnan(b)
    return bool(np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[num], b[num])
                and np.array_equal(np.signbit(a[num]), np.signbit(b[num])))


def check_fp8_decode_all_codes(lib):
    """All 256 codes of E4M3 and E5M2 against torch's float8 dtypes (values, NaNs and signs of zero)."""
    codes = np.arange(256, dtype=np.uint8)
    for fmt in (0, 1):
        assert _same_values(oracle.fp8_to_f64(codes, fmt, lib=lib), _torch_fp8(codes, fmt)), fmt
    # Facts of the formats: E4M3 max 448 and no infinities; E5M2 max 57344 and +-inf.
    assert oracle.fp8_to_f64([0x7E], 0, lib=lib)[0] == 448.0
    assert oracle.fp8_to_f64([0x7C], 1, lib=lib)[0] == math.inf


def check_ue8m0_decode_all_codes(lib):
    import torch
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert _same_values(oracle.ue8m0_to_f64(codes, lib=lib), want)
    assert oracle.ue8m0_to_f64([127], lib=lib)[0] == 1.0


def _bf16_value(bits):
    import torch
    t = torch.from_numpy(np.asarray(bits, np.uint16).astype(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def check_bf16_rne_vs_torch(lib, n=1 << 15, seed=77):
    """float32-representable doubles: torch's float32 -> bfloat16 (RNE) is a single rounding there."""
    import torch
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16_bits(f.astype(np.float64), lib=lib)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], want[~nan])


def check_bf16_rne_edges(lib):
    """Hand-derived bfloat16 facts (8 significant bits, fp32's exponent range)."""
    cases = [
        (1.0, 0x3F80), (-2.0, 0xC000), (0.0, 0x0000), (-0.0, 0x8000),
        (1 + 2 ** -8, 0x3F80),            # tie between 1 and 1 + 2^-7: to even (1)
        (1 + 3 * 2 ** -8, 0x3F82),        # tie between 1 + 2^-7 and 1 + 2^-6: to even
        (1 + 2 ** -8 + 2 ** -40, 0x3F81), # just above the tie: up (a double-only input)
        ((2 - 2 ** -7) * 2.0 ** 127, 0x7F7F),   # largest finite
        ((2 - 2 ** -8) * 2.0 ** 127, 0x7F80),   # halfway to 2^128: ties to even overflow to inf
        (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000), (3 * 2.0 ** -134, 0x0002),
        (2.0 ** -126, 0x0080), ((1 - 2 ** -9) * 2.0 ** -126, 0x0080),
        (1.5 * 2.0 ** 128, 0x7F80), (-(2.0 ** 200), 0xFF80),   # doubles beyond bfloat16's range
        (math.inf, 0x7F80), (-math.inf, 0xFF80),
    ]
    got = oracle.f64_to_bf16_bits([c[0] for c in cases], lib=lib)
    for (x, want), g in zip(cases, got):
        assert int(g) == want, (x, hex(int(g)), hex(want))


def _mx_problem(m_sizes, N, K, seed, int_values=True, scale_range=(124, 130)):
    """Codes, scales and row offsets for a grouped problem (rows padded to 128 per group)."""
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum([(m + 127) // 128 * 128 for m in m_sizes])[:-1]]).astype(np.int64)
    rows = int(sum((m + 127) // 128 * 128 for m in m_sizes))
    G = len(m_sizes)
    if int_values:
        # E4M3 codes of the integers -3..3: 0, 1 (0x38), 2 (0x40), 3 (0x44) and their negatives.
        table = np.array([0xC4, 0xC0, 0xB8, 0x00, 0x38, 0x40, 0x44], np.uint8)
        A = table[rng.integers(0, 7, size=(rows, K))]
        B = table[rng.integers(0, 7, size=(G, N, K))]
    else:
        A = rng.integers(0, 256, size=(rows, K)).astype(np.uint8)
        B = rng.integers(0, 256, size=(G, N, K)).astype(np.uint8)
        A[(A & 0x7F) == 0x7F] = 0x30   # no NaN codes
        B[(B & 0x7F) == 0x7F] = 0x30
    SFA = rng.integers(scale_range[0], scale_range[1], size=(rows, K // 32)).astype(np.uint8)
    SFB = rng.integers(scale_range[0], scale_range[1], size=(G, N, K // 32)).astype(np.uint8)
    return A, SFA, B, SFB, offs


def _nearest_bf16(frac_values):
    """Exact rationals -> bfloat16 bits by search over every finite bfloat16 (ties to even pattern)."""
    allbits = np.arange(1 << 16, dtype=np.uint32)
    vals = _bf16_value(allbits.astype(np.uint16))
    fin = np.isfinite(vals) & ~((allbits == 0x8000))
    cand_bits, cand_vals = allbits[fin], vals[fin]
    order = np.argsort(cand_vals, kind="stable")
    cand_bits, cand_vals = cand_bits[order], cand_vals[order]
    out = []
    for q in frac_values:
        x = float(q)
        i = int(np.searchsorted(cand_vals, x))
        best = None
        for j in (i - 1, i, i + 1):
            if 0 <= j < cand_vals.size:
                d = abs(Fraction(cand_vals[j]) - q)
                key = (d, int(cand_bits[j]) & 1)
                if best is None or key < best[0]:
                    best = (key, int(cand_bits[j]))
        out.append(best[1])
    return np.array(out, np.uint16)


def check_mxf8_exact_rational_tiny(lib):
    """Brute force: exact rational sums of torch-decoded scaled values, rounded by search."""
    m_sizes, N, K = [3, 2], 5, 64
    for fmt in (0, 1):
        A, SFA, B, SFB, offs = _mx_problem(m_sizes, N, K, seed=fmt + 1, int_values=False, scale_range=(120, 134))
        if fmt == 1:
            A[(A & 0x7C) == 0x7C] = 0x3C  # no E5M2 inf/NaN codes
            B[(B & 0x7C) == 0x7C] = 0x3C
        got = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, fmt, fmt, lib=lib)
        av, bv = _torch_fp8(A, fmt), _torch_fp8(B, fmt)
        for g, (m, o) in enumerate(zip(m_sizes, offs)):
            for i in range(m):
                r = o + i
                q = []
                for j in range(N):
                    tot = Fraction(0)
                    for k in range(K):
                        tot += (Fraction(av[r, k]) * Fraction(2) ** (int(SFA[r, k // 32]) - 127)
                                * Fraction(bv[g, j, k]) * Fraction(2) ** (int(SFB[g, j, k // 32]) - 127))
                    q.append(tot)
                assert np.array_equal(got[r], _nearest_bf16(q)), (fmt, g, i)


def check_mxf8_integer_exact(lib):
    """Integer values with unit scales: the sums are exact integers below 2^24; torch rounds them to bf16."""
    import torch
    m_sizes, N, K = [130, 1, 64], 24, 96
    A, SFA, B, SFB, offs = _mx_problem(m_sizes, N, K, seed=5, scale_range=(127, 128))
    av, bv = _torch_fp8(A, 0).astype(np.int64), _torch_fp8(B, 0).astype(np.int64)
    got = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib, relu=True)
    for g, (m, o) in enumerate(zip(m_sizes, offs)):
        S = np.maximum(av[o:o + m] @ bv[g].T, 0).astype(np.float32)
        want = torch.from_numpy(S).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got[o:o + m], want), g


def check_mxf8_identity_and_groups(lib):
    """A = identity (code 0x38 = 1.0, unit scales): group g's rows are rows of B_g^T, i.e.
    C[o_g + i, j] = b_g(j, i); rows between groups are left untouched."""
    m_sizes, N, K = [40, 7, 64], 48, 64
    G = len(m_sizes)
    A, SFA, B, SFB, offs = _mx_problem(m_sizes, N, K, seed=9, int_values=False, scale_range=(127, 128))
    A[:] = 0
    for o, m in zip(offs, m_sizes):
        A[o + np.arange(m), np.arange(m)] = 0x38
    guard = np.full(A.shape[0] * N, 0x7E55, np.uint16)
    got = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, C=guard, lib=lib)
    bv = _torch_fp8(B, 0)
    covered = np.zeros(A.shape[0], bool)
    for g, (o, m) in enumerate(zip(offs, m_sizes)):
        want = _bf16_bits_exact(bv[g, :, :m].T + 0.0)      # a sum that starts at +0 is never -0
        assert np.array_equal(got[o:o + m], want), g
        covered[o:o + m] = True
    assert np.all(got[~covered] == 0x7E55)


def _bf16_bits_exact(x):
    """bfloat16 bits of values known to be exactly representable in bfloat16 (fp8 values are)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def check_mxf8_scale_invariance(lib):
    """Moving a power of two between an element block and its scale changes nothing: doubling
    every E4M3 value of A's block (r, s) (exponent field + 1) and lowering its scale by one
    gives the same C; raising one of B's scales by one doubles that block's contribution."""
    m_sizes, N, K = [5], 16, 96
    A, SFA, B, SFB, offs = _mx_problem(m_sizes, N, K, seed=13, scale_range=(126, 129))
    base = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib)
    A2, SFA2 = A.copy(), SFA.copy()
    blk = A2[2, 32:64]
    nz = (blk & 0x7F) != 0
    blk[nz] = blk[nz] + 0x08                 # exponent + 1 (values are normal and small)
    SFA2[2, 1] -= 1
    got = oracle.gemm_mxf8_grouped(A2, SFA2, B, SFB, m_sizes, offs, N, K, lib=lib)
    assert np.array_equal(got, base)
    # Only B's block 2 nonzero: raising its scale doubles every output exactly.
    B3 = B.copy()
    B3[:, :, :64] = 0
    c1 = _bf16_value(oracle.gemm_mxf8_grouped(A, SFA, B3, SFB, m_sizes, offs, N, K, lib=lib))
    SFB3 = SFB.copy()
    SFB3[:, :, 2] += 1
    c2 = _bf16_value(oracle.gemm_mxf8_grouped(A, SFA, B3, SFB3, m_sizes, offs, N, K, lib=lib))
    assert np.array_equal(c2, 2 * c1)


def check_mxf8_relu_and_nan(lib):
    """Without ReLU negative sums stay negative; with it they are +0.  A NaN scale (255) makes
    its rows NaN without ReLU and +0 with it."""
    m_sizes, N, K = [9], 12, 32
    A, SFA, B, SFB, offs = _mx_problem(m_sizes, N, K, seed=17, scale_range=(127, 128))
    plain = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib)
    relu = oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, relu=True, lib=lib)
    pv = _bf16_value(plain[:9])
    assert (pv < 0).any()
    assert np.array_equal(relu[:9], np.where(pv > 0, plain[:9], 0).astype(np.uint16))
    SFA[4, 0] = 255
    nanrow = _bf16_value(oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib)[4])
    assert np.all(np.isnan(nanrow))
    assert np.all(oracle.gemm_mxf8_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, relu=True, lib=lib)[4] == 0)


# --------------------------------------------------------------------------
# NVF4 grouped GEMM
# --------------------------------------------------------------------------

def _golden_e2m1():
    rows = []
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                code, val = line.split()[:2]
                rows.append((int(code, 16), float(val)))
    return rows


def check_e2m1_decode_golden(lib):
    rows = _golden_e2m1()
    assert len(rows) == 16
    got = oracle.e2m1_to_f64([c for c, _ in rows], lib=lib)
    want = np.array([v for _, v in rows])
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))
    # Only the low nibble is a code: the high nibble of the byte is ignored.
    assert np.array_equal(oracle.e2m1_to_f64([0xF7, 0x35], lib=lib), [6.0, 3.0])


def check_ue4m3_decode(lib):
    """Scale codes with a clear sign bit are E4M3 values (torch's decoder); a set sign bit is invalid."""
    codes = np.arange(128, dtype=np.uint8)
    assert _same_values(oracle.ue4m3_to_f64(codes, lib=lib), _torch_fp8(codes, 0))
    assert np.all(np.isnan(oracle.ue4m3_to_f64(np.arange(128, 256, dtype=np.uint8), lib=lib)))


# E2M1 codes of the integers -4..4 that E2M1 holds: 0, +-1, +-2, +-3, +-4.
_E2M1_INT = {0: 0x0, 1: 0x2, 2: 0x4, 3: 0x5, 4: 0x6, -1: 0xA, -2: 0xC, -3: 0xD, -4: 0xE}


def _pack_nibbles(codes):
    """Codes (..., K) -> bytes (..., K/2), element 2i in the low nibble."""
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def _nvf4_problem(m_sizes, N, K, seed, int_values=True, scale_codes=(0x38,)):
    rng = np.random.default_rng(seed)
    offs, rows = inputs.mx_group_offsets(m_sizes)
    G = len(m_sizes)
    if int_values:
        keys = np.array(sorted(_E2M1_INT))
        av = keys[rng.integers(0, len(keys), size=(rows, K))]
        bv = keys[rng.integers(0, len(keys), size=(G, N, K))]
        ac = np.vectorize(_E2M1_INT.get)(av).astype(np.uint8)
        bc = np.vectorize(_E2M1_INT.get)(bv).astype(np.uint8)
    else:
        ac = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
        bc = rng.integers(0, 16, size=(G, N, K)).astype(np.uint8)
        av = bv = None
    sc = np.asarray(scale_codes, np.uint8)
    SFA = sc[rng.integers(0, sc.size, size=(rows, K // 16))]
    SFB = sc[rng.integers(0, sc.size, size=(G, N, K // 16))]
    return _pack_nibbles(ac), SFA, _pack_nibbles(bc), SFB, offs, (ac, bc, av, bv)


def check_nvf4_integer_exact(lib):
    """Integer E2M1 values with unit scales (0x38 = 1.0): exact int64 products, rounded by torch."""
    import torch
    m_sizes, N, K = [130, 3], 24, 128
    A, SFA, B, SFB, offs, (_, _, av, bv) = _nvf4_problem(m_sizes, N, K, seed=2)
    got = oracle.gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib)
    for g, (o, m) in enumerate(zip(offs, m_sizes)):
        S = (av[o:o + m].astype(np.int64) @ bv[g].astype(np.int64).T).astype(np.float32)
        want = torch.from_numpy(S).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got[o:o + m], want), g


def check_nvf4_identity_nibble_order(lib):
    """A = identity in E2M1 (code 0x2 = 1.0): row i of group g is column i of B_g's stored rows, so the
    element order inside each packed byte (low nibble first) decides every output."""
    m_sizes, N, K = [20], 16, 32
    A, SFA, B, SFB, offs, (_, bc, _, _) = _nvf4_problem(m_sizes, N, K, seed=4, int_values=False)
    ac = np.zeros((A.shape[0], K), np.uint8)
    ac[np.arange(20), np.arange(20)] = 0x2
    SFA[:] = 0x38
    SFB[:] = 0x38
    got = oracle.gemm_nvf4_grouped(_pack_nibbles(ac), SFA, B, SFB, m_sizes, offs, N, K, lib=lib)
    table = dict(_golden_e2m1())
    want = np.array([[table[int(bc[0, j, i])] for j in range(N)] for i in range(20)], np.float32) + 0.0
    assert np.array_equal(got[:20], _bf16_bits_exact(want))


def check_nvf4_exact_rational_tiny(lib):
    """Brute force with golden element values, torch-decoded scales, exact sums and alpha."""
    m_sizes, N, K = [2, 3], 4, 48
    alpha = 0.3  # not a power of two: the product alpha * sum is rounded once, to bf16
    A, SFA, B, SFB, offs, (ac, bc, _, _) = _nvf4_problem(m_sizes, N, K, seed=6, int_values=False,
                                                          scale_codes=(0x20, 0x30, 0x38, 0x41, 0x4C, 0x57))
    got = oracle.gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, alpha=alpha, lib=lib)
    table = {c: Fraction(v) for c, v in _golden_e2m1()}
    sc = {int(c): Fraction(float(v)) for c, v in zip(range(127), _torch_fp8(np.arange(127, dtype=np.uint8), 0))}
    for g, (o, m) in enumerate(zip(offs, m_sizes)):
        for i in range(m):
            r = o + i
            q = []
            for j in range(N):
                tot = sum(table[int(ac[r, k])] * sc[int(SFA[r, k // 16])] * table[int(bc[g, j, k])]
                          * sc[int(SFB[g, j, k // 16])] for k in range(K))
                q.append(Fraction(alpha) * tot)
            assert np.array_equal(got[r], _nearest_bf16(q)), (g, i)


def check_nvf4_alpha_relu(lib):
    """alpha = 2^-3 scales every output exactly; ReLU maps the non-positive ones to +0."""
    m_sizes, N, K = [7], 10, 64
    A, SFA, B, SFB, offs, _ = _nvf4_problem(m_sizes, N, K, seed=8)
    base = _bf16_value(oracle.gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, lib=lib)[:7])
    scaled = _bf16_value(oracle.gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, alpha=0.125, lib=lib)[:7])
    assert np.array_equal(scaled, base / 8)
    assert (base < 0).any()
    relu = _bf16_value(oracle.gemm_nvf4_grouped(A, SFA, B, SFB, m_sizes, offs, N, K, alpha=0.125, relu=True,
                                                lib=lib)[:7])
    assert np.array_equal(relu, np.where(base > 0, base / 8, 0.0))


# --------------------------------------------------------------------------
# Dequantized (W4A16) GEMM
# --------------------------------------------------------------------------

def _pack4(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def check_dequant_all_codes_all_scales(lib):
    """Every code 0..15 against every finite fp16 scale: numpy's float32 product (exact) rounded by
    numpy's float16 conversion (an independent implementation)."""
    scales = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    scales = scales[np.isfinite(scales)]
    N, K = scales.size, 16
    codes = np.tile(np.arange(16, dtype=np.uint8), (N, 1))
    S = scales.reshape(N, 1)
    got = oracle.dequant_w4_f16(_pack4(codes), S, N, K, 16, lib=lib)
    with np.errstate(over="ignore"):  # large scales times 8 overflow to inf, as they should
        want = ((np.arange(16, dtype=np.float32) - 8)[None, :] * scales.astype(np.float32)[:, None]).astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def check_dequant_groups_and_nibbles(lib):
    """Hand-checkable structure: code k % 16 at column k, scale 2^g for group g, group size 32:
    W[n, k] = (k % 16 - 8) * 2^(k // 32) exactly (small integers times powers of two)."""
    N, K, group = 3, 128, 32
    codes = np.tile(np.arange(K) % 16, (N, 1)).astype(np.uint8)
    S = np.tile(np.array([1.0, 2.0, 4.0, 8.0], np.float16), (N, 1))
    got = oracle.dequant_w4_f16(_pack4(codes), S, N, K, group, lib=lib).astype(np.float64)
    k = np.arange(K)
    want = np.tile((k % 16 - 8) * 2.0 ** (k // 32), (N, 1))
    assert np.array_equal(got, want)
    # Row-specific scales: row n uses its own scale row.
    S2 = np.array([[1.0] * 4, [0.5] * 4, [-3.0] * 4], np.float16)
    got2 = oracle.dequant_w4_f16(_pack4(codes), S2, N, K, group, lib=lib).astype(np.float64)
    assert np.array_equal(got2, (k % 16 - 8)[None, :] * np.array([1.0, 0.5, -3.0])[:, None])


def check_w4a16_gemm_integer_exact(lib):
    """Unit scales make W the integers q - 8; with integer A the product is exact (int64 matmul)."""
    import torch
    rng = np.random.default_rng(31)
    M, N, K, group = 7, 20, 256, 64
    A = rng.integers(-2, 3, size=(M, K)).astype(np.float16)
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    S = np.ones((N, K // group), np.float16)
    got = oracle.gemm_relu_w4a16(A, _pack4(codes), S, group, lib=lib)
    exact = np.maximum(A.astype(np.int64) @ (codes.astype(np.int64) - 8).T, 0).astype(np.float32)
    want = torch.from_numpy(exact).to(torch.float16).numpy()
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


ALL_CHECKS = [
    check_f16_to_f32_all_patterns,
    check_f32_to_f16_golden,
    check_f32_to_f16_vs_numpy,
    check_f32_to_f16_ties,
    check_worked_examples,
    check_integer_exact,
    check_all_ones,
    check_overflow,
    check_identity,
    check_zero_operands,
    check_nonnegative,
    check_exact_rational_bound,
    check_sequential_fp32_tiny,
    check_rows_and_threads,
    check_ex_dense_equals_base,
    check_ex_weight_layout,
    check_ex_transposed_a,
    check_ex_strides,
    check_ex_bias_exact,
    check_ex_bias_closed_form,
    check_fp8_decode_all_codes,
    check_ue8m0_decode_all_codes,
    check_bf16_rne_vs_torch,
    check_bf16_rne_edges,
    check_mxf8_exact_rational_tiny,
    check_mxf8_integer_exact,
    check_mxf8_identity_and_groups,
    check_mxf8_scale_invariance,
    check_mxf8_relu_and_nan,
    check_e2m1_decode_golden,
    check_ue4m3_decode,
    check_nvf4_integer_exact,
    check_nvf4_identity_nibble_order,
    check_nvf4_exact_rational_tiny,
    check_nvf4_alpha_relu,
    check_dequant_all_codes_all_scales,
    check_dequant_groups_and_nibbles,
    check_w4a16_gemm_integer_exact,
]
