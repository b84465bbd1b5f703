/*
 * oracle.c -- CPU oracle for C = ReLU(A . B) with fp16 operands, fp32
 * accumulation and an fp16 result.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * What it computes (the quick-start matmul_relu kernel, "TileLang" wiki page,
 * section "Programming model"):
 *   - A is an M x K fp16 tensor and B is a K x N fp16 tensor; C is a fresh
 *     M x N fp16 tensor (the kernel's tensor declarations).  All three are
 *     dense and row-major: element (r, c) of an R x S matrix sits at r*S + c.
 *   - The accumulator is an fp32 fragment (alloc_fragment of float32) that is
 *     cleared to zero (T.clear) before the K loop.
 *   - The K loop walks ceildiv(K, block_K) tiles and accumulates the tile
 *     products (T.gemm).  Tiling only partitions the sum, so the plain
 *     definition is the full sum over k = 0 .. K-1.
 *   - The epilogue takes max(C_local, 0) on the fp32 values, then T.copy
 *     writes them into the fp16 output, which converts fp32 -> fp16.
 *
 * Readings where the page is silent (each one is listed in the design notes):
 *   - Accumulation is IEEE fp32, sequential in k = 0, 1, ..., K-1, with
 *     round-to-nearest-even at every add.  Every fp16 x fp16 product is exact
 *     in fp32 (11-bit x 11-bit significands need at most 22 bits), so the
 *     only rounding in the loop is in the adds, and a fused multiply-add would
 *     give the same bits.
 *   - The fp32 -> fp16 conversion is IEEE 754 round-to-nearest, ties to even,
 *     with gradual underflow and overflow to +inf.
 *   - ReLU maps every value that is not > 0 (negative values, -0 and NaN) to
 *     +0, so the output never carries the bit pattern 0x8000.
 *
 * Parity pins: every function here is pinned by tests that do not run this
 * code's arithmetic a second time (numpy's independent float16 conversion on
 * all 65536 halves and on random and edge fp32 values, hand-derived IEEE 754
 * edge values, exact integer matrix products, exact rational sums with the
 * standard fp32 summation error bound, and closed forms such as identity and
 * all-ones matrices).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * binary16 -> binary32, from the IEEE 754 binary16 definition:
 *   exponent field 0      : value = (-1)^s * frac * 2^-24   (zero, subnormal)
 *   exponent field 1..30  : value = (-1)^s * (1024 + frac) * 2^(e - 25)
 *   exponent field 31     : +-inf (frac == 0) or NaN
 * ldexpf of an integer below 2^11 is exact.
 */
float oracle_f16_to_f32(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int expo = (h >> 10) & 0x1f;
    const int frac = h & 0x3ff;
    float mag;
    if (expo == 0)
        mag = ldexpf((float)frac, -24);
    else if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexpf((float)(1024 + frac), expo - 25);
    return sign ? -mag : mag;
}

/*
 * binary32 -> binary16, round to nearest, ties to even.
 * The value's fp16 quantum is 2^(e-10) for |x| in [2^e, 2^(e+1)), e >= -14,
 * and 2^-24 below 2^-14.  |x| / quantum is computed exactly in double (a
 * float has 24 significant bits), rounded to an integer q with ties to even,
 * and q * quantum is encoded.  A value that rounds to 2^16 or above is out of
 * range and becomes inf.
 */
uint16_t oracle_f32_to_f16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(x))
        return (uint16_t)(sign | 0x7e00u);
    const double a = fabs((double)x);
    if (isinf(x))
        return (uint16_t)(sign | 0x7c00u);
    if (a == 0.0)
        return sign;

    int e2;
    (void)frexp(a, &e2); /* a = m * 2^e2 with m in [0.5, 1): 2^(e2-1) <= a */
    int e = e2 - 1;      /* a in [2^e, 2^(e+1)) */
    const int subnormal = e < -14;
    const int qexp = subnormal ? -24 : e - 10; /* quantum = 2^qexp */

    const double q = ldexp(a, -qexp); /* exact */
    double qi = floor(q);
    const double r = q - qi; /* exact */
    if (r > 0.5 || (r == 0.5 && fmod(qi, 2.0) != 0.0))
        qi += 1.0;
    long qn = (long)qi;

    if (subnormal) {
        /* qn in [0, 1024]; 1024 is the smallest normal, 2^-14. */
        if (qn == 1024)
            return (uint16_t)(sign | (1u << 10));
        return (uint16_t)(sign | (uint16_t)qn);
    }
    /* qn in [1024, 2048]; 2048 carries into the next binade. */
    if (qn == 2048) {
        qn = 1024;
        e += 1;
    }
    if (e > 15)
        return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(qn - 1024));
}

/* Element-wise helpers over arrays, for the tests. */
void oracle_f16_to_f32_array(const uint16_t *h, float *f, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        f[i] = oracle_f16_to_f32(h[i]);
}

void oracle_f32_to_f16_rne_array(const float *f, uint16_t *h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_f32_to_f16_rne(f[i]);
}

/*
 * C[i, j] = f16_rne( relu( sum_{k=0}^{K-1} f32(A[i, k]) * f32(B[k, j]) ) )
 *
 * A: M x K, B: K x N, C: M x N, all row-major fp16 bit patterns.
 * The sum for each (i, j) runs in k order with an fp32 accumulator.  The
 * loop nest is i, k, j: a row of accumulators acc[0..N) is cleared, then for
 * each k the row acc += A[i,k] * B[k, :] is added; the order of the adds into
 * any one acc[j] is still k = 0, 1, ..., K-1.  Rows i are independent, so
 * splitting them over threads changes no rounding.
 *
 * nthreads <= 0 means "whatever OpenMP picks".  Returns 0 on success and -1
 * if a work buffer cannot be allocated.
 */
int oracle_gemm_relu_f16(const uint16_t *A, const uint16_t *B, uint16_t *C,
                         int64_t M, int64_t N, int64_t K, int nthreads)
{
    if (M <= 0 || N <= 0)
        return 0;

    /* Widen B once: B[k, j] -> Bf[k*N + j]. */
    float *Bf = NULL;
    if (K > 0) {
        Bf = (float *)malloc((size_t)K * (size_t)N * sizeof(float));
        if (!Bf)
            return -1;
        oracle_f16_to_f32_array(B, Bf, K * N);
    }

    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        float *acc = (float *)malloc((size_t)N * sizeof(float));
        if (!acc) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t i = 0; i < M; ++i) {
            if (!acc)
                continue;
            for (int64_t j = 0; j < N; ++j)
                acc[j] = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                const float a = oracle_f16_to_f32(A[i * K + k]);
                const float *brow = Bf + k * N;
                for (int64_t j = 0; j < N; ++j)
                    acc[j] = acc[j] + a * brow[j];
            }
            for (int64_t j = 0; j < N; ++j) {
                const float v = acc[j] > 0.0f ? acc[j] : 0.0f;
                C[i * N + j] = oracle_f32_to_f16_rne(v);
            }
        }
        free(acc);
    }
    free(Bf);
    return failed ? -1 : 0;
}

/*
 * General layouts and a per-column bias:
 *
 *   C[i*ldc + j] = f16_rne( relu( fp32( sum_k a(i,k) * b(k,j) ) + f32(bias[j]) ) )
 *
 * with a(i,k) = A[i*lda + k] when a_km == 0 (A stored M x K) and A[k*lda + i]
 * when a_km == 1 (A stored K x M, so C = A^T . B); b(k,j) = B[k*ldb + j] when
 * b_nk == 0 (B stored K x N) and B[j*ldb + k] when b_nk == 1 (B stored N x K,
 * so C = A . B^T);
 * bias may be NULL (no bias term).  The sum runs in k order with an fp32
 * accumulator exactly as in oracle_gemm_relu_f16; the bias is added to the
 * finished sum with one fp32 addition, then ReLU, then the fp16 rounding.
 * Elements of C outside the M x N block (padding of ldc) are not written.
 * Returns 0, or -1 if a work buffer cannot be allocated.
 */
int oracle_gemm_relu_f16_ex(const uint16_t *A, const uint16_t *B, uint16_t *C, int64_t M, int64_t N,
                            int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int a_km, int b_nk,
                            const uint16_t *bias, int nthreads)
{
    if (M <= 0 || N <= 0)
        return 0;

    /* Widen B once into the K x N order the i-k-j loop walks: Bf[k*N + j]. */
    float *Bf = NULL;
    if (K > 0) {
        Bf = (float *)malloc((size_t)K * (size_t)N * sizeof(float));
        if (!Bf)
            return -1;
        for (int64_t k = 0; k < K; ++k)
            for (int64_t j = 0; j < N; ++j)
                Bf[k * N + j] = oracle_f16_to_f32(b_nk ? B[j * ldb + k] : B[k * ldb + j]);
    }

    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        float *acc = (float *)malloc((size_t)N * sizeof(float));
        if (!acc) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t i = 0; i < M; ++i) {
            if (!acc)
                continue;
            for (int64_t j = 0; j < N; ++j)
                acc[j] = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                const float a = oracle_f16_to_f32(a_km ? A[k * lda + i] : A[i * lda + k]);
                const float *brow = Bf + k * N;
                for (int64_t j = 0; j < N; ++j)
                    acc[j] = acc[j] + a * brow[j];
            }
            for (int64_t j = 0; j < N; ++j) {
                const float y = bias ? acc[j] + oracle_f16_to_f32(bias[j]) : acc[j];
                const float v = y > 0.0f ? y : 0.0f;
                C[i * ldc + j] = oracle_f32_to_f16_rne(v);
            }
        }
        free(acc);
    }
    free(Bf);
    return failed ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * MXFP8 block-scaled grouped GEMM (the "Blackwell MXFP8 grouped GEMM with
 * block scaling + transposed B matrix" milestone, page 3, "Key Technical
 * Milestones").  The page names the operation only; its number formats are
 * the OCP Microscaling (MX) v1.0 definitions, which is the reading taken:
 *   - elements are FP8 E4M3 ("fn": no infinities, S.1111.111 is NaN, bias 7)
 *     or FP8 E5M2 (IEEE-style, bias 15, exponent 31 is inf/NaN);
 *   - every 32 consecutive elements along K share one UE8M0 scale, the
 *     power of two 2^(e - 127), with e = 255 meaning NaN;
 *   - a scaled element is value(code) * scale, so one output is
 *       sum over k of (a[i,k] * sa[i, k/32]) * (b[j,k] * sb[j, k/32]).
 * B is "transposed": each group's weight is stored N x K (rows of length K).
 * Readings where the page is silent: the sum is formed in double precision
 * (every product of two scaled fp8 values is exact in double; the only
 * rounding is in the adds, far below the output's precision); an optional
 * ReLU maps every value not > 0 to +0; the result is rounded once to
 * bfloat16, round to nearest, ties to even, overflow to +inf.
 * ------------------------------------------------------------------------ */

/* FP8 code -> value.  format 0: E4M3 (fn), format 1: E5M2. */
double oracle_fp8_to_f64(uint8_t code, int format)
{
    const int sign = code >> 7;
    double mag;
    if (format == 0) {
        const int e = (code >> 3) & 0xf, m = code & 0x7;
        if (e == 15 && m == 7)
            return NAN;
        mag = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10); /* (1 + m/8) 2^(e-7) */
    } else {
        const int e = (code >> 2) & 0x1f, m = code & 0x3;
        if (e == 31)
            return m ? NAN : (sign ? -INFINITY : INFINITY);
        mag = e == 0 ? ldexp((double)m, -16) : ldexp((double)(4 + m), e - 17); /* (1 + m/4) 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* UE8M0 scale code -> 2^(e - 127); 255 is NaN. */
double oracle_ue8m0_to_f64(uint8_t e)
{
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

/*
 * double -> bfloat16 bits, round to nearest, ties to even (one rounding).
 * bfloat16 has 8 significant bits and fp32's exponent range: for |x| in
 * [2^e, 2^(e+1)), e >= -126, the quantum is 2^(e-7); below 2^-126 it is
 * 2^-133.  A value that rounds to 2^128 or above becomes inf.
 */
uint16_t oracle_f64_to_bf16_rne(double x)
{
    if (isnan(x))
        return 0x7fc0u;
    const uint16_t sign = signbit(x) ? 0x8000u : 0;
    const double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | 0x7f80u);
    if (a == 0.0)
        return sign;
    int e2;
    (void)frexp(a, &e2);
    int e = e2 - 1; /* a in [2^e, 2^(e+1)) */
    const int subnormal = e < -126;
    const int qexp = subnormal ? -133 : e - 7;
    const double q = ldexp(a, -qexp); /* exact: a scaling by a power of two */
    double qi = floor(q);
    const double r = q - qi;
    if (r > 0.5 || (r == 0.5 && fmod(qi, 2.0) != 0.0))
        qi += 1.0;
    long qn = (long)qi;
    if (subnormal) {
        if (qn == 128) /* rounds up to the smallest normal, 2^-126 */
            return (uint16_t)(sign | (1u << 7));
        return (uint16_t)(sign | (uint16_t)qn);
    }
    if (qn == 256) {
        qn = 128;
        e += 1;
    }
    if (e > 127)
        return (uint16_t)(sign | 0x7f80u);
    return (uint16_t)(sign | (uint16_t)((e + 127) << 7) | (uint16_t)(qn - 128));
}

/*
 * Grouped, block-scaled GEMM over G groups that share N and K:
 *
 *   C[r*N + j] = bf16_rne( [relu]( sum_{k<K} a(r,k) sa(r,k/32) * b_g(j,k) sb_g(j,k/32) ) )
 *
 * for the rows r = row_offset[g] .. row_offset[g] + m_sizes[g] - 1 of group g:
 *   a(r,k)   = fp8(A[r*K + k], a_format)            A: stacked rows x K codes
 *   sa(r,s)  = ue8m0(SFA[r*(K/32) + s])             plain row-major scales
 *   b_g(j,k) = fp8(B[(g*N + j)*K + k], b_format)    B: G x N x K codes
 *   sb_g(j,s)= ue8m0(SFB[(g*N + j)*(K/32) + s])
 * K must be a multiple of 32.  Rows of C outside every group are not
 * written.  The sum for one output is taken in k order in double.  Returns
 * 0, or -1 on bad arguments.
 */
int oracle_gemm_mxf8_grouped(const uint8_t *A, const uint8_t *SFA, const uint8_t *B, const uint8_t *SFB,
                             uint16_t *C, const int64_t *row_offset, const int64_t *m_sizes, int G, int64_t N,
                             int64_t K, int a_format, int b_format, int relu, int nthreads)
{
    if (K % 32 != 0 || N < 0 || G < 0)
        return -1;
    const int64_t S = K / 32;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#else
    (void)nthreads;
#endif
    for (int g = 0; g < G; ++g) {
        const int64_t r0 = row_offset[g], mg = m_sizes[g];
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
        for (int64_t i = 0; i < mg; ++i) {
            const int64_t r = r0 + i;
            for (int64_t j = 0; j < N; ++j) {
                const int64_t brow = (int64_t)g * N + j;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const double av = oracle_fp8_to_f64(A[r * K + k], a_format) * oracle_ue8m0_to_f64(SFA[r * S + k / 32]);
                    const double bv = oracle_fp8_to_f64(B[brow * K + k], b_format) * oracle_ue8m0_to_f64(SFB[brow * S + k / 32]);
                    acc += av * bv;
                }
                const double y = relu ? (acc > 0.0 ? acc : 0.0) : acc;
                C[r * N + j] = oracle_f64_to_bf16_rne(y);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * NVF4 block-scaled grouped GEMM (the NVF4 block-scaled MMA path whose
 * 8192^3 throughput the tilelang-ai project page quotes, "Three backends
 * under one language dialect").  The page names the operation only; the
 * reading taken is NVIDIA's NVFP4 format:
 *   - elements are FP4 E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa
 *     bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), two per byte,
 *     element 2i in the low nibble and element 2i+1 in the high nibble;
 *   - every 16 consecutive elements along K share one scale, an FP8 E4M3
 *     value with its sign bit clear (UE4M3);
 *   - one fp32 factor alpha multiplies the whole sum (the per-tensor scale);
 *   - sum in double, optional ReLU, one RNE rounding to bfloat16, as above.
 * ------------------------------------------------------------------------ */

/* E2M1 code (low 4 bits of `code`) -> value. */
double oracle_e2m1_to_f64(uint8_t code)
{
    const int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* UE4M3 scale code -> value: the E4M3 value of a code with the sign bit
 * clear; a set sign bit is not a valid scale (NaN here). */
double oracle_ue4m3_to_f64(uint8_t code)
{
    return (code & 0x80) ? NAN : oracle_fp8_to_f64(code, 0);
}

/*
 *   C[r*N + j] = bf16_rne( [relu]( alpha * sum_{k<K} a(r,k) sa(r,k/16) * b_g(j,k) sb_g(j,k/16) ) )
 *
 * for the rows r = row_offset[g] .. + m_sizes[g] - 1 of group g, with
 *   a(r,k)    = e2m1(nibble k of row r of A)   A: stacked rows x K/2 bytes
 *   sa(r,s)   = ue4m3(SFA[r*(K/16) + s])
 *   b_g(j,k)  = e2m1(nibble k of row g*N + j of B)   B: G x N x K/2 bytes
 *   sb_g(j,s) = ue4m3(SFB[(g*N + j)*(K/16) + s])
 * where nibble k of a row is the low half of byte k/2 for even k and the
 * high half for odd k.  K must be a multiple of 16.  Returns 0, or -1 on bad
 * arguments.
 */
int oracle_gemm_nvf4_grouped(const uint8_t *A, const uint8_t *SFA, const uint8_t *B, const uint8_t *SFB, uint16_t *C,
                             const int64_t *row_offset, const int64_t *m_sizes, int G, int64_t N, int64_t K,
                             double alpha, int relu, int nthreads)
{
    if (K % 16 != 0 || N < 0 || G < 0)
        return -1;
    const int64_t S = K / 16, KB = K / 2;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#else
    (void)nthreads;
#endif
    for (int g = 0; g < G; ++g) {
        const int64_t r0 = row_offset[g], mg = m_sizes[g];
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
        for (int64_t i = 0; i < mg; ++i) {
            const int64_t r = r0 + i;
            for (int64_t j = 0; j < N; ++j) {
                const int64_t brow = (int64_t)g * N + j;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const int hi = (int)(k & 1);
                    const uint8_t abyte = A[r * KB + k / 2], bbyte = B[brow * KB + k / 2];
                    const double av = oracle_e2m1_to_f64(hi ? (uint8_t)(abyte >> 4) : (uint8_t)(abyte & 0xf)) *
                                      oracle_ue4m3_to_f64(SFA[r * S + k / 16]);
                    const double bv = oracle_e2m1_to_f64(hi ? (uint8_t)(bbyte >> 4) : (uint8_t)(bbyte & 0xf)) *
                                      oracle_ue4m3_to_f64(SFB[brow * S + k / 16]);
                    acc += av * bv;
                }
                const double y = alpha * acc;
                C[r * N + j] = oracle_f64_to_bf16_rne(relu ? (y > 0.0 ? y : 0.0) : y);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Dequantized (low-bit weight) GEMM: the dequantize_gemm workload that the
 * TileLang pages name among the kernels the language targets (aiwiki.ai
 * "TileLang", opening paragraph; the BitBLAS dequantized-GEMM comparisons
 * under "Ecosystem").  The pages name the operation only; the reading taken
 * is the common 4-bit weight-only scheme (W4A16):
 *   - the weight W is N x K, stored as 4-bit codes q in 0..15, two per byte,
 *     element 2i of a row in the low nibble (as for NVF4 above);
 *   - each run of `group` consecutive elements of a weight row along K shares
 *     one fp16 scale s; the zero point is the fixed code 8, so a weight is
 *     (q - 8) * s;
 *   - the dequantized weight is rounded to fp16 (the type the fp16 GEMM
 *     consumes): w = f16_rne((q - 8) * s), the exact product rounded once;
 *   - the GEMM is then the base operation with the weight in the linear-layer
 *     layout: C = ReLU(A . W^T), fp32 accumulation, fp16 output
 *     (oracle_gemm_relu_f16_ex with b_nk = 1).
 * ------------------------------------------------------------------------ */

/*
 * W[n*K + k] = f16_rne( (q(n,k) - 8) * f32(S[n*(K/group) + k/group]) ) for the
 * N x K weight, with q(n,k) nibble k of row n of Wq (rows of K/2 bytes).  The
 * product of an integer in -8..7 and an fp16 value is exact in fp32, so one
 * rounding happens.  K must be a multiple of `group` and of 2.  Returns 0, or
 * -1 on bad arguments.
 */
int oracle_dequant_w4_f16(const uint8_t *Wq, const uint16_t *S, uint16_t *W, int64_t N, int64_t K, int64_t group)
{
    if (N < 0 || K < 0 || group <= 0 || K % group != 0 || K % 2 != 0)
        return -1;
    const int64_t G = K / group;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            const uint8_t byte = Wq[n * (K / 2) + k / 2];
            const int q = (k & 1) ? (byte >> 4) : (byte & 0xf);
            const float scale = oracle_f16_to_f32(S[n * G + k / group]);
            W[n * K + k] = oracle_f32_to_f16_rne((float)(q - 8) * scale);
        }
    }
    return 0;
}

/* Number of threads OpenMP would use by default (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
