/*
 * tg_gemm.h -- C ABI of the B200 (sm_100a) tiled fp16 GEMM + ReLU library.
 *
 * The operation (the matmul_relu quick-start kernel, "TileLang" wiki page,
 * section "Programming model"):
 *
 *     C[i, j] = fp16( max( sum_k fp32(A[i, k]) * fp32(B[k, j]), 0 ) )
 *
 * with A an M x K fp16 matrix, B a K x N fp16 matrix, an fp32 accumulator
 * that starts at zero, ReLU applied to the fp32 value, and the result rounded
 * to fp16 (round to nearest, ties to even; values >= 65520 become +inf).
 * ReLU maps every value that is not > 0 (including -0 and NaN) to +0.  The
 * order in which the tensor cores add the K products is not specified, so
 * for non-integer inputs results agree with a sequential fp32 sum up to
 * rounding; integer-valued inputs whose partial sums stay below 2^24 give
 * bit-identical results.
 *
 * Layout: A, B and C are dense and row-major (leading dimensions K, N and N
 * elements), fp16 (IEEE binary16), in device memory of the current CUDA
 * device.  The caller owns all three buffers and the library keeps no
 * pointer to them after a call returns.  No call allocates or frees device
 * memory at run time.  Scratch memory comes from two places:
 *   - the caller: tg_gemm_relu_f16_ws, tg_gemm_relu_f16_ex and
 *     tg_gemm_relu_w4a16 take an optional (or, for some layouts, required)
 *     workspace pointer and size;
 *   - one fixed module buffer of TG_STATIC_WORKSPACE_BYTES (16 MiB) that the
 *     library holds on every GPU where it is loaded, until the process
 *     exits; only tg_gemm_relu_f16_static_ws uses it.
 * tg_gemm_relu_f16 itself needs no scratch.
 *
 * Threading and streams: calls are asynchronous on `stream` (a cudaStream_t
 * passed as void*; NULL is the legacy default stream).  On TG_OK the work is
 * enqueued; on any error nothing was enqueued.  The functions are
 * thread-safe.
 *
 * Device: NVIDIA B200 class GPU, compute capability 10.0 (sm_100a).
 */
#ifndef TG_GEMM_H
#define TG_GEMM_H

#include <stdint.h>

#if defined(__GNUC__)
#define TG_API __attribute__((visibility("default")))
#else
#define TG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tg_status {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,        /* bad pointer, size, alignment or overlap    */
    TG_ERR_UNSUPPORTED_DEVICE = 2, /* no device, or not compute capability 10.0 */
    TG_ERR_LAUNCH = 3,             /* a kernel launch or CUDA call failed         */
    TG_ERR_TIMEOUT = 4,            /* a bounded device-side wait ran out          */
    TG_ERR_INTERNAL = 5,           /* invariant broken inside the library         */
    TG_ERR_TOO_LARGE = 6           /* needs more scratch than the library's fixed
                                      device buffer holds (tg_gemm_relu_f16_static_ws) */
} tg_status;

/* Kernel paths.  TG_PATH_AUTO lets the dispatcher choose (see
 * tg_select_path); the others force one kernel, for tests and tuning. */
typedef enum tg_path {
    TG_PATH_NONE = -1,   /* nothing to launch: M == 0 or N == 0            */
    TG_PATH_AUTO = 0,
    TG_PATH_TC = 1,      /* TMA + tcgen05 persistent kernel, 128x256 tiles;
                            needs K % 8 == 0, N % 8 == 0 and 16-byte
                            aligned A and B (any 2-byte aligned C)          */
    TG_PATH_TC_EDGE = 2, /* same kernel, operands staged by predicated
                            loads: any K, N and 2-byte alignment            */
    TG_PATH_SKINNY = 3,  /* small-M split-K tcgen05 kernel (computes
                            C^T = B^T A^T), M <= 256 (this kernel also
                            serves M = 1); same alignment needs as TC       */
    TG_PATH_ZERO = 5,    /* K == 0: C is filled with +0 (empty sum)         */
    TG_PATH_TC_PAIR = 6, /* the TMA + tcgen05 kernel on SM pairs
                            (cta_group::2), 256x256 tiles; same alignment
                            needs as TC                                     */
    TG_PATH_TC_PAIR512 = 7, /* as TC_PAIR with 256x512 tiles                */
    TG_PATH_REPACK = 8,  /* operands TMA cannot describe are first copied
                            into zero-padded rows in the caller's workspace,
                            then a TMA kernel runs (tg_gemm_relu_f16_ws)    */
    TG_PATH_RC = 9       /* no scratch, any 2-byte alignment of A, B and C:
                            A's rows are loaded by TMA in residue classes
                            (row mod 8, rows sharing one 16-byte offset),
                            B's k-rows shifted to match; B's rows read in
                            place and realigned into the operand tile when
                            TMA cannot describe them; A stored M x K,
                            B stored K x N only                              */
} tg_path;

/*
 * C = ReLU(A . B).  (tg_gemm_relu_f16_ex below adds strides, the N x K
 * layout of B, a bias and batches.)
 *   A      device pointer, M x K fp16, row-major (may be NULL if M*K == 0)
 *   B      device pointer, K x N fp16, row-major (may be NULL if K*N == 0)
 *   C      device pointer, M x N fp16, row-major, written in full; must not
 *          overlap A or B (may be NULL if M*N == 0)
 *   M,N,K  sizes, each in [0, 2^31 - 1]
 *   stream cudaStream_t as void*
 * Returns TG_OK, or TG_ERR_INVALID_ARG (negative or too large size, NULL
 * pointer with a non-empty matrix, pointer not 2-byte aligned, C overlapping
 * A or B), TG_ERR_UNSUPPORTED_DEVICE or TG_ERR_LAUNCH.  M == 0 or N == 0 is
 * TG_OK with nothing enqueued; K == 0 fills C with +0.
 */
TG_API tg_status tg_gemm_relu_f16(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                           void *stream);

/*
 * As tg_gemm_relu_f16, with the kernel path forced (a tg_path value).
 * Forcing a path whose requirements the arguments do not meet returns
 * TG_ERR_INVALID_ARG, and so does TG_PATH_REPACK (it needs a workspace: use
 * tg_gemm_relu_f16_ws).  TG_PATH_AUTO behaves like tg_gemm_relu_f16.
 */
TG_API tg_status tg_gemm_relu_f16_path(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                                void *stream, int path);

/*
 * C = ReLU(A . B) with a caller-provided device workspace.  Identical to
 * tg_gemm_relu_f16 except where the workspace lets a faster route run:
 *   - TMA cannot describe A or B (a row stride that is not a multiple of 16
 *     bytes, or a base that is not 16-byte aligned).  Where the residue-class
 *     kernel takes them (1/N + 1/K > 1/2400, TG_PATH_RC), B alone is first
 *     copied into zero-padded rows in the workspace and loaded by TMA, except
 *     where realigning B in place is the faster route (tiles narrower than
 *     256 columns, 32 or more k-blocks per CTA, B's tile no wider than the
 *     tile's rows of A): then nothing is copied.  Elsewhere (TG_PATH_REPACK)
 *     A and B are copied into zero-padded rows and a TMA kernel runs on the
 *     copies;
 *   - the rows of C are not 16-byte aligned, M > 256, and the workspace also
 *     holds a padded C (tg_workspace_size covers it): the GEMM writes that
 *     copy with its aligned stores and a realigning copy moves it into C.
 * With less workspace the call behaves like tg_gemm_relu_f16.
 *   workspace        device pointer, 256-byte aligned, not overlapping A, B
 *                    or C; owned by the caller and free to reuse once the
 *                    call's work on `stream` has finished (may be NULL if
 *                    workspace_bytes == 0)
 *   workspace_bytes  size of the workspace in bytes
 * Errors as tg_gemm_relu_f16, plus TG_ERR_INVALID_ARG for a misaligned or
 * overlapping workspace, or a negative size.
 */
TG_API tg_status tg_gemm_relu_f16_ws(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                                     void *stream, void *workspace, int64_t workspace_bytes);

/*
 * C = ReLU(A . B) for callers that cannot allocate device memory at all --
 * code running where cudaMalloc is off limits (an allocator-free runtime, a
 * process whose memory budget is fixed up front, a plugin that must not grow
 * the device footprint) -- but still want the fast repack path for operands
 * TMA cannot describe.  The paper has no counterpart to this entry point.
 *
 * It behaves like tg_gemm_relu_f16_ws, with the workspace taken from a fixed
 * device buffer of TG_STATIC_WORKSPACE_BYTES (16 MiB) that the library holds
 * on every GPU where it is loaded, until the process exits.  It calls no
 * allocating routine.  The caller still passes A, B and C.
 *   - Problems whose copies of A and B would need more than
 *     TG_STATIC_WORKSPACE_BYTES are rejected with TG_ERR_TOO_LARGE and
 *     nothing is enqueued; problems whose A and B TMA can describe need no
 *     scratch and always run.  The padded C of tg_gemm_relu_f16_ws is used
 *     only when it fits in the buffer beside those copies.
 *   - The first call on a device looks up the buffer's device address for
 *     that device (with that device current); make that first call before
 *     any stream capture.
 *   - Every call shares the one buffer.  Calls whose work can overlap on the
 *     GPU (different streams, or different host threads) race on it: order
 *     them on one stream or synchronise between them.  Each call writes every
 *     scratch byte it reads before reading it, so nothing needs clearing.
 */
#define TG_STATIC_WORKSPACE_BYTES (16ll * 1024 * 1024)
TG_API tg_status tg_gemm_relu_f16_static_ws(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                                            void *stream);

/*
 * General operand layouts, a fused bias and strided batches.
 *
 * For each batch entry e = 0 .. batch-1:
 *
 *   C_e[i*ldc + j] = fp16( max( sum_k a_e(i, k) * b_e(k, j) + bias[j], 0 ) )
 *
 * with A_e = A + e*stride_a, B_e = B + e*stride_b, C_e = C + e*stride_c
 * (element offsets); a_e(i, k) = A_e[i*lda + k] when A is stored M x K
 * (TG_A_MK) or A_e[k*lda + i] when it is stored K x M (TG_A_KM: C = A^T . B);
 * b_e(k, j) = B_e[k*ldb + j] when B is stored K x N (TG_B_KN) or
 * B_e[j*ldb + k] when it is stored N x K (TG_B_NK, the layout of a linear
 * layer's weight: C = A . W^T).  The sum is accumulated in fp32;
 * the bias (fp16, N values, optional) is added to it in fp32 before ReLU.
 * This widens the quick-start kernel's dense row-major operands to the
 * layouts its T.gemm tile operator accepts ("TileLang" wiki page,
 * "Programming model": layouts inferred per operand; symbolic shapes).
 *
 * A zero-initialised tg_gemm_options (or NULL) means: dense row-major A, B
 * (K x N) and C, no bias, one problem, automatic kernel choice.
 */
enum { TG_A_MK = 0, TG_A_KM = 1 };
enum { TG_B_KN = 0, TG_B_NK = 1 };

typedef struct tg_gemm_options {
    int64_t lda;        /* elements between rows of A as stored; 0 = K (TG_A_MK)
                           or M (TG_A_KM); must be at least that                */
    int64_t ldb;        /* elements between rows of B as stored; 0 = N (TG_B_KN)
                           or K (TG_B_NK); must be at least that                */
    int64_t ldc;        /* elements between rows of C; 0 = N; must be >= N        */
    int32_t a_layout;   /* TG_A_MK or TG_A_KM                                    */
    int32_t b_layout;   /* TG_B_KN or TG_B_NK                                    */
    int32_t path;       /* TG_PATH_AUTO (0) or a forced kernel path (testing)     */
    int32_t reserved;   /* must be 0                                             */
    const void *bias;   /* device fp16[N], or NULL                                */
    int64_t batch;      /* number of problems; 0 = 1                             */
    int64_t stride_a;   /* elements between consecutive A, B and C entries;     */
    int64_t stride_b;   /* C entries must not overlap each other                */
    int64_t stride_c;
} tg_gemm_options;

/*
 * C = ReLU(A . B + bias) with the layouts and batching of `options`.
 * Operands TMA cannot describe (row or batch strides that are not multiples
 * of 8 elements, bases that are not 16-byte aligned) take, for A stored M x K
 * with B stored K x N, the residue-class kernel (with B's padded copy when
 * the workspace holds it and the rule of tg_gemm_relu_f16_ws asks for it) or
 * the repack path; the other layouts need the repack path's workspace
 * (tg_workspace_size_ex) and are refused without it (TG_ERR_INVALID_ARG).  A stored K x M runs on the
 * 128- and 256-row tensor-core kernels (not the small-M kernel).  Batch entries run in order on `stream` and share the
 * workspace.  Errors as tg_gemm_relu_f16_ws, plus TG_ERR_INVALID_ARG for
 * strides below the row lengths, overlapping C entries, an unknown b_layout
 * or a forced path that cannot run these operands.
 */
TG_API tg_status tg_gemm_relu_f16_ex(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                                     const tg_gemm_options *options, void *stream, void *workspace,
                                     int64_t workspace_bytes);

/* Workspace bytes tg_gemm_relu_f16_ex needs for its repack path (0: none;
 * -1: invalid arguments).  Host logic only. */
TG_API int64_t tg_workspace_size_ex(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K,
                                    const tg_gemm_options *options);

/* The path tg_gemm_relu_f16_ex takes with `workspace_bytes` of workspace
 * (-2: invalid arguments).  Host logic only. */
TG_API int tg_select_path_ex(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K,
                             const tg_gemm_options *options, int64_t workspace_bytes);

/*
 * Workspace bytes tg_gemm_relu_f16_ws needs for its fastest path with these
 * arguments: when TMA cannot describe A or B, B's padded copy on the
 * residue-class route (or nothing, where B is realigned in place; see
 * tg_gemm_relu_f16_ws), else copies of A and B, plus, when the rows of C are
 * not 16-byte aligned and a tensor-core kernel runs (M > 256), a padded C
 * that the GEMM writes and a realigning copy moves into C.  Less workspace
 * still takes the repack path as long as the A and B copies fit.  0 when
 * none applies, -1 for invalid arguments.  Host logic only (it assumes the
 * 148 SMs of a B200 where the choice depends on the SM count).
 */
TG_API int64_t tg_workspace_size(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K);

/* The path tg_gemm_relu_f16_ws would take with `workspace_bytes` of workspace. */
TG_API int tg_select_path_ws(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K,
                             int64_t workspace_bytes);

/*
 * The path tg_gemm_relu_f16 would take for these arguments (a tg_path value;
 * TG_PATH_NONE for an empty C), or -2 when the arguments are invalid.  Host
 * logic only: makes no CUDA call and needs no GPU.  Rules: K == 0 -> ZERO;
 * A or B rows not TMA-describable (strides or bases off 16 bytes) -> RC;
 * M <= 128, or M <= 256 with N * K >= 2^23 -> SKINNY; otherwise the
 * tensor-core kernel (TC, TC_PAIR or TC_PAIR512) with the least estimated
 * time from its tile count in waves of a 148-SM device.
 */
TG_API int tg_select_path(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K);

/*
 * Whether `path` can run these arguments (1) or not (0).  Host logic only.
 */
TG_API int tg_path_supports(int path, const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K);

/*
 * Synchronizes the current device, then reads and clears the library's
 * device-side error word.  Returns TG_OK, TG_ERR_TIMEOUT if a bounded wait
 * inside a kernel gave up since the last call (the kernel then stopped early
 * and its output is incomplete), or TG_ERR_LAUNCH if the device reported an
 * error.  `detail` (may be NULL) receives the raw error word.
 */
TG_API tg_status tg_device_status(uint32_t *detail);

/*
 * Failure-detection self-test: launches one CTA on `stream` that waits on an
 * mbarrier nothing will ever arrive on, with a budget of `budget_ns`
 * nanoseconds (clamped to [1e3, 1e10]).  The wait gives up, records
 * TG_ERR_TIMEOUT in the device error word and the kernel returns normally;
 * tg_device_status() then reports it.  No trap, no fault, no hang.
 */
TG_API tg_status tg_wait_timeout_selftest(int64_t budget_ns, void *stream);

/* Static description of a status or path value. */
TG_API const char *tg_status_string(int status);
TG_API const char *tg_path_name(int path);

/* Library version, major * 10000 + minor * 100 + patch. */
TG_API int tg_version(void);

/* ---------------------------------------------------------------------------
 * MXFP8 block-scaled grouped GEMM
 *
 * The Blackwell "MXFP8 grouped GEMM with block scaling + transposed B matrix"
 * (zhichai.net TileLang topic page, "Key Technical Milestones"), with the
 * number formats of the OCP Microscaling (MX) definitions.  For G groups that
 * share N and K, group g owning m_sizes[g] rows:
 *
 *   C[r*N + j] = bf16( [relu]( sum_{k<K} a(r,k) sa(r,k/32) * b_g(j,k) sb_g(j,k/32) ) )
 *
 * A: stacked rows x K fp8 codes, row-major (K-major).  Group g's rows start at
 *    row o_g = sum_{h<g} roundup(m_sizes[h], 128): every group starts on a
 *    multiple of 128 rows.  rows = tg_mx_grouped_rows(m_sizes, G).  Rows
 *    between groups are read but do not affect C.
 * B: G x N x K fp8 codes; group g's weight is stored N x K (transposed B).
 * a(r,k), b_g(j,k): E4M3 (TG_FP8_E4M3, OCP "fn": no inf, 0x7F/0xFF NaN) or
 *    E5M2 (TG_FP8_E5M2) values, chosen per operand.
 * SFA, SFB: UE8M0 scales (2^(e-127); 255 = NaN), one per 32 elements of a
 *    row along K, in the 128 x 4 blocked layout: for a matrix of R rows and
 *    S = K/32 scale columns, padded to R' = roundup(R, 128) and
 *    S' = roundup(S, 4), scale (r, s) is the byte at
 *      ((r/128) * (S'/4) + s/4) * 512 + (r%32) * 16 + ((r/32)%4) * 4 + s%4.
 *    SFA covers A's stacked rows; SFB holds G such arrays back to back, group
 *    g's for its N rows at offset g * tg_mx_scale_bytes(N, K).  Padding bytes
 *    never affect a stored output (any byte is a valid UE8M0 code).
 * C: stacked rows x N bf16, row-major; only the m_sizes[g] rows of each group
 *    are written.  relu = 1 maps every value that is not > 0 to +0.
 * The sum is accumulated in fp32 by the tensor core; the result is rounded to
 * bf16 (nearest even).
 *
 * Requirements (else TG_ERR_INVALID_ARG, nothing enqueued): 0 <= G <= 256,
 * m_sizes[g] >= 0, K % 32 == 0, N % 8 == 0, 16-byte aligned A, B, SFA, SFB
 * and C, C not overlapping any input.  m_sizes is a HOST array.  G == 0,
 * N == 0 or all-empty groups: TG_OK with nothing enqueued; K == 0 writes +0.
 * Asynchronous on `stream`; no device memory is allocated.
 * ------------------------------------------------------------------------- */
enum { TG_FP8_E4M3 = 0, TG_FP8_E5M2 = 1 };

TG_API tg_status tg_gemm_mxf8_grouped(const void *A, const void *SFA, const void *B, const void *SFB, void *C,
                                      const int64_t *m_sizes, int32_t groups, int64_t N, int64_t K,
                                      int32_t a_format, int32_t b_format, int32_t relu, void *stream);

/* Stacked rows for these group sizes (each padded to 128), or -1 if invalid. */
TG_API int64_t tg_mx_grouped_rows(const int64_t *m_sizes, int32_t groups);

/* Bytes of one blocked UE8M0 scale array for `rows` rows and K elements
 * (roundup(rows, 128) * roundup(K/32, 4)), or -1 if K % 32 != 0. */
TG_API int64_t tg_mx_scale_bytes(int64_t rows, int64_t K);

/* ---------------------------------------------------------------------------
 * NVF4 block-scaled grouped GEMM
 *
 * The NVF4 block-scaled MMA path (tilelang-ai project page, "Three backends
 * under one language dialect", quoted there at 8192^3), read as NVIDIA's
 * NVFP4 format, with the grouping and row layout of tg_gemm_mxf8_grouped:
 *
 *   C[r*N + j] = bf16( [relu]( alpha * sum_{k<K} a(r,k) sa(r,k/16) * b_g(j,k) sb_g(j,k/16) ) )
 *
 * A: stacked rows x K/2 bytes, B: G x N x K/2 bytes; each byte packs two FP4
 *    E2M1 elements (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives), element 2i in
 *    the low nibble.  Group g's rows start at o_g = sum_{h<g} roundup(m_h, 128).
 * SFA, SFB: one UE4M3 scale (an FP8 E4M3 code with the sign bit clear) per 16
 *    elements along K, in the 128 x 4 blocked layout described above with
 *    S = K/16 scale columns; group g's SFB at g * tg_nvf4_scale_bytes(N, K).
 *    Every byte of both arrays, padding included, must be a finite UE4M3
 *    code (0x00 .. 0x7E): the tensor core reads the padding rows' scales too
 *    (their outputs are discarded), and other codes are not valid scales.
 * alpha: a finite fp32 factor applied to the fp32 accumulator (the per-tensor
 *    scale of NVFP4).
 * C: stacked rows x N bf16; only the rows of the groups are written.
 * Requirements (else TG_ERR_INVALID_ARG, nothing enqueued): K % 64 == 0, the
 * rest as tg_gemm_mxf8_grouped.  m_sizes is a HOST array.
 * ------------------------------------------------------------------------- */
TG_API tg_status tg_gemm_nvf4_grouped(const void *A, const void *SFA, const void *B, const void *SFB, void *C,
                                      const int64_t *m_sizes, int32_t groups, int64_t N, int64_t K, float alpha,
                                      int32_t relu, void *stream);

/* Bytes of one blocked UE4M3 scale array for `rows` rows and K elements
 * (roundup(rows, 128) * roundup(K/16, 4)), or -1 if K % 16 != 0. */
TG_API int64_t tg_nvf4_scale_bytes(int64_t rows, int64_t K);

/* ---------------------------------------------------------------------------
 * 4-bit weight-only GEMM (W4A16)
 *
 * The dequantize_gemm workload of the TileLang pages ("TileLang" wiki page,
 * opening paragraph), read as the common W4A16 scheme:
 *
 *   w(n,k)  = fp16( (q(n,k) - 8) * s(n, k/group) )      (exact product, one RNE rounding)
 *   C[m*N + n] = fp16( max( sum_k A[m*K + k] * w(n,k), 0 ) )   (fp32 accumulation)
 *
 * A: M x K fp16, row-major.  Wq: the N x K weight as 4-bit codes q, rows of
 * K/2 bytes, element 2i of a row in the low nibble of byte i.  scales: N x
 * (K/group) fp16, row-major.  C: M x N fp16, row-major.  group is a power of
 * two >= 32 that divides K; K % 64 == 0.
 * M <= 256 runs one fused kernel that streams the packed weight once (for
 * M <= 16 and K % 256 == 0, K <= 16384, a decode kernel that dequantizes in
 * registers; tg_w4a16_kernel tells which).  Larger
 * M dequantizes the weight into `workspace` (tg_w4a16_workspace_size bytes,
 * 16-byte aligned, 2*N*K rounded up) and runs the fp16 tensor-core GEMM.
 * Errors (TG_ERR_INVALID_ARG, nothing enqueued): bad sizes or group, A or Wq
 * not 16-byte aligned, scales or C not 2-byte aligned, C overlapping an
 * input, too small a workspace.  K == 0 writes +0.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
TG_API tg_status tg_gemm_relu_w4a16(const void *A, const void *Wq, const void *scales, void *C, int64_t M,
                                    int64_t N, int64_t K, int32_t group, void *stream, void *workspace,
                                    int64_t workspace_bytes);

/* The kernels tg_gemm_relu_w4a16 runs for these sizes (host logic only). */
typedef enum tg_w4a16_kernel_kind {
    TG_W4_INVALID = -1,  /* the sizes or the group are invalid                 */
    TG_W4_NONE = 0,      /* nothing to compute: M == 0 or N == 0, or K == 0 (C = +0) */
    TG_W4_DECODE = 1,    /* M <= 16, K % 256 == 0, K <= 16384: dequantization in
                            registers feeding warp-level MMAs, split-K over a
                            cluster of up to 8 CTAs reduced in shared memory */
    TG_W4_FUSED = 2,     /* M <= 256: the tcgen05 kernel with a dequantization
                            stage in front of the MMA                         */
    TG_W4_DEQUANT_GEMM = 3 /* larger M: dequantize into the workspace, then
                            the fp16 tensor-core GEMM                        */
} tg_w4a16_kernel_kind;
TG_API int tg_w4a16_kernel(int64_t M, int64_t N, int64_t K, int32_t group);

/* Workspace bytes tg_gemm_relu_w4a16 needs for these sizes (0 for M <= 256),
 * or -1 if the sizes are invalid. */
TG_API int64_t tg_w4a16_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group);

/* The dequantized weight alone: W (N x K fp16, 16-byte aligned) = w(n,k) as
 * above.  Same requirements on Wq, scales, K and group. */
TG_API tg_status tg_dequant_w4_f16(const void *Wq, const void *scales, void *W, int64_t N, int64_t K,
                                   int32_t group, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TG_GEMM_H */
