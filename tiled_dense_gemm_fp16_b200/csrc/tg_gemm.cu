// tg_gemm.cu -- C ABI, argument checks, path choice, TMA descriptor encoding
// and kernel launches for C = ReLU(A . B) on sm_100a.
//
// The whole device side is one translation unit: the kernels live in the
// headers included below and share the device error word of ptx.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tg_gemm.h"
#include "gemm_mx.cuh"
#include "gemm_rc.cuh"
#include "gemm_skinny.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc_pair.cuh"
#include "gemm_w4a16.cuh"
#include "ptx.cuh"
#include "repack.cuh"

namespace tg {
namespace {

constexpr uint64_t kWaitBudgetNs = 4000000000ull;  // 4 s per pipeline wait, plus:
constexpr uint64_t kWaitPerKBlockNs = 4000ull;      // 4 us per k-block (waits that span a tile's K loop)

// Bound of one wait: generous for a single pipeline step, and longer than a
// whole tile's K loop (about 0.5 us per 64-deep k-block at full speed) for the
// waits that span one.
uint64_t wait_budget(int64_t k_blocks) {
  return kWaitBudgetNs + static_cast<uint64_t>(k_blocks > 0 ? k_blocks : 0) * kWaitPerKBlockNs;
}
constexpr int kMaxDevices = 64;
constexpr int64_t kSkinnyMaxM = 256;               // largest M the small-M path takes

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  bool tc_attr = false;
  bool tc_edge_attr = false;
  bool skinny_attr = false;
  unsigned tc_pair_attr = 0;  // one bit per (stages, tile width) instance with its attribute set
  bool mx_attr[2] = {false, false};       // per block-scaled kind
  unsigned rc_attr = 0;       // one bit per residue-class kernel instance with its attribute set
  bool w4_attr = false;
  bool w4_decode_attr = false;
  void* static_ws = nullptr;  // device address of g_static_workspace on this device
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

// Fixed scratch for tg_gemm_relu_f16_static_ws, one per device that loads the
// library.  In host code this name is only a handle: its device address comes
// from cudaGetSymbolAddress with the device current.
__device__ __align__(256) uint8_t g_static_workspace[TG_STATIC_WORKSPACE_BYTES];

// Tuning knobs.  The shipped library always uses the tuned defaults: the
// environment cannot change a kernel configuration, and no launch pays for
// a lookup.  A build with -DTG_TUNING reads TG_TUNE_* variables instead,
// each once per process (for sweeps).
#ifdef TG_TUNING
int tune_int(const char* name, int dflt) {
  static std::mutex m;
  static const char* names[64];
  static int values[64];
  static bool present[64];
  static int count = 0;
  std::lock_guard<std::mutex> lock(m);
  for (int i = 0; i < count; ++i)
    if (std::strcmp(names[i], name) == 0) return present[i] ? values[i] : dflt;
  const char* v = std::getenv(name);
  if (count < 64) {
    names[count] = name;
    present[count] = v && *v;
    values[count] = present[count] ? std::atoi(v) : 0;
    ++count;
  }
  return (v && *v) ? std::atoi(v) : dflt;
}
#else
constexpr int tune_int(const char*, int dflt) { return dflt; }
#endif
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
bool g_encode_probed = false;

// One problem as the caller describes it: batch entries of
//   C[i*ldc + j] = f16(relu(sum_k A[i*lda + k] * b(k, j) + bias[j]))
// with b(k, j) = B[k*ldb + j] (B stored K x N) or B[j*ldb + k] (B stored
// N x K), entry e starting at A + e*sa, B + e*sb, C + e*sc (elements).
struct Problem {
  const void* A;
  const void* B;
  void* C;
  int64_t M, N, K;
  int64_t lda, ldb, ldc;
  bool a_km;  // A stored K x M (C = A^T . B)
  bool b_nk;  // B stored N x K (C = A . B^T)
  const void* bias;
  int64_t batch, sa, sb, sc;
};

Problem dense_problem(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K) {
  return Problem{A, B, C, M, N, K, K, N, N, false, false, nullptr, 1, 0, 0, 0};
}

// One GEMM as the kernels see it (one batch entry, possibly repacked).
struct Operands {
  const void* A;
  int64_t lda;
  bool a_km;
  const void* B;
  int64_t ldb;
  bool b_nk;
  void* C;
  int64_t ldc;
  const void* bias;
  int64_t M, N, K;
  bool c_aligned;  // every row of C starts on a 16-byte boundary
};

// ---------------------------------------------------------------------------
// Host-side argument logic (no CUDA calls)
// ---------------------------------------------------------------------------
constexpr int64_t kMaxStride = int64_t(1) << 40;  // elements; keeps every byte offset in int64

bool ranges_overlap(const void* a, int64_t a_bytes, const void* b, int64_t b_bytes) {
  if (a_bytes <= 0 || b_bytes <= 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + static_cast<uintptr_t>(b_bytes) && b0 < a0 + static_cast<uintptr_t>(a_bytes);
}

// Bytes each operand spans over all batch entries.
int64_t span_a(const Problem& p) {
  if (p.M <= 0 || p.K <= 0) return 0;
  const int64_t one = p.a_km ? (p.K - 1) * p.lda + p.M : (p.M - 1) * p.lda + p.K;
  return 2 * ((p.batch - 1) * p.sa + one);
}
int64_t span_b(const Problem& p) {
  if (p.K <= 0 || p.N <= 0) return 0;
  const int64_t one = p.b_nk ? (p.N - 1) * p.ldb + p.K : (p.K - 1) * p.ldb + p.N;
  return 2 * ((p.batch - 1) * p.sb + one);
}
int64_t span_c_one(const Problem& p) { return (p.M > 0 && p.N > 0) ? (p.M - 1) * p.ldc + p.N : 0; }
int64_t span_c(const Problem& p) { return (p.M > 0 && p.N > 0) ? 2 * ((p.batch - 1) * p.sc + span_c_one(p)) : 0; }

bool problem_valid(const Problem& p) {
  if (p.M < 0 || p.N < 0 || p.K < 0) return false;
  if (p.M > INT_MAX || p.N > INT_MAX || p.K > INT_MAX) return false;
  if (p.batch < 1 || p.batch > INT_MAX) return false;
  if (p.M == 0 || p.N == 0) return true;
  if (p.lda < (p.a_km ? p.M : (p.K > 0 ? p.K : 0)) || p.ldc < p.N) return false;
  if (p.ldb < (p.b_nk ? p.K : p.N)) return false;
  if (p.lda > kMaxStride || p.ldb > kMaxStride || p.ldc > kMaxStride) return false;
  if (p.sa < 0 || p.sb < 0 || p.sc < 0 || p.sa > kMaxStride || p.sb > kMaxStride || p.sc > kMaxStride)
    return false;
  if (p.batch > 1 && p.sc < span_c_one(p)) return false;  // C entries must not overlap each other
  if (p.C == nullptr) return false;
  if (p.K > 0 && (p.A == nullptr || p.B == nullptr)) return false;
  const uintptr_t bits = reinterpret_cast<uintptr_t>(p.A) | reinterpret_cast<uintptr_t>(p.B) |
                         reinterpret_cast<uintptr_t>(p.C) | reinterpret_cast<uintptr_t>(p.bias);
  if (bits & 1u) return false;
  const int64_t c_bytes = span_c(p);
  if (p.K > 0 && (ranges_overlap(p.C, c_bytes, p.A, span_a(p)) || ranges_overlap(p.C, c_bytes, p.B, span_b(p))))
    return false;
  if (p.bias && ranges_overlap(p.C, c_bytes, p.bias, 2 * p.N)) return false;
  // Tile counts must fit the kernels' 32-bit tile indices.
  const int64_t tiles = ((p.M + 127) / 128) * ((p.N + 255) / 256);
  if (tiles > INT_MAX) return false;
  return true;
}

// TMA can describe A (B) in every batch entry: 16-byte aligned bases, row
// strides and batch strides.
bool tma_ok_a(const Problem& p) {
  return (reinterpret_cast<uintptr_t>(p.A) & 15u) == 0 && p.lda % 8 == 0 && (p.batch == 1 || p.sa % 8 == 0);
}
bool tma_ok_b(const Problem& p) {
  return (reinterpret_cast<uintptr_t>(p.B) & 15u) == 0 && p.ldb % 8 == 0 && (p.batch == 1 || p.sb % 8 == 0);
}
bool tma_ok(const Problem& p) { return tma_ok_a(p) && tma_ok_b(p); }

// The residue-class kernel reads A stored M x K and B stored K x N.
bool rc_ok(const Problem& p) { return !p.a_km && !p.b_nk; }

// Operands TMA cannot describe, with a workspace: the residue-class kernel
// (on a padded copy of B when B needs one) or the repack path (padded copies
// of A, B and C around the faster CTA-pair kernel).  The repack path moves
// about 2 (MK + MN) more bytes twice; its kernel saves about a fifth of the
// main loop's time on 2 MNK flops.  With copies at about 5 TB/s and the loop
// at about 1.2 PFLOP/s, the residue-class kernel wins when
// 1/N + 1/K > 1/2400 (measured at (3001, 5003, 1021) and (8191, 129, 8193),
// and the other way at (777, 12289, 4095)).
bool rc_preferred(const Problem& p) {
  return rc_ok(p) && 2400.0 * static_cast<double>(p.N + p.K) > static_cast<double>(p.N) * static_cast<double>(p.K);
}

// Tile plan of the residue-class kernel (host logic only): tile width, rows
// per tile, K split and ring, for a device of `sms` SMs.
struct RcPlan {
  int bn = 0, n_tiles = 0, panels = 0, msub = 1, splits = 1, ring = 0, ring_bytes = 0;
  int kb_per_cta = 0;    // k-blocks a CTA walks per tile (upper bound over the classes)
  bool b_deep = false;   // B realigned in place keeps two k-blocks in flight
};
constexpr int kRcSmemMax = 232448, kRcFixed = 1024 + 512;
constexpr int kRcPlanSms = 148;  // SMs assumed by the host-only queries

// One class when A's row stride is a multiple of 8 elements and covers the
// widened rows; else the eight residue classes of the rows.
int rc_a_classes(const void* A, int64_t lda, int64_t K) {
  const int64_t e0 = static_cast<int64_t>((reinterpret_cast<uintptr_t>(A) & 15u) / 2);
  return (lda % 8 == 0 && lda >= K + e0) ? 1 : kRcClasses;
}

bool rc_plan(int64_t M, int64_t N, int64_t K, int a_classes, int sms, RcPlan* out) {
  RcPlan pl;
  const int kb_min = static_cast<int>((K + 63) / 64);
  pl.bn = N <= 240 ? static_cast<int>((N + 15) / 16 * 16) : 256;
  int64_t m128 = 0;
  for (int c = 0; c < a_classes; ++c) {
    const int64_t n = M > c ? (M - c + a_classes - 1) / a_classes : 0;
    m128 += (n + 127) / 128;
  }
  // The persistent CTAs take the tiles in waves.  When 256-wide tiles fill
  // at least one wave, pick the width w (a multiple of 16, 128..256) with
  // the least waves x bytes per k-block (16 KiB of A and 128 w of B: the
  // kernel moves operands rather than multiplies), so that the last wave is
  // not mostly idle; ties go to the wider tile.
  if (N > 240 && m128 * ((N + 255) / 256) >= sms) {
    int64_t best = -1;
    for (int w = 256; w >= 128; w -= 16) {
      const int64_t cost = (m128 * ((N + w - 1) / w) + sms - 1) / sms * (16384 + 128 * w);
      if (best < 0 || cost < best) {
        best = cost;
        pl.bn = w;
      }
    }
  }
  pl.bn = tune_int("TG_TUNE_RC_BN", pl.bn);
  if (pl.bn < 16 || pl.bn > 256 || pl.bn % 16 != 0) return false;
  pl.n_tiles = static_cast<int>((N + pl.bn - 1) / pl.bn);
  pl.panels = (pl.bn + 63) / 64;
  auto tiles_for = [&](int rows) {
    int t = 0;
    for (int c = 0; c < a_classes; ++c) {
      const int64_t n = M > c ? (M - c + a_classes - 1) / a_classes : 0;
      t += static_cast<int>((n + rows - 1) / rows);
    }
    return t * pl.n_tiles;
  };
  auto ring_for = [&](int msub, int* stages, int* stage_bytes) {
    *stage_bytes = msub * RcCfg<false>::A_BYTES + pl.panels * RcCfg<false>::PANEL_BYTES;
    int r = (kRcSmemMax - kRcFixed) / *stage_bytes;
    *stages = r > RcCfg<false>::MAX_RING ? RcCfg<false>::MAX_RING : r;
  };
  // Few tiles: split K over a cluster of S CTAs (each keeps at least 4
  // k-blocks), when the cluster's partials of one tile's rows (S slots of
  // ceil(R / S) rows) fit in the ring.  For one column of narrow tiles (A
  // streams from memory) a tile takes 2 x 128 class rows, two accumulators
  // sharing each B stage, when that still splits.
  auto splits_for = [&](int tiles, int msub) {
    int st, sb;
    ring_for(msub, &st, &sb);
    if (st < 2 || 2 * tiles > sms) return 1;
    int s = sms / tiles;
    s = s > 8 ? 8 : s;
    while (s > 1 && kb_min / s < 4) --s;
    s = tune_int("TG_TUNE_RC_SPLITS", s);
    if (s > 8) s = 8;
    const int R = 128 * msub;
    while (s > 1 && s * ((R + s - 1) / s) * pl.bn * 4 > st * sb) --s;
    return s;
  };
  pl.splits = splits_for(tiles_for(128), 1);
  if (pl.splits > 1 && pl.bn <= 240 && tiles_for(256) < tiles_for(128) && tune_int("TG_TUNE_RC_MSUB2", 1)) {
    const int s2 = splits_for(tiles_for(256), 2);
    if (s2 > 1) {
      pl.msub = 2;
      pl.splits = s2;
    }
  }
  ring_for(pl.msub, &pl.ring, &pl.ring_bytes);
  if (pl.ring < 2) return false;
  // B realigned in place keeps two k-blocks in flight with tiles narrower
  // than 256 columns (at most 31 chunks per row, so no lane needs a 33rd
  // block) and long K walks (32 or more k-blocks per CTA and tile).
  // Measured without a workspace: (8191, 129, 8193) 47.0 -> 44.5 us, (777,
  // 12289, 4095) 192.8 -> 179.6 us; with 16 k-blocks, (3001, 5003, 1021) went
  // from 72.5 to 75-76 us, so short walks keep one.
  const int kb_walk = static_cast<int>((K + 7 + 63) / 64);
  pl.kb_per_cta = (kb_walk + pl.splits - 1) / pl.splits;
  pl.b_deep = pl.bn < 256 && pl.kb_per_cta >= 32 && tune_int("TG_TUNE_RC_B_DEEP", 1);
  *out = pl;
  return true;
}

// Bytes of the padded copy of B (rows rounded up to 8 elements) that the
// residue-class kernel reads when TMA cannot describe B, else 0.  No copy
// either where realigning B in place is the faster route: two k-blocks in
// flight and a B tile no wider than the tile's rows of A (bn <= 128 msub), so
// that B is the smaller stream.  Measured at (8191, 129, 8193): 44.5 us in
// place against 49.7 us with the copy (a dependent kernel between GEMMs).
int64_t rc_b_copy_bytes(const Problem& p) {
  if (p.K <= 0 || p.N <= 0 || tma_ok_b(p)) return 0;
  RcPlan pl;
  if (!p.a_km && rc_plan(p.M, p.N, p.K, rc_a_classes(p.A, p.lda, p.K), kRcPlanSms, &pl) && pl.b_deep &&
      pl.bn <= 128 * pl.msub)
    return 0;
  return (2 * p.K * ((p.N + 7) / 8 * 8) + 255) / 256 * 256;
}

// Every row of C, in every batch entry, starts on a 16-byte boundary.
bool c_rows_aligned(const Problem& p) {
  return (reinterpret_cast<uintptr_t>(p.C) & 15u) == 0 && p.ldc % 8 == 0 && (p.batch == 1 || p.sc % 8 == 0);
}

// The small-M kernel (A stored M x K) for M <= 128, where two CTAs share an
// SM and the split-K partials are small; for 128 < M <= 256 only when B is
// large (N x K >= 2^23), since the partials (M x 128 fp32 per CTA) then cost
// less than the tile kernels' few waves.  Measured, µs (small-M vs best tile
// kernel): 256 x 256 x 256 10.5 / 7.2, 256 x 2048 x 2048 23.8 / 16.9,
// 256 x 4096 x 4096 18.4 / 27.4; at M <= 128 the small-M kernel wins down to
// 64 x 512 x 512 (6.1 / 7.5).
bool skinny_route(const Problem& p) {
  return p.M <= kSkinnyMaxM && !p.a_km && (p.M <= 128 || p.N * p.K >= (int64_t(1) << 23));
}

// The tensor-core kernels store C fastest when its rows start on 16-byte
// boundaries (whole 16-byte pieces, or TMA boxes); the small-M kernel writes
// C element by element either way.
bool c_pad_useful(const Problem& p) {
  return !c_rows_aligned(p) && !skinny_route(p);
}

// Workspace of the repack path: zero-padded copies (rows rounded up to 8
// elements) of one batch entry of whichever of A and B TMA cannot describe,
// and, with `with_c`, a padded C (M x N rounded up to 8) that the GEMM writes
// and a realigning copy then moves into C when C's rows are not 16-byte
// aligned; each 256-byte aligned; batch entries reuse it in stream order.
struct RepackPlan {
  bool pad_a = false, pad_b = false, pad_c = false;
  int64_t kp = 0, np = 0, mp = 0;
  int64_t off_a = 0, off_b = 0, off_c = 0, bytes = 0;
};

RepackPlan repack_plan(const Problem& p, bool with_c) {
  RepackPlan r;
  r.kp = (p.K + 7) / 8 * 8;
  r.np = (p.N + 7) / 8 * 8;
  r.mp = (p.M + 7) / 8 * 8;
  r.pad_a = !tma_ok_a(p);
  r.pad_b = !tma_ok_b(p);
  r.pad_c = with_c && c_pad_useful(p);
  auto up256 = [](int64_t x) { return (x + 255) / 256 * 256; };
  const int64_t bytes_a = r.pad_a ? up256(p.a_km ? 2 * p.K * r.mp : 2 * p.M * r.kp) : 0;
  const int64_t bytes_b = r.pad_b ? up256(p.b_nk ? 2 * p.N * r.kp : 2 * p.K * r.np) : 0;
  const int64_t bytes_c = r.pad_c ? up256(2 * p.M * r.np) : 0;
  r.off_a = 0;
  r.off_b = bytes_a;
  r.off_c = bytes_a + bytes_b;
  r.bytes = bytes_a + bytes_b + bytes_c;
  return r;
}

// Workspace the call needs at the least (the A and B copies when TMA cannot
// describe them) and for its fastest path (plus the padded C).
int64_t repack_bytes_needed(const Problem& p) {
  if (p.M == 0 || p.N == 0 || p.K == 0 || tma_ok(p)) return 0;
  return rc_preferred(p) ? rc_b_copy_bytes(p) : repack_plan(p, false).bytes;
}
int64_t workspace_bytes_needed(const Problem& p) {
  if (p.M == 0 || p.N == 0 || p.K == 0) return 0;
  if (!tma_ok(p) && rc_preferred(p)) return rc_b_copy_bytes(p);
  return repack_plan(p, true).bytes;
}

// The repack plan a call with `ws_bytes` of workspace takes: with the padded
// C when it fits.
RepackPlan chosen_plan(const Problem& p, int64_t ws_bytes) {
  const RepackPlan full = repack_plan(p, true);
  return ws_bytes >= full.bytes ? full : repack_plan(p, false);
}

bool path_supports(int path, const Problem& p) {
  if (!problem_valid(p)) return false;
  if (p.M == 0 || p.N == 0) return path == TG_PATH_NONE || path == TG_PATH_AUTO;
  if (p.K == 0) return path == TG_PATH_ZERO || path == TG_PATH_AUTO;
  switch (path) {
    case TG_PATH_AUTO:
      return true;
    case TG_PATH_TC_EDGE:
      return !p.b_nk && !p.a_km;  // the realigning producer reads A stored M x K, B stored K x N
    case TG_PATH_TC:
    case TG_PATH_TC_PAIR:
    case TG_PATH_TC_PAIR512:
      return tma_ok(p);
    case TG_PATH_SKINNY:
      return tma_ok(p) && p.M <= kSkinnyMaxM && !p.a_km;
    case TG_PATH_REPACK:
      return !tma_ok(p) || c_pad_useful(p);
    case TG_PATH_RC:
      return rc_ok(p);
    default:
      return false;
  }
}

// Estimated relative time of the three tensor-core kernels on a 148-SM
// device: waves of tiles x per-SM work of one tile.  The main loop of a tile
// costs its per-SM MACs over the kernel's measured relative efficiency
// (single CTA 0.85, pair 256x256 0.88, pair 256x512 1.0 at 8192^3).  The
// 256x512 tile has one accumulator, so each tile's epilogue (draining TMEM,
// worth about 384 k-steps of MMA, twice that when the rows of C are only
// 2-byte aligned) adds to every tile; the double-buffered kernels hide it
// behind the next tile and pay it once at the end.
int pick_tc_kernel(int64_t M, int64_t N, int64_t K, bool c_aligned) {
  constexpr int64_t kSms = 148, kPairs = 74;
  auto waves = [](int64_t tiles, int64_t units) { return static_cast<double>((tiles + units - 1) / units); };
  const double kepi = c_aligned ? 384.0 : 768.0;
  const double k = static_cast<double>(K);
  const double area1 = 128.0 * 256.0, area3 = 128.0 * 512.0;
  const double t1 = waves(((M + 127) / 128) * ((N + 255) / 256), kSms) * area1 * k / 0.85 + area1 * kepi;
  const double t2 = waves(((M + 255) / 256) * ((N + 255) / 256), kPairs) * area1 * k / 0.88 + area1 * kepi;
  const double t3 = waves(((M + 255) / 256) * ((N + 511) / 512), kPairs) * area3 * (k + kepi);
  if (t3 <= t2 && t3 <= t1) return TG_PATH_TC_PAIR512;
  return t2 <= t1 ? TG_PATH_TC_PAIR : TG_PATH_TC;
}

// The tensor-core kernel that runs on TMA-describable (possibly repacked) operands.
int inner_path(const Problem& p, bool c_padded = false) {
  return skinny_route(p) ? TG_PATH_SKINNY : pick_tc_kernel(p.M, p.N, p.K, c_padded || c_rows_aligned(p));
}

// The path a call takes with `ws_bytes` of workspace (-2: invalid arguments).
// Operands TMA cannot describe take the repack path when the workspace
// suffices, else the edge mode (B stored K x N) or, for B stored N x K, the
// repack path that run() then refuses for want of a workspace.
int select_path(const Problem& p, int64_t ws_bytes) {
  if (!problem_valid(p)) return -2;
  if (p.M == 0 || p.N == 0) return TG_PATH_NONE;
  if (p.K == 0) return TG_PATH_ZERO;
  if (!tma_ok(p)) {
    // rc_preferred: with a workspace holding B's copy, run() pads B first.
    if (rc_preferred(p)) return TG_PATH_RC;
    if (ws_bytes >= repack_plan(p, false).bytes || p.b_nk || p.a_km) return TG_PATH_REPACK;
    return rc_ok(p) ? TG_PATH_RC : TG_PATH_TC_EDGE;
  }
  // Operands TMA can read, but C's rows are not 16-byte aligned: the GEMM
  // writes a padded C in the workspace when there is room for it.
  if (c_pad_useful(p) && ws_bytes >= repack_plan(p, true).bytes) return TG_PATH_REPACK;
  return inner_path(p);
}

// ---------------------------------------------------------------------------
// Device probing and TMA descriptors
// ---------------------------------------------------------------------------
tg_status current_device(int& dev, DeviceInfo*& info) {
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return TG_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return TG_ERR_UNSUPPORTED_DEVICE;
    }
    d.probed = true;
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
  }
  info = &d;
  return d.supported ? TG_OK : TG_ERR_UNSUPPORTED_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_encode_probed) {
    g_encode_probed = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaGetLastError();
  }
  return g_encode_tiled;
}

// Row-major fp16 matrix of rows x cols with a row stride of `ld` elements
// (ld * 2 a multiple of 16); box = box_cols x box_rows, 128-byte swizzle
// (box_cols * 2 must be 128; with the 64-byte swizzle, 64).  Columns past
// `cols` read as zero, and stores past them are dropped.
bool encode_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_cols,
               int box_rows, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp16 matrix (rows x cols, row stride cols) with an unswizzled box.
bool encode_2d_f16_plain(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor maps of one GEMM's A (stored M x K: boxes of 64 k x a_rows; stored
// K x M: boxes of 64 m x 64 k) and B (stored K x N: boxes of 64 n x 64 k;
// stored N x K: boxes of 64 k x b_rows).
bool encode_operands(const Operands& o, CUtensorMap* ta, CUtensorMap* tb, int a_rows, int b_rows) {
  if (o.a_km) {
    if (!encode_2d(ta, o.A, o.K, o.M, o.lda, 64, 64)) return false;
  } else if (!encode_2d(ta, o.A, o.M, o.K, o.lda, 64, a_rows)) {
    return false;
  }
  if (o.b_nk) return encode_2d(tb, o.B, o.N, o.K, o.ldb, 64, b_rows);
  return encode_2d(tb, o.B, o.K, o.N, o.ldb, 64, 64);
}

void fill_tc_params(TcParams& p, const Operands& o) {
  std::memset(&p, 0, sizeof p);
  p.A = static_cast<const __half*>(o.A);
  p.B = static_cast<const __half*>(o.B);
  p.C = static_cast<__half*>(o.C);
  p.bias = static_cast<const __half*>(o.bias);
  p.lda = o.lda;
  p.ldb = o.ldb;
  p.ldc = o.ldc;
  p.b_kmajor = o.b_nk ? 1 : 0;
  p.a_mnmajor = o.a_km ? 1 : 0;
  p.M = static_cast<int>(o.M);
  p.N = static_cast<int>(o.N);
  p.K = static_cast<int>(o.K);
  p.c_aligned = o.c_aligned ? 1 : 0;
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
// Every kernel is launched with programmatic stream serialization: it may be
// scheduled while the previous kernel on the stream drains, runs its
// prologue (barriers, TMEM), and waits for that kernel before touching
// global memory.  `cluster_x` > 1 adds a cluster dimension.
struct LaunchAttrs {
  cudaLaunchAttribute attr[2];
  unsigned count = 0;
  void fill(cudaLaunchConfig_t& cfg, unsigned cluster_x) {
    count = 0;
    attr[count].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[count].val.programmaticStreamSerializationAllowed = tune_int("TG_TUNE_PDL", 1) ? 1 : 0;
    ++count;
    if (cluster_x > 1) {
      attr[count].id = cudaLaunchAttributeClusterDimension;
      attr[count].val.clusterDim.x = cluster_x;
      attr[count].val.clusterDim.y = 1;
      attr[count].val.clusterDim.z = 1;
      ++count;
    }
    cfg.attrs = attr;
    cfg.numAttrs = count;
  }
};

template <bool EDGE>
tg_status launch_tc(const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  using Cfg = TcCfg<EDGE>;
  const int64_t M = o.M, N = o.N, K = o.K;
  auto kernel = gemm_relu_tc_kernel<EDGE>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    bool& attr = EDGE ? info->tc_edge_attr : info->tc_attr;
    if (!attr) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) !=
          cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      attr = true;
    }
  }
  CUtensorMap ta, tb;
  std::memset(&ta, 0, sizeof ta);
  std::memset(&tb, 0, sizeof tb);
  if (!EDGE && !encode_operands(o, &ta, &tb, Cfg::BM, Cfg::BN)) return TG_ERR_LAUNCH;
  TcParams p;
  fill_tc_params(p, o);
  p.m_tiles = static_cast<int>((M + Cfg::BM - 1) / Cfg::BM);
  p.n_tiles = static_cast<int>((N + Cfg::BN - 1) / Cfg::BN);
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.k_blocks = static_cast<int>((K + Cfg::BK - 1) / Cfg::BK);
  p.group_m = tune_int("TG_TUNE_GROUP_M", 16);
  if (p.group_m < 1) p.group_m = 1;
  p.wait_budget_ns = wait_budget(p.k_blocks);
  const int grid = p.num_tiles < info->sm_count ? p.num_tiles : info->sm_count;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::SMEM_BYTES);
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, 1);
  if (cudaLaunchKernelEx(&cfg, kernel, ta, tb, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

// 2-CTA path: 256 x 256 tiles on SM pairs, clusters of 2 along x.
template <int STAGES, int BN>
tg_status launch_tc_pair_cfg(const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  using Cfg = TcPairCfg<STAGES, BN>;
  const int64_t M = o.M, N = o.N, K = o.K;
  auto kernel = gemm_relu_tc_pair_kernel<STAGES, BN>;
  constexpr unsigned kAttrBit = 1u << (STAGES + (BN == 512 ? 16 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(info->tc_pair_attr & kAttrBit)) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) !=
          cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->tc_pair_attr |= kAttrBit;
    }
  }
  CUtensorMap ta, tb, tc;
  if (!encode_operands(o, &ta, &tb, Cfg::BM, 128)) return TG_ERR_LAUNCH;
  // C for the TMA-store epilogue: 32 x 32 boxes.
  std::memset(&tc, 0, sizeof tc);
  if (Cfg::C_STAGE_BYTES > 0 && o.c_aligned &&
      !encode_2d(&tc, o.C, o.M, o.N, o.ldc, Cfg::C_BOX_COLS, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return TG_ERR_LAUNCH;
  TcParams p;
  fill_tc_params(p, o);
  p.m_tiles = static_cast<int>((M + Cfg::PAIR_M - 1) / Cfg::PAIR_M);
  p.n_tiles = static_cast<int>((N + Cfg::BN - 1) / Cfg::BN);
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.k_blocks = static_cast<int>((K + Cfg::BK - 1) / Cfg::BK);
  p.group_m = tune_int("TG_TUNE_GROUP_M", BN == 512 ? 16 : 12);
  if (p.group_m < 1) p.group_m = 1;
  p.store_streaming = tune_int("TG_TUNE_STORE_CS", 1);
  p.l2_hints = tune_int("TG_TUNE_L2_HINTS", BN == 512 ? 2 : 5);
  p.prefetch_kb = tune_int("TG_TUNE_PREFETCH_KB", 0);
  p.wait_budget_ns = wait_budget(p.k_blocks);
  const int pairs = info->sm_count / 2;
  const int clusters = p.num_tiles < pairs ? p.num_tiles : pairs;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::SMEM_BYTES);
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, 2);
  if (cudaLaunchKernelEx(&cfg, kernel, ta, tb, tc, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

tg_status launch_tc_pair(const Operands& o, cudaStream_t stream, DeviceInfo* info, int bn) {
  if (bn == 512) {
    switch (tune_int("TG_TUNE_PAIR_STAGES", 4)) {
      case 3: return launch_tc_pair_cfg<3, 512>(o, stream, info);
      default: return launch_tc_pair_cfg<4, 512>(o, stream, info);
    }
  }
  switch (tune_int("TG_TUNE_PAIR_STAGES", 6)) {
    case 5: return launch_tc_pair_cfg<5, 256>(o, stream, info);
    default: return launch_tc_pair_cfg<6, 256>(o, stream, info);
  }
}

// Small-M path: grid (S, P) with clusters of S CTAs along K.
tg_status launch_skinny(const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  const int64_t M = o.M, N = o.N, K = o.K;
  using Cfg = SkinnyCfg;
  constexpr int kMaxSmem = 1024 + 220 * 1024 + Cfg::BAR_BYTES;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!info->skinny_attr) {
      if (cudaFuncSetAttribute(gemm_relu_skinny_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) !=
          cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->skinny_attr = true;
    }
  }
  SkinnyParams p;
  std::memset(&p, 0, sizeof p);
  p.C = static_cast<__half*>(o.C);
  p.bias = static_cast<const __half*>(o.bias);
  p.ldc = o.ldc;
  p.b_kmajor = o.b_nk ? 1 : 0;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.c_aligned = (reinterpret_cast<uintptr_t>(o.C) % 8 == 0 && o.ldc % 4 == 0) ? 1 : 0;
  p.m_pad = static_cast<int>((M + 15) / 16 * 16);
  p.k_blocks = static_cast<int>((K + Cfg::BK - 1) / Cfg::BK);
  // Two CTAs per SM fit while the ring stays within ~112 KiB (M_pad <= 128).
  const bool two_per_sm = p.m_pad <= 128;
  // Measured: M_pad <= 32 streams best with a 3-stage ring, larger M_pad
  // with ~112 KiB (4 stages at M_pad = 64).
  int budget_kb = tune_int("TG_TUNE_SKINNY_SMEM_KB", p.m_pad <= 32 ? 64 : (two_per_sm ? 112 : 220));
  budget_kb = budget_kb < 32 ? 32 : (budget_kb > 220 ? 220 : budget_kb);
  const int budget = budget_kb * 1024;
  const int stage_bytes = Cfg::stage_bytes(p.m_pad);
  int stages = budget / stage_bytes;
  stages = stages > 8 ? 8 : stages;
  if (stages < 2) return TG_ERR_INTERNAL;
  // The fp32 partial [M_pad][128] reuses the ring after the main loop.
  if (stages * stage_bytes < p.m_pad * Cfg::PANEL * 4) return TG_ERR_INTERNAL;
  p.stages = stages;
  p.a_stage_bytes = static_cast<uint32_t>(p.m_pad * 128);
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.m_pad)) cols <<= 1;
  p.tmem_cols = cols;
  p.idesc = make_idesc_f16_f32(Cfg::PANEL, p.m_pad, !o.b_nk, false);
  p.prefetch_kb = tune_int("TG_TUNE_SKINNY_PREFETCH_KB", 0);
  p.wait_budget_ns = wait_budget(p.k_blocks);
  const int panels = static_cast<int>((N + Cfg::PANEL - 1) / Cfg::PANEL);  // panels past N are not stored
  const int slots = (two_per_sm ? 2 : 1) * info->sm_count;
  int splits = tune_int("TG_TUNE_SKINNY_SPLITS", slots / panels);
  splits = splits < 1 ? 1 : (splits > 8 ? 8 : splits);
  if (splits > p.k_blocks) splits = p.k_blocks;
  p.splits = splits;
  if (panels > 65535) return TG_ERR_INVALID_ARG;

  CUtensorMap ta, tb;
  if (!encode_operands(o, &ta, &tb, p.m_pad, Cfg::PANEL)) return TG_ERR_LAUNCH;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(panels), 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::smem_bytes(p.m_pad, stages));
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, static_cast<unsigned>(splits));
  if (cudaLaunchKernelEx(&cfg, gemm_relu_skinny_kernel, ta, tb, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}


// Tensor map of a row-major fp16 matrix given by a 16-byte aligned base, its
// inner extent (elements), row count and row stride in bytes.
bool encode_2d_raw(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int64_t stride_bytes,
                   int box_inner, int box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Residue classes of a row-major matrix's rows: `classes` maps, class c
// holding rows c, c + classes, ...  Each map starts at the 16-byte boundary at
// or below its first row and is `shift[c]` elements wider than the rows
// (column x of the map is element x - shift[c] of a row).  Classes without a
// row get no map (rows[c] = 0).
bool encode_classes(CUtensorMap* maps, const void* base, int64_t rows, int64_t cols, int64_t ld, int classes,
                    int box_inner, int box_rows, CUtensorMapSwizzle swizzle, int* shift, int* class_rows) {
  for (int c = 0; c < classes; ++c) {
    const int64_t n = rows > c ? (rows - c + classes - 1) / classes : 0;
    class_rows[c] = static_cast<int>(n);
    shift[c] = 0;
    if (n == 0) continue;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(base) + static_cast<uintptr_t>(2 * c * ld);
    const uintptr_t aligned = addr & ~uintptr_t(15);
    shift[c] = static_cast<int>((addr - aligned) / 2);
    if (!encode_2d_raw(&maps[c], reinterpret_cast<const void*>(aligned), cols + shift[c], n, 2 * classes * ld,
                       box_inner, box_rows, swizzle))
      return false;
  }
  return true;
}

template <bool REALIGN_B, bool SPLIT, bool B_DEEP = false>
tg_status launch_rc_cfg(const RcMaps& maps, const RcParams& p, int smem, int grid_x, int grid_y,
                        cudaStream_t stream, DeviceInfo* info) {
  auto kernel = gemm_relu_rc_kernel<REALIGN_B, SPLIT, B_DEEP>;
  constexpr unsigned kBit = 1u << ((REALIGN_B ? 1 : 0) + (SPLIT ? 2 : 0) + (B_DEEP ? 4 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(info->rc_attr & kBit)) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->rc_attr |= kBit;
    }
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(grid_x), static_cast<unsigned>(grid_y), 1);
  cfg.blockDim = dim3(RcCfg<REALIGN_B>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, SPLIT ? static_cast<unsigned>(p.splits) : 1u);
  if (cudaLaunchKernelEx(&cfg, kernel, maps, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

// Residue-class path: see gemm_rc.cuh.  When TMA cannot describe B, the
// kernel's realigning warps read B's rows in place.
tg_status launch_rc(const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  const int64_t M = o.M, N = o.N, K = o.K;
  RcMaps maps;
  std::memset(&maps, 0, sizeof maps);
  RcParams p;
  std::memset(&p, 0, sizeof p);
  p.C = static_cast<__half*>(o.C);
  p.bias = static_cast<const __half*>(o.bias);
  p.ldc = o.ldc;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.a_classes = rc_a_classes(o.A, o.lda, K);
  const int sms = info->sm_count;
  RcPlan pl;
  if (!rc_plan(M, N, K, p.a_classes, sms, &pl)) return TG_ERR_INTERNAL;  // a bad tuning width, or no room for two stages
  p.bn = pl.bn;
  p.n_tiles = pl.n_tiles;
  p.panels = pl.panels;
  const int msub = pl.msub, splits = pl.splits;
  p.msub = msub;
  if (!encode_classes(maps.a, o.A, M, K, o.lda, p.a_classes, 64, 128 * msub, CU_TENSOR_MAP_SWIZZLE_128B, p.a_shift,
                      p.rows_in_class))
    return TG_ERR_LAUNCH;
  int mt = 0, kb_max = 0;
  for (int c = 0; c < p.a_classes; ++c) {
    p.tile_start[c] = mt;
    mt += (p.rows_in_class[c] + 128 * msub - 1) / (128 * msub);
    const int kb = static_cast<int>((K + p.a_shift[c] + 63) / 64);
    kb_max = kb > kb_max ? kb : kb_max;
  }
  p.tile_start[p.a_classes] = mt;
  p.m_tiles = mt;
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.group_m = tune_int("TG_TUNE_RC_GROUP_M", 8);
  if (p.group_m < 1) p.group_m = 1;
  const bool realign_b = !((reinterpret_cast<uintptr_t>(o.B) & 15u) == 0 && o.ldb % 8 == 0);
  p.B = static_cast<const __half*>(o.B);
  p.ldb = o.ldb;
  if (!realign_b && !encode_2d(&maps.b, o.B, K, N, o.ldb, 64, 64)) {
    return TG_ERR_LAUNCH;
  }
  const int ring = pl.ring;
  p.ring_stage_bytes = pl.ring_bytes;
  p.ring_stages = ring;
  p.idesc = make_idesc_f16_f32(128, p.bn, false, true);
  p.wait_budget_ns = wait_budget(kb_max);
  const int smem = kRcFixed + ring * p.ring_stage_bytes;
  p.splits = splits;
  const bool b_deep = realign_b && pl.b_deep;
  if (splits > 1) {
    if (p.num_tiles > 65535) return TG_ERR_INVALID_ARG;
    if (!realign_b) return launch_rc_cfg<false, true>(maps, p, smem, splits, p.num_tiles, stream, info);
    return b_deep ? launch_rc_cfg<true, true, true>(maps, p, smem, splits, p.num_tiles, stream, info)
                  : launch_rc_cfg<true, true>(maps, p, smem, splits, p.num_tiles, stream, info);
  }
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  if (!realign_b) return launch_rc_cfg<false, false>(maps, p, smem, grid, 1, stream, info);
  return b_deep ? launch_rc_cfg<true, false, true>(maps, p, smem, grid, 1, stream, info)
                : launch_rc_cfg<true, false>(maps, p, smem, grid, 1, stream, info);
}

__global__ void wait_timeout_selftest_kernel(uint64_t budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: this wait must give up by itself.
    mbar_wait(&bar, 0, &abort_flag, budget_ns, 0xEE);
  }
  __syncthreads();
}

tg_status launch_path(int path, const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  switch (path) {
    case TG_PATH_TC:
      return launch_tc<false>(o, stream, info);
    case TG_PATH_TC_EDGE:
      return launch_tc<true>(o, stream, info);
    case TG_PATH_SKINNY:
      return launch_skinny(o, stream, info);
    case TG_PATH_TC_PAIR:
      return launch_tc_pair(o, stream, info, 256);
    case TG_PATH_TC_PAIR512:
      return launch_tc_pair(o, stream, info, 512);
    case TG_PATH_RC:
      return launch_rc(o, stream, info);
    default:
      return TG_ERR_INTERNAL;
  }
}

template <typename Kernel, typename Params>
tg_status launch_simple(Kernel kernel, const Params& params, int64_t work_items, int per_thread,
                        cudaStream_t stream, DeviceInfo* info) {
  int64_t blocks = (work_items + 256 * per_thread - 1) / (256 * per_thread);
  const int64_t cap = static_cast<int64_t>(info->sm_count) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, 1);
  if (cudaLaunchKernelEx(&cfg, kernel, params) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

tg_status launch_pad(const void* src, int64_t src_ld, void* dst, int64_t rows, int64_t cols, int64_t cols_pad,
                     cudaStream_t stream, DeviceInfo* info) {
  RepackParams rp;
  rp.src = static_cast<const __half*>(src);
  rp.dst = static_cast<__half*>(dst);
  rp.src_ld = src_ld;
  rp.rows = static_cast<int>(rows);
  rp.cols = static_cast<int>(cols);
  rp.cols_pad = static_cast<int>(cols_pad);
  rp.chunks = rows * (cols_pad / 8);
  return launch_simple(pad_rows_kernel, rp, rp.chunks, 4, stream, info);
}

tg_status launch_unpad(const void* src, int64_t cols_pad, void* dst, int64_t dst_ld, int64_t rows, int64_t cols,
                       cudaStream_t stream, DeviceInfo* info) {
  UnpadParams up;
  up.src = static_cast<const __half*>(src);
  up.dst = static_cast<__half*>(dst);
  up.dst_ld = dst_ld;
  up.rows = static_cast<int>(rows);
  up.cols = static_cast<int>(cols);
  up.cols_pad = static_cast<int>(cols_pad);
  up.blocks_per_row = static_cast<int>(cols / 8 + 2);
  up.blocks = rows * up.blocks_per_row;
  return launch_simple(unpad_rows_kernel, up, up.blocks, 4, stream, info);
}

// K == 0: C = ReLU(bias), or +0 without a bias (the empty sum).
tg_status launch_k_zero(const Operands& o, cudaStream_t stream, DeviceInfo* info) {
  if (o.bias == nullptr) {
    const cudaError_t e = (o.ldc == o.N)
        ? cudaMemsetAsync(o.C, 0, static_cast<size_t>(2 * o.M * o.N), stream)
        : cudaMemset2DAsync(o.C, static_cast<size_t>(2 * o.ldc), 0, static_cast<size_t>(2 * o.N),
                            static_cast<size_t>(o.M), stream);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return TG_ERR_LAUNCH;
    }
    return TG_OK;
  }
  BiasRowsParams bp;
  bp.C = static_cast<__half*>(o.C);
  bp.bias = static_cast<const __half*>(o.bias);
  bp.ldc = o.ldc;
  bp.M = static_cast<int>(o.M);
  bp.N = static_cast<int>(o.N);
  return launch_simple(bias_relu_rows_kernel, bp, o.M * o.N, 1, stream, info);
}

tg_status run(const Problem& p, void* stream_ptr, int path, void* ws, int64_t ws_bytes) {
  if (!problem_valid(p)) return TG_ERR_INVALID_ARG;
  if (ws_bytes < 0 || (ws_bytes > 0 && ws == nullptr)) return TG_ERR_INVALID_ARG;
  if (path == TG_PATH_AUTO) path = select_path(p, ws ? ws_bytes : 0);
  if (!path_supports(path, p)) return TG_ERR_INVALID_ARG;
  if (path == TG_PATH_NONE) return TG_OK;
  RepackPlan plan;
  if (path == TG_PATH_REPACK) {
    plan = chosen_plan(p, ws ? ws_bytes : 0);
    if (ws == nullptr || ws_bytes < plan.bytes || plan.bytes == 0 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
      return TG_ERR_INVALID_ARG;
    if (ranges_overlap(ws, plan.bytes, p.A, span_a(p)) || ranges_overlap(ws, plan.bytes, p.B, span_b(p)) ||
        ranges_overlap(ws, plan.bytes, p.C, span_c(p)) || (p.bias && ranges_overlap(ws, plan.bytes, p.bias, 2 * p.N)))
      return TG_ERR_INVALID_ARG;
  }
  // The residue-class kernel reads a padded copy of B when the workspace holds one.
  int64_t rc_b_bytes = 0;
  if (path == TG_PATH_RC && ws != nullptr) {
    const int64_t need = rc_b_copy_bytes(p);
    if (need > 0 && ws_bytes >= need) {
      if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ranges_overlap(ws, need, p.A, span_a(p)) ||
          ranges_overlap(ws, need, p.B, span_b(p)) || ranges_overlap(ws, need, p.C, span_c(p)) ||
          (p.bias && ranges_overlap(ws, need, p.bias, 2 * p.N)))
        return TG_ERR_INVALID_ARG;
      rc_b_bytes = need;
    }
  }
  int dev = 0;
  DeviceInfo* info = nullptr;
  tg_status st = current_device(dev, info);
  if (st != TG_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int inner = (path == TG_PATH_REPACK) ? inner_path(p, plan.pad_c) : path;
  for (int64_t e = 0; e < p.batch; ++e) {
    Operands o{static_cast<const uint8_t*>(p.A) + 2 * e * p.sa,
               p.lda,
               p.a_km,
               static_cast<const uint8_t*>(p.B) + 2 * e * p.sb,
               p.ldb,
               p.b_nk,
               static_cast<uint8_t*>(p.C) + 2 * e * p.sc,
               p.ldc,
               p.bias,
               p.M,
               p.N,
               p.K,
               c_rows_aligned(p)};
    if (path == TG_PATH_ZERO) {
      st = launch_k_zero(o, stream, info);
    } else if (path == TG_PATH_RC && rc_b_bytes > 0) {
      // B padded into the workspace, so TMA loads it as it is.
      const int64_t np = (p.N + 7) / 8 * 8;
      st = launch_pad(o.B, o.ldb, ws, p.K, p.N, np, stream, info);
      if (st != TG_OK) return st;
      o.B = ws;
      o.ldb = np;
      st = launch_path(path, o, stream, info);
    } else if (path == TG_PATH_REPACK) {
      uint8_t* base = static_cast<uint8_t*>(ws);
      if (plan.pad_a) {
        const int64_t rows = p.a_km ? p.K : p.M, cols = p.a_km ? p.M : p.K, cols_pad = p.a_km ? plan.mp : plan.kp;
        st = launch_pad(o.A, o.lda, base + plan.off_a, rows, cols, cols_pad, stream, info);
        if (st != TG_OK) return st;
        o.A = base + plan.off_a;
        o.lda = cols_pad;
      }
      if (plan.pad_b) {
        const int64_t rows = p.b_nk ? p.N : p.K, cols = p.b_nk ? p.K : p.N, cols_pad = p.b_nk ? plan.kp : plan.np;
        st = launch_pad(o.B, o.ldb, base + plan.off_b, rows, cols, cols_pad, stream, info);
        if (st != TG_OK) return st;
        o.B = base + plan.off_b;
        o.ldb = cols_pad;
      }
      if (plan.pad_c) {
        // The GEMM writes the padded C; the realigning copy moves it into C.
        void* c_final = o.C;
        o.C = base + plan.off_c;
        o.ldc = plan.np;
        o.c_aligned = true;
        st = launch_path(inner, o, stream, info);
        if (st != TG_OK) return st;
        st = launch_unpad(base + plan.off_c, plan.np, c_final, p.ldc, p.M, p.N, stream, info);
      } else {
        st = launch_path(inner, o, stream, info);
      }
    } else {
      st = launch_path(path, o, stream, info);
    }
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

// Options of tg_gemm_relu_f16_ex as a Problem (NULL options: dense defaults).
bool problem_from_options(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                          const tg_gemm_options* opt, Problem& p, int& path) {
  p = dense_problem(A, B, C, M, N, K);
  path = TG_PATH_AUTO;
  if (opt == nullptr) return true;
  if (opt->b_layout != TG_B_KN && opt->b_layout != TG_B_NK) return false;
  if (opt->a_layout != TG_A_MK && opt->a_layout != TG_A_KM) return false;
  if (opt->reserved != 0) return false;
  p.b_nk = opt->b_layout == TG_B_NK;
  p.a_km = opt->a_layout == TG_A_KM;
  p.lda = opt->lda ? opt->lda : (p.a_km ? M : K);
  p.ldb = opt->ldb ? opt->ldb : (p.b_nk ? K : N);
  p.ldc = opt->ldc ? opt->ldc : N;
  p.bias = opt->bias;
  p.batch = opt->batch ? opt->batch : 1;
  p.sa = opt->stride_a;
  p.sb = opt->stride_b;
  p.sc = opt->stride_c;
  path = opt->path;
  if (path == TG_PATH_REPACK) return false;  // chosen by the library when a workspace is given
  return true;
}

// ---------------------------------------------------------------------------
// MXFP8 grouped GEMM
// ---------------------------------------------------------------------------

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Stacked rows of A / C for these group sizes (each group padded to 128
// rows), or -1 if a size is negative or there are too many groups.
int64_t mx_rows(const int64_t* m_sizes, int32_t groups) {
  if (groups < 0 || groups > kMxMaxGroups || (groups > 0 && m_sizes == nullptr)) return -1;
  int64_t rows = 0;
  for (int32_t g = 0; g < groups; ++g) {
    if (m_sizes[g] < 0 || m_sizes[g] > INT_MAX) return -1;
    rows += round_up(m_sizes[g], 128);
    if (rows > INT_MAX) return -1;
  }
  return rows;
}

// Bytes of a blocked UE8M0 scale array for `rows` rows and K elements.
int64_t mx_scale_bytes(int64_t rows, int64_t K) { return round_up(rows, 128) * round_up(K / 32, 4); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool encode_2d_u8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows,
                  bool swizzle128 = true) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Bytes of a blocked scale array for `rows` rows and `scales` scale columns.
int64_t blocked_scale_bytes(int64_t rows, int64_t scales) { return round_up(rows, 128) * round_up(scales, 4); }

// Instruction descriptor of a block-scaled MMA of M x 256.
template <int KIND>
uint32_t blockscaled_idesc(int M, int a_format, int b_format) {
  return KIND == kKindNvf4 ? make_idesc_nvf4(M, 256) : make_idesc_mxf8(M, 256, a_format, b_format, 0, 0);
}

// Shared launcher of the block-scaled grouped kernels (one kind each):
// persistent 128 x 256 tiles over the stacked rows of all groups.
template <int KIND>
tg_status run_blockscaled_grouped(const void* A, const void* SFA, const void* B, const void* SFB, void* C,
                                  const int64_t* m_sizes, int32_t groups, int64_t N, int64_t K, int a_format,
                                  int b_format, float alpha, int32_t relu, void* stream) {
  using Cfg = MxCfg<KIND>;
  constexpr int kBlock = KIND == kKindNvf4 ? 16 : 32;
  constexpr int kMmaK = KIND == kKindNvf4 ? 64 : 32;
  constexpr int kElemsPerByte = KIND == kKindNvf4 ? 2 : 1;
  const int64_t rows = mx_rows(m_sizes, groups);
  if (rows < 0 || N < 0 || K < 0 || K % kMmaK != 0 || N % 8 != 0 || K > INT_MAX || (relu != 0 && relu != 1))
    return TG_ERR_INVALID_ARG;
  if (static_cast<int64_t>(groups) * N > INT_MAX - 256) return TG_ERR_INVALID_ARG;
  if (rows == 0 || N == 0) return TG_OK;
  if (C == nullptr || !aligned16(C)) return TG_ERR_INVALID_ARG;
  const int64_t c_bytes = rows * N * 2;
  const int64_t row_bytes = K / kElemsPerByte;
  if (K > 0) {
    if (!A || !B || !SFA || !SFB || !aligned16(A) || !aligned16(B) || !aligned16(SFA) || !aligned16(SFB))
      return TG_ERR_INVALID_ARG;
    const int64_t a_bytes = rows * row_bytes, b_bytes = static_cast<int64_t>(groups) * N * row_bytes;
    const int64_t sfa_bytes = blocked_scale_bytes(rows, K / kBlock);
    const int64_t sfb_bytes = groups * blocked_scale_bytes(N, K / kBlock);
    if (ranges_overlap(C, c_bytes, A, a_bytes) || ranges_overlap(C, c_bytes, B, b_bytes) ||
        ranges_overlap(C, c_bytes, SFA, sfa_bytes) || ranges_overlap(C, c_bytes, SFB, sfb_bytes))
      return TG_ERR_INVALID_ARG;
  }
  int dev = 0;
  DeviceInfo* info = nullptr;
  tg_status st = current_device(dev, info);
  if (st != TG_OK) return st;

  MxParams p;
  std::memset(&p, 0, sizeof p);
  p.SFA = static_cast<const uint8_t*>(SFA);
  p.SFB = static_cast<const uint8_t*>(SFB);
  p.C = static_cast<__nv_bfloat16*>(C);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.k_stages = static_cast<int>((row_bytes + Cfg::BK - 1) / Cfg::BK);
  p.k_mmas = static_cast<int>(K / kMmaK);
  p.atoms_k = static_cast<int>(round_up(K / kBlock, 4) / 4);
  p.alpha = alpha;
  p.n_tiles = static_cast<int>((N + Cfg::BN - 1) / Cfg::BN);
  p.m_tiles = static_cast<int>(rows / Cfg::BM);
  p.groups = groups;
  p.n_atoms = static_cast<int>((N + 127) / 128);
  p.relu = relu;
  p.wait_budget_ns = wait_budget(p.k_stages * 2);
  int tile = 0;
  for (int32_t g = 0; g < groups; ++g) {
    p.tile_start[g] = tile;
    p.m_size[g] = static_cast<int>(m_sizes[g]);
    tile += static_cast<int>(round_up(m_sizes[g], 128) / 128);
  }
  p.tile_start[groups] = tile;

  CUtensorMap ta, tb;
  std::memset(&ta, 0, sizeof ta);
  std::memset(&tb, 0, sizeof tb);
  if (K > 0) {
    if (!encode_2d_u8(&ta, A, rows, row_bytes, Cfg::BK, Cfg::BM)) return TG_ERR_LAUNCH;
    if (!encode_2d_u8(&tb, B, static_cast<int64_t>(groups) * N, row_bytes, Cfg::BK, Cfg::BN)) return TG_ERR_LAUNCH;
  }
  auto kernel = gemm_blockscaled_grouped_kernel<KIND>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!info->mx_attr[KIND]) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) !=
          cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->mx_attr[KIND] = true;
    }
  }
  p.group_m = tune_int("TG_TUNE_MX_GROUP_M", 16);
  if (p.group_m < 1) p.group_m = 1;
  p.num_tiles = static_cast<int>(static_cast<int64_t>(p.m_tiles) * p.n_tiles);
  p.idesc = blockscaled_idesc<KIND>(Cfg::BM, a_format, b_format);
  const int ctas = tune_int("TG_TUNE_MX_CTAS", info->sm_count);
  if (ctas < 1) return TG_ERR_INVALID_ARG;
  const int grid = p.num_tiles < ctas ? p.num_tiles : ctas;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::SMEM_BYTES);
  LaunchAttrs la;
  la.fill(cfg, 1);
  if (cudaLaunchKernelEx(&cfg, kernel, ta, tb, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

tg_status run_mxf8_grouped(const void* A, const void* SFA, const void* B, const void* SFB, void* C,
                           const int64_t* m_sizes, int32_t groups, int64_t N, int64_t K, int32_t a_format,
                           int32_t b_format, int32_t relu, void* stream) {
  if ((a_format != TG_FP8_E4M3 && a_format != TG_FP8_E5M2) || (b_format != TG_FP8_E4M3 && b_format != TG_FP8_E5M2))
    return TG_ERR_INVALID_ARG;
  return run_blockscaled_grouped<kKindMxf8>(A, SFA, B, SFB, C, m_sizes, groups, N, K, a_format, b_format, 1.0f, relu,
                                            stream);
}

tg_status run_nvf4_grouped(const void* A, const void* SFA, const void* B, const void* SFB, void* C,
                           const int64_t* m_sizes, int32_t groups, int64_t N, int64_t K, float alpha, int32_t relu,
                           void* stream) {
  if (!std::isfinite(alpha)) return TG_ERR_INVALID_ARG;
  return run_blockscaled_grouped<kKindNvf4>(A, SFA, B, SFB, C, m_sizes, groups, N, K, 0, 0, alpha, relu, stream);
}

// ---------------------------------------------------------------------------
// 4-bit weight-only GEMM (W4A16)
// ---------------------------------------------------------------------------

constexpr int64_t kW4FusedMaxM = 256;

bool w4_sizes_valid(int64_t M, int64_t N, int64_t K, int32_t group) {
  if (M < 0 || N < 0 || K < 0 || M > INT_MAX || N > INT_MAX || K > INT_MAX) return false;
  return !(group < 32 || (group & (group - 1)) != 0 || K % 64 != 0 || (K > 0 && K % group != 0));
}

bool w4_args_valid(const void* A, const void* Wq, const void* S, const void* C, int64_t M, int64_t N, int64_t K,
                   int32_t group) {
  if (!w4_sizes_valid(M, N, K, group)) return false;
  if (M == 0 || N == 0) return true;
  if (!C || (reinterpret_cast<uintptr_t>(C) & 1u)) return false;
  if (K == 0) return true;
  if (!A || !Wq || !S || !aligned16(A) || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(S) & 1u)) return false;
  const int64_t c_bytes = 2 * M * N;
  return !(ranges_overlap(C, c_bytes, A, 2 * M * K) || ranges_overlap(C, c_bytes, Wq, N * K / 2) ||
           ranges_overlap(C, c_bytes, S, 2 * N * (K / group)));
}

int64_t w4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return (M > kW4FusedMaxM && N > 0 && K > 0) ? round_up(2 * N * K, 256) : 0;
}

tg_status launch_dequant_w4(const void* Wq, const void* S, void* W, int64_t N, int64_t K, int32_t group,
                            cudaStream_t stream, DeviceInfo* info) {
  DequantParams dp;
  dp.Wq = static_cast<const uint8_t*>(Wq);
  dp.S = static_cast<const __half*>(S);
  dp.W = static_cast<__half*>(W);
  dp.N = N;
  dp.K = K;
  dp.group = group;
  dp.chunks = N * K / 8;
  return launch_simple(dequant_w4_kernel, dp, dp.chunks, 4, stream, info);
}

tg_status launch_w4a16_fused(const void* A, const void* Wq, const void* S, void* C, int64_t M, int64_t N, int64_t K,
                             int32_t group, cudaStream_t stream, DeviceInfo* info) {
  using Cfg = W4Cfg;
  constexpr int kMaxSmem = 227 * 1024;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!info->w4_attr) {
      if (cudaFuncSetAttribute(gemm_relu_w4a16_skinny_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kMaxSmem) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->w4_attr = true;
    }
  }
  W4Params p;
  std::memset(&p, 0, sizeof p);
  p.C = static_cast<__half*>(C);
  p.S = static_cast<const __half*>(S);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.group = group;
  p.m_pad = static_cast<int>((M + 15) / 16 * 16);
  p.k_blocks = static_cast<int>(K / Cfg::BK);
  p.a_stage_bytes = static_cast<uint32_t>(p.m_pad * 128);
  const int ring = Cfg::ring_stage_bytes(p.m_pad);
  // Two CTAs per SM for small M (each within half the shared memory), one
  // with a deeper ring otherwise.
  const bool two_per_sm = tune_int("TG_TUNE_W4_TWO_PER_SM", p.m_pad <= 32 ? 1 : 0) != 0;
  p.wdq_slots = tune_int("TG_TUNE_W4_WDQ", two_per_sm ? 3 : Cfg::MAX_WDQ_SLOTS);
  if (p.wdq_slots < 2 || p.wdq_slots > Cfg::MAX_WDQ_SLOTS) return TG_ERR_INVALID_ARG;
  const int budget = two_per_sm ? 113 * 1024 : kMaxSmem;
  int stages = (budget - Cfg::smem_bytes(p.m_pad, 0, p.wdq_slots)) / ring;
  const int cap = tune_int("TG_TUNE_W4_STAGES", Cfg::MAX_STAGES);
  if (stages > cap) stages = cap;
  if (stages > Cfg::MAX_STAGES) stages = Cfg::MAX_STAGES;
  if (stages < 2) return TG_ERR_INTERNAL;
  // The fp32 partial [M_pad][128] reuses the rings after the main loop.
  if (p.wdq_slots * Cfg::WDQ_BYTES + stages * ring < p.m_pad * Cfg::PANEL * 4) return TG_ERR_INTERNAL;
  p.stages = stages;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.m_pad)) cols <<= 1;
  p.tmem_cols = cols;
  p.idesc = make_idesc_f16_f32(Cfg::PANEL, p.m_pad, false, false);
  p.c_aligned = ((reinterpret_cast<uintptr_t>(C) & 7u) == 0 && N % 4 == 0) ? 1 : 0;
  p.wait_budget_ns = wait_budget(p.k_blocks);
  const int panels = static_cast<int>((N + Cfg::PANEL - 1) / Cfg::PANEL);
  if (panels > 65535) return TG_ERR_INVALID_ARG;
  int splits = tune_int("TG_TUNE_W4_SPLITS", (two_per_sm ? 2 : 1) * info->sm_count / panels);
  splits = splits < 1 ? 1 : (splits > 8 ? 8 : splits);
  if (splits > p.k_blocks) splits = p.k_blocks;
  p.splits = splits;

  CUtensorMap ta, tw, ts;
  std::memset(&ts, 0, sizeof ts);
  if (!encode_2d(&ta, A, M, K, K, 64, p.m_pad)) return TG_ERR_LAUNCH;
  if (!encode_2d_u8(&tw, Wq, N, K / 2, Cfg::BK / 2, Cfg::PANEL, false)) return TG_ERR_LAUNCH;
  // Scales by TMA when a row of them is a multiple of 16 bytes (and the base
  // is 16-byte aligned); otherwise the dequantizing threads read them.
  const int64_t groups_per_row = K / group;
  p.scale_tma = (groups_per_row % 8 == 0 && aligned16(S) && tune_int("TG_TUNE_W4_SCALE_TMA", 1)) ? 1 : 0;
  if (p.scale_tma && !encode_2d_f16_plain(&ts, S, N, groups_per_row, 8, Cfg::PANEL)) return TG_ERR_LAUNCH;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(panels), 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::smem_bytes(p.m_pad, stages, p.wdq_slots));
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, static_cast<unsigned>(splits));
  if (cudaLaunchKernelEx(&cfg, gemm_relu_w4a16_skinny_kernel, ta, tw, ts, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

// Splits of K for the decode kernel (M <= 16): the most (up to 8) that keep
// each CTA's slice a multiple of kW4DecodeStepK and at most
// kW4DecodeMaxSplit; 0 when the shape does not suit it (K % 256 != 0, K too
// long, or turned off).
int w4_decode_splits(int64_t M, int64_t N, int64_t K) {
  if (M > 16 || K <= 0 || K % kW4DecodeStepK != 0 || (N + kW4DecodePanel - 1) / kW4DecodePanel > 65535) return 0;
  if (!tune_int("TG_TUNE_W4_DECODE", 1)) return 0;
  for (int s = 8; s >= 1; s >>= 1)
    if (K % (kW4DecodeStepK * s) == 0 && K / s <= kW4DecodeMaxSplit) return s;
  return 0;
}

tg_status launch_w4a16_decode(const void* A, const void* Wq, const void* S, void* C, int64_t M, int64_t N,
                              int64_t K, int32_t group, int splits, cudaStream_t stream, DeviceInfo* info) {
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!info->w4_decode_attr) {
      if (cudaFuncSetAttribute(gemm_relu_w4a16_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               w4_decode_smem_bytes(kW4DecodeMaxSplit)) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->w4_decode_attr = true;
    }
  }
  W4DecodeParams p;
  std::memset(&p, 0, sizeof p);
  p.A = static_cast<const __half*>(A);
  p.Wq = static_cast<const uint8_t*>(Wq);
  p.S = static_cast<const __half*>(S);
  p.C = static_cast<__half*>(C);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  int shift = 0;
  while ((1 << shift) < group) ++shift;
  p.group_shift = shift;
  p.k_split = static_cast<int>(K / splits);
  const int panels = static_cast<int>((N + kW4DecodePanel - 1) / kW4DecodePanel);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(panels), 1);
  cfg.blockDim = dim3(kW4DecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(w4_decode_smem_bytes(p.k_split));
  cfg.stream = stream;
  LaunchAttrs la;
  la.fill(cfg, static_cast<unsigned>(splits));
  if (cudaLaunchKernelEx(&cfg, gemm_relu_w4a16_decode_kernel, p) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  return TG_OK;
}

tg_status run_w4a16(const void* A, const void* Wq, const void* S, void* C, int64_t M, int64_t N, int64_t K,
                    int32_t group, void* stream_ptr, void* ws, int64_t ws_bytes) {
  if (!w4_args_valid(A, Wq, S, C, M, N, K, group)) return TG_ERR_INVALID_ARG;
  if (ws_bytes < 0 || (ws_bytes > 0 && ws == nullptr)) return TG_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return TG_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  int dev = 0;
  DeviceInfo* info = nullptr;
  tg_status st = current_device(dev, info);
  if (st != TG_OK) return st;
  if (K == 0) {
    if (cudaMemsetAsync(C, 0, static_cast<size_t>(2 * M * N), stream) != cudaSuccess) {
      cudaGetLastError();
      return TG_ERR_LAUNCH;
    }
    return TG_OK;
  }
  if (const int splits = w4_decode_splits(M, N, K))
    return launch_w4a16_decode(A, Wq, S, C, M, N, K, group, splits, stream, info);
  if (M <= kW4FusedMaxM) return launch_w4a16_fused(A, Wq, S, C, M, N, K, group, stream, info);
  // Large M: dequantize into the workspace, then the fp16 tensor-core GEMM
  // with the weight in the N x K layout.
  const int64_t need = w4_workspace_bytes(M, N, K);
  if (ws_bytes < need || !aligned16(ws) || ranges_overlap(ws, need, A, 2 * M * K) ||
      ranges_overlap(ws, need, C, 2 * M * N) || ranges_overlap(ws, need, Wq, N * K / 2) ||
      ranges_overlap(ws, need, S, 2 * N * (K / group)))
    return TG_ERR_INVALID_ARG;
  st = launch_dequant_w4(Wq, S, ws, N, K, group, stream, info);
  if (st != TG_OK) return st;
  Problem p = dense_problem(A, ws, C, M, N, K);
  p.b_nk = true;
  p.ldb = K;
  return run(p, stream_ptr, TG_PATH_AUTO, nullptr, 0);
}

}  // namespace
}  // namespace tg

extern "C" {

tg_status tg_gemm_mxf8_grouped(const void* A, const void* SFA, const void* B, const void* SFB, void* C,
                               const int64_t* m_sizes, int32_t groups, int64_t N, int64_t K, int32_t a_format,
                               int32_t b_format, int32_t relu, void* stream) {
  return tg::run_mxf8_grouped(A, SFA, B, SFB, C, m_sizes, groups, N, K, a_format, b_format, relu, stream);
}

int64_t tg_mx_grouped_rows(const int64_t* m_sizes, int32_t groups) { return tg::mx_rows(m_sizes, groups); }

int64_t tg_mx_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 32 != 0) return -1;
  return tg::mx_scale_bytes(rows, K);
}

tg_status tg_gemm_nvf4_grouped(const void* A, const void* SFA, const void* B, const void* SFB, void* C,
                               const int64_t* m_sizes, int32_t groups, int64_t N, int64_t K, float alpha,
                               int32_t relu, void* stream) {
  return tg::run_nvf4_grouped(A, SFA, B, SFB, C, m_sizes, groups, N, K, alpha, relu, stream);
}

tg_status tg_gemm_relu_w4a16(const void* A, const void* Wq, const void* scales, void* C, int64_t M, int64_t N,
                              int64_t K, int32_t group, void* stream, void* workspace, int64_t workspace_bytes) {
  return tg::run_w4a16(A, Wq, scales, C, M, N, K, group, stream, workspace, workspace_bytes);
}

int tg_w4a16_kernel(int64_t M, int64_t N, int64_t K, int32_t group) {
  if (!tg::w4_sizes_valid(M, N, K, group)) return TG_W4_INVALID;
  if (M == 0 || N == 0 || K == 0) return TG_W4_NONE;
  if (tg::w4_decode_splits(M, N, K) > 0) return TG_W4_DECODE;
  return M <= tg::kW4FusedMaxM ? TG_W4_FUSED : TG_W4_DEQUANT_GEMM;
}

int64_t tg_w4a16_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group) {
  if (M < 0 || N < 0 || K < 0 || group < 32 || (group & (group - 1)) != 0 || K % 64 != 0 || (K > 0 && K % group != 0))
    return -1;
  return tg::w4_workspace_bytes(M, N, K);
}

tg_status tg_dequant_w4_f16(const void* Wq, const void* scales, void* W, int64_t N, int64_t K, int32_t group,
                            void* stream) {
  if (N < 0 || K < 0 || group < 32 || (group & (group - 1)) != 0 || K % 64 != 0 || (K > 0 && K % group != 0))
    return TG_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return TG_OK;
  if (!Wq || !scales || !W || !tg::aligned16(Wq) || !tg::aligned16(W) ||
      (reinterpret_cast<uintptr_t>(scales) & 1u) ||
      tg::ranges_overlap(W, 2 * N * K, Wq, N * K / 2) || tg::ranges_overlap(W, 2 * N * K, scales, 2 * N * (K / group)))
    return TG_ERR_INVALID_ARG;
  int dev = 0;
  tg::DeviceInfo* info = nullptr;
  tg_status st = tg::current_device(dev, info);
  if (st != TG_OK) return st;
  return tg::launch_dequant_w4(Wq, scales, W, N, K, group, static_cast<cudaStream_t>(stream), info);
}

int64_t tg_nvf4_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 16 != 0) return -1;
  return tg::blocked_scale_bytes(rows, K / 16);
}

tg_status tg_gemm_relu_f16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* stream) {
  return tg::run(tg::dense_problem(A, B, C, M, N, K), stream, TG_PATH_AUTO, nullptr, 0);
}

tg_status tg_gemm_relu_f16_path(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                                void* stream, int path) {
  if (path == TG_PATH_REPACK) return TG_ERR_INVALID_ARG;  // needs a workspace: tg_gemm_relu_f16_ws
  return tg::run(tg::dense_problem(A, B, C, M, N, K), stream, path, nullptr, 0);
}

tg_status tg_gemm_relu_f16_ws(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* stream,
                              void* workspace, int64_t workspace_bytes) {
  return tg::run(tg::dense_problem(A, B, C, M, N, K), stream, TG_PATH_AUTO, workspace, workspace_bytes);
}

tg_status tg_gemm_relu_f16_ex(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                              const tg_gemm_options* options, void* stream, void* workspace,
                              int64_t workspace_bytes) {
  tg::Problem p;
  int path = TG_PATH_AUTO;
  if (!tg::problem_from_options(A, B, C, M, N, K, options, p, path)) return TG_ERR_INVALID_ARG;
  return tg::run(p, stream, path, workspace, workspace_bytes);
}

int64_t tg_workspace_size_ex(const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K,
                             const tg_gemm_options* options) {
  tg::Problem p;
  int path = TG_PATH_AUTO;
  if (!tg::problem_from_options(A, B, const_cast<void*>(C), M, N, K, options, p, path) || !tg::problem_valid(p))
    return -1;
  return tg::workspace_bytes_needed(p);
}

int tg_select_path_ex(const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K,
                      const tg_gemm_options* options, int64_t workspace_bytes) {
  tg::Problem p;
  int path = TG_PATH_AUTO;
  if (!tg::problem_from_options(A, B, const_cast<void*>(C), M, N, K, options, p, path)) return -2;
  if (path != TG_PATH_AUTO) return tg::path_supports(path, p) ? path : -2;
  return tg::select_path(p, workspace_bytes);
}

tg_status tg_gemm_relu_f16_static_ws(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                                     void* stream) {
  const tg::Problem p = tg::dense_problem(A, B, C, M, N, K);
  if (!tg::problem_valid(p)) return TG_ERR_INVALID_ARG;
  // Only the copies of the operands are required (B's alone on the
  // residue-class route; A's and B's on the repack route, with a padded C
  // when it fits too).
  const int64_t need = tg::repack_bytes_needed(p);
  if (need > TG_STATIC_WORKSPACE_BYTES) return TG_ERR_TOO_LARGE;
  if (M == 0 || N == 0) return TG_OK;  // empty C: nothing to do
  int dev = 0;
  tg::DeviceInfo* info = nullptr;
  const tg_status st = tg::current_device(dev, info);
  if (st != TG_OK) return st;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(tg::g_mutex);
    if (info->static_ws == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, tg::g_static_workspace) != cudaSuccess || ptr == nullptr) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
      }
      info->static_ws = ptr;
    }
    ws = info->static_ws;
  }
  return tg::run(p, stream, TG_PATH_AUTO, ws, TG_STATIC_WORKSPACE_BYTES);
}

int64_t tg_workspace_size(const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K) {
  const tg::Problem p = tg::dense_problem(A, B, const_cast<void*>(C), M, N, K);
  if (!tg::problem_valid(p)) return -1;
  return tg::workspace_bytes_needed(p);
}

int tg_select_path_ws(const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K,
                      int64_t workspace_bytes) {
  return tg::select_path(tg::dense_problem(A, B, const_cast<void*>(C), M, N, K), workspace_bytes);
}

int tg_select_path(const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K) {
  return tg::select_path(tg::dense_problem(A, B, const_cast<void*>(C), M, N, K), 0);
}

int tg_path_supports(int path, const void* A, const void* B, const void* C, int64_t M, int64_t N, int64_t K) {
  return tg::path_supports(path, tg::dense_problem(A, B, const_cast<void*>(C), M, N, K)) ? 1 : 0;
}

tg_status tg_device_status(uint32_t* detail) {
  int dev = 0;
  tg::DeviceInfo* info = nullptr;
  tg_status st = tg::current_device(dev, info);
  if (st != TG_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, tg::g_device_error, sizeof word) != cudaSuccess ||
      cudaMemcpyToSymbol(tg::g_device_error, &zero, sizeof zero) != cudaSuccess) {
    cudaGetLastError();
    return TG_ERR_LAUNCH;
  }
  if (detail) *detail = word;
  if (word == 0) return TG_OK;
  if ((word & 0xff00u) == tg::kDevErrWaitTimeout) return TG_ERR_TIMEOUT;
  return TG_ERR_INTERNAL;
}

tg_status tg_wait_timeout_selftest(int64_t budget_ns, void* stream) {
  int dev = 0;
  tg::DeviceInfo* info = nullptr;
  tg_status st = tg::current_device(dev, info);
  if (st != TG_OK) return st;
  if (budget_ns < 1000) budget_ns = 1000;
  if (budget_ns > 10000000000ll) budget_ns = 10000000000ll;
  tg::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(budget_ns));
  return cudaGetLastError() == cudaSuccess ? TG_OK : TG_ERR_LAUNCH;
}

const char* tg_status_string(int status) {
  switch (status) {
    case TG_OK: return "ok";
    case TG_ERR_INVALID_ARG: return "invalid argument";
    case TG_ERR_UNSUPPORTED_DEVICE: return "unsupported or missing device (needs compute capability 10.0)";
    case TG_ERR_LAUNCH: return "kernel launch or CUDA call failed";
    case TG_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case TG_ERR_INTERNAL: return "internal error";
    case TG_ERR_TOO_LARGE: return "problem needs more scratch than the library's 16 MiB static workspace holds";
    default: return "unknown status";
  }
}

const char* tg_path_name(int path) {
  switch (path) {
    case TG_PATH_NONE: return "none";
    case TG_PATH_AUTO: return "auto";
    case TG_PATH_TC: return "tc";
    case TG_PATH_TC_EDGE: return "tc_edge";
    case TG_PATH_SKINNY: return "skinny";
    case TG_PATH_ZERO: return "zero";
    case TG_PATH_TC_PAIR: return "tc_pair";
    case TG_PATH_TC_PAIR512: return "tc_pair512";
    case TG_PATH_REPACK: return "repack";
    case TG_PATH_RC: return "rc";
    default: return "invalid";
  }
}

int tg_version(void) { return 100; }

}  // extern "C"
