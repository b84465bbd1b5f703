// gemm_tc.cuh -- persistent, warp-specialised tcgen05 kernel for
// C = ReLU(A . B), A (M x K) and B (K x N) row-major fp16, fp32 accumulation
// in tensor memory, fp16 C (M x N) row-major.
//
// The tile model follows the matmul_relu quick-start kernel ("TileLang" wiki
// page, "Programming model"): one output tile per (block_M x block_N) block
// of C over a ceildiv grid, A and B tiles staged in shared memory through a
// multi-stage pipelined K loop, a cleared fp32 accumulator, tile MMAs, then
// max(acc, 0) and a copy into the fp16 output.  On sm_100a:
//   * tiles are 128 x 256 x 64 (BM x BN x BK); a persistent grid of one CTA
//     per SM walks the tiles in grouped (L2-friendly) order;
//   * role warps: producer(s), one MMA-issuing warp that also owns TMEM, and
//     four epilogue warps;
//   * the fp32 accumulator lives in TMEM, double-buffered (2 x 256 columns),
//     so the epilogue of tile i overlaps the main loop of tile i+1;
//   * the first MMA of each tile runs with accumulate disabled, which is the
//     accumulator clear.
// Two operand-staging modes share the rest:
//   * TMA mode: one producer thread issues 2-D TMA loads with 128-byte
//     swizzle (needs 16-byte aligned bases and row strides); the hardware
//     zero-fills out-of-bounds boxes.
//   * EDGE mode: four producer warps load A and B with predicated 2-byte
//     loads (zero outside the matrix) and write the same swizzled layout, for
//     row strides that TMA cannot describe.
// The epilogue reads TMEM with tcgen05.ld, applies ReLU on fp32 (every value
// that is not > 0 becomes +0), rounds to fp16 (round to nearest even) and
// stores the rows that lie inside C.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace tg {

struct TcParams {
  const __half* A;
  const __half* B;
  __half* C;
  const __half* bias;    // optional fp16[N], added to every row before ReLU; nullptr = none
  int64_t lda, ldb, ldc; // row strides (elements) of A, of B as stored, and of C
  int b_kmajor;          // 1: B is stored N x K (rows of length K; C = A . B^T)
  int a_mnmajor;         // 1: A is stored K x M (rows of length M; C = A^T . B)
  int M, N, K;
  int m_tiles, n_tiles, num_tiles, k_blocks;
  int group_m;           // tile rows per raster group
  int store_streaming;   // 1: C stores with the streaming (evict-first) cache hint
  int l2_hints;          // bit 0: A loads evict-last; bit 1: B loads evict-last; bit 2: B loads evict-first
  int prefetch_kb;       // > 0: also prefetch into L2 the boxes this many k-blocks ahead
  int c_aligned;         // 1: every row of C starts on a 16-byte boundary (C aligned, N % 8 == 0)
  uint64_t wait_budget_ns;
};

template <bool EDGE>
struct TcCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 256;
  static constexpr int BK = 64;
  static constexpr int STAGES = 4;
  static constexpr int PRODUCER_WARPS = EDGE ? 8 : 1;
  static constexpr int MMA_WARP = PRODUCER_WARPS;
  static constexpr int EPI_WARP0 = MMA_WARP + 1;
  static constexpr int EPI_WARPS = 4;
  static constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
  static constexpr int A_BYTES = BM * BK * 2;          // 16 KiB
  static constexpr int B_BYTES = BK * BN * 2;          // 32 KiB
  static constexpr int B_CHUNK_BYTES = BK * 64 * 2;    // one 64-column swizzle panel: 8 KiB
  static constexpr int NUM_ACC = 2;
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + STAGES * (A_BYTES + B_BYTES) + BAR_BYTES;
  static constexpr uint32_t FULL_COUNT = EDGE ? PRODUCER_WARPS * 32 : 1;
};

// ReLU on two fp32 accumulator values (every value that is not > 0 becomes
// +0), rounded to fp16 (nearest even) and packed, the first in the low half.
__device__ __forceinline__ uint32_t relu_pack_f16x2(uint32_t a, uint32_t b) {
  const float x0 = __uint_as_float(a);
  const float x1 = __uint_as_float(b);
  const __half2 v = __floats2half2_rn(x0 > 0.0f ? x0 : 0.0f, x1 > 0.0f ? x1 : 0.0f);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 16 bias values bias[col .. col + 16) as fp32 (0 past N or without bias).
// All lanes of a warp ask for the same columns, so each load is a broadcast.
__device__ __forceinline__ void load_bias16(const __half* bias, int col, int N, float (&b)[16]) {
  if (bias == nullptr) {
#pragma unroll
    for (int e = 0; e < 16; ++e) b[e] = 0.0f;
    return;
  }
  const __half* src = bias + col;
  if (col + 16 <= N && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __half2 h2 = *reinterpret_cast<const __half2*>(&w[q]);
      const float2 f = __half22float2(h2);
      b[2 * q] = f.x;
      b[2 * q + 1] = f.y;
    }
    return;
  }
  const unsigned short* s16 = reinterpret_cast<const unsigned short*>(src);
#pragma unroll
  for (int e = 0; e < 16; ++e)
    b[e] = (col + e < N) ? __half2float(__ushort_as_half(__ldg(s16 + e))) : 0.0f;
}

// 8 bias values bias[col .. col + 8) as fp32 (0 past N or without bias): the
// narrower form of load_bias16 for epilogues short of registers.
__device__ __forceinline__ void load_bias8(const __half* bias, int col, int N, float (&b)[8]) {
  if (bias == nullptr) {
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = 0.0f;
    return;
  }
  const __half* src = bias + col;
  if (col + 8 <= N && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[q]));
      b[2 * q] = f.x;
      b[2 * q + 1] = f.y;
    }
    return;
  }
  const unsigned short* s16 = reinterpret_cast<const unsigned short*>(src);
#pragma unroll
  for (int e = 0; e < 8; ++e)
    b[e] = (col + e < N) ? __half2float(__ushort_as_half(__ldg(s16 + e))) : 0.0f;
}

// relu_pack_f16x2 of (a + bias_a, b + bias_b): the bias is added to the fp32
// accumulator with one fp32 addition before ReLU.
__device__ __forceinline__ uint32_t relu_pack_f16x2_bias(uint32_t a, uint32_t b, float ba, float bb) {
  return relu_pack_f16x2(__float_as_uint(__uint_as_float(a) + ba), __float_as_uint(__uint_as_float(b) + bb));
}

// Store 32 consecutive fp16 values of one row of C, packed two per word in
// h[0..15] (low half first), to crow[col0 .. col0 + n) with
// n = min(32, N - col0) >= 1.  With aligned rows: 16-byte stores (streaming
// cache hint on request).  Otherwise the row start is only 2-byte aligned:
// 4-byte stores of aligned pairs and 2-byte stores at either end.
__device__ __forceinline__ void store_row_chunk(__half* crow, int col0, int N, const uint32_t (&h)[16],
                                                bool aligned16, bool streaming) {
  if (aligned16) {
    uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (col0 + q * 8 < N) {
        const uint4 v = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        if (streaming)
          __stcs(reinterpret_cast<int4*>(dst + q), *reinterpret_cast<const int4*>(&v));
        else
          dst[q] = v;
      }
    }
    return;
  }
  unsigned short* dst = reinterpret_cast<unsigned short*>(crow + col0);
  const int n_here = min(32, N - col0);
  if ((reinterpret_cast<uintptr_t>(dst) & 2u) == 0) {
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (2 * q + 1 < n_here) reinterpret_cast<uint32_t*>(dst)[q] = h[q];
    if (n_here & 1) dst[n_here - 1] = static_cast<unsigned short>(h[(n_here - 1) >> 1] & 0xffffu);
  } else {
    dst[0] = static_cast<unsigned short>(h[0] & 0xffffu);
    uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + 1);
#pragma unroll
    for (int q = 0; q < 15; ++q)
      if (2 * q + 2 < n_here) d32[q] = __funnelshift_r(h[q], h[q + 1], 16);
    if (n_here >= 2 && (n_here & 1) == 0) dst[n_here - 1] = static_cast<unsigned short>(h[(n_here - 1) >> 1] >> 16);
  }
}

__device__ __forceinline__ void tile_coords(const TcParams& p, int t, int& m_blk, int& n_blk) {
  const int group_tiles = p.group_m * p.n_tiles;
  const int g = t / group_tiles;
  const int first_m = g * p.group_m;
  const int gm = min(p.m_tiles - first_m, p.group_m);
  const int local = t - g * group_tiles;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

// Swizzled byte offset of the 16-byte chunk `chunk` (0..7) of row `row` in a
// tile whose rows are 128 bytes: chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// EDGE mode: one 16-byte chunk of 8 consecutive fp16 values from a row-major
// matrix, zero where (row >= rows) or (col >= cols).  Scalar reference form.
__device__ __forceinline__ uint4 load_chunk_pred(const __half* base, int64_t ld, int row, int rows, int col,
                                                 int cols) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (row < rows) {
    const unsigned short* p = reinterpret_cast<const unsigned short*>(base) + static_cast<int64_t>(row) * ld;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = col + e;
      const uint32_t v = (c < cols) ? static_cast<uint32_t>(__ldg(p + c)) : 0u;
      w[e >> 1] |= v << ((e & 1) * 16);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// EDGE mode, fast form of load_chunk_pred for rows whose start is only
// 2-byte aligned, split so that a thread can issue the loads of several
// chunks before it uses any of them.  When the 8 values lie inside the row
// and the two 16-byte aligned blocks that cover them lie inside
// [base, end), the chunk is read with two aligned 16-byte loads and shifted
// into place; otherwise the caller falls back to the scalar form.  No byte
// outside [base, end) is ever read.
struct EdgeChunk {
  const uint4* src;  // first aligned block (valid when fast)
  uint32_t shift;    // byte offset of the chunk in the 32 loaded bytes: 0, 2, ..., 14
  bool fast;
};

__device__ __forceinline__ EdgeChunk edge_chunk_plan(const __half* base, const __half* end, int64_t ld, int row,
                                                     int rows, int col, int cols) {
  EdgeChunk c;
  c.fast = false;
  c.shift = 0;
  c.src = reinterpret_cast<const uint4*>(base);
  if (row < rows && col + 8 <= cols) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(base + static_cast<int64_t>(row) * ld + col);
    const uintptr_t a0 = a & ~uintptr_t(15);
    if (a0 >= reinterpret_cast<uintptr_t>(base) && a0 + 32 <= reinterpret_cast<uintptr_t>(end)) {
      c.fast = true;
      c.src = reinterpret_cast<const uint4*>(a0);
      c.shift = static_cast<uint32_t>(a - a0);
    }
  }
  return c;
}

__device__ __forceinline__ uint4 edge_realign(const uint4& lo, const uint4& hi, uint32_t sh) {
  uint32_t w0 = lo.x, w1 = lo.y, w2 = lo.z, w3 = lo.w, w4 = hi.x, w5 = hi.y, w6 = hi.z, w7 = hi.w;
  if (sh & 8u) {
    w0 = w2; w1 = w3; w2 = w4; w3 = w5; w4 = w6; w5 = w7;
  }
  if (sh & 4u) {
    w0 = w1; w1 = w2; w2 = w3; w3 = w4; w4 = w5;
  }
  const uint32_t bits = (sh & 2u) * 8u;  // 0 or 16
  return make_uint4(__funnelshift_r(w0, w1, bits), __funnelshift_r(w1, w2, bits), __funnelshift_r(w2, w3, bits),
                    __funnelshift_r(w3, w4, bits));
}

template <bool EDGE>
__global__ void __launch_bounds__(TcCfg<EDGE>::THREADS, 1)
    gemm_relu_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const TcParams p) {
  using Cfg = TcCfg<EDGE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + Cfg::STAGES * Cfg::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::STAGES * (Cfg::A_BYTES + Cfg::B_BYTES));
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + Cfg::STAGES;
  uint64_t* acc_full_bar = bars + 2 * Cfg::STAGES;
  uint64_t* acc_empty_bar = acc_full_bar + Cfg::NUM_ACC;
  uint64_t* mma_done_bar = acc_empty_bar + Cfg::NUM_ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full_bar[s], Cfg::FULL_COUNT);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < Cfg::NUM_ACC; ++b) {
      mbar_init(&acc_full_bar[b], 1);
      mbar_init(&acc_empty_bar[b], Cfg::EPI_WARPS);
    }
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    if (!EDGE) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
    }
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_alloc_permit();
  }
  tcgen05_fence_before_sync();
  __syncthreads();
  tcgen05_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched only shared memory, TMEM and kernel parameters;
  // global memory is used only after the previous grid on the stream is done.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp < Cfg::PRODUCER_WARPS) {
    // ------------------------------------------------------------------
    // Producer: stage A (BM x BK) and B (BK x BN) tiles into the ring.
    // ------------------------------------------------------------------
    if (!EDGE) {
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int last_parity[Cfg::STAGES];
#pragma unroll
        for (int s = 0; s < Cfg::STAGES; ++s) last_parity[s] = -1;
        bool ok = true;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
          int m_blk, n_blk;
          tile_coords(p, t, m_blk, n_blk);
          const int m0 = m_blk * Cfg::BM;
          const int n0 = n_blk * Cfg::BN;
          for (int kb = 0; kb < p.k_blocks; ++kb) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full_bar[stage], Cfg::A_BYTES + Cfg::B_BYTES);
            const int k0 = kb * Cfg::BK;
            if (p.a_mnmajor) {
              // A stored K x M: two 64-row (m) x 64 k boxes, MN-major like B.
              tma_load_2d(a_smem + stage * Cfg::A_BYTES, &tmap_a, &full_bar[stage], m0, k0);
              tma_load_2d(a_smem + stage * Cfg::A_BYTES + Cfg::B_CHUNK_BYTES, &tmap_a, &full_bar[stage], m0 + 64, k0);
            } else {
              tma_load_2d(a_smem + stage * Cfg::A_BYTES, &tmap_a, &full_bar[stage], k0, m0);
            }
            uint8_t* bdst = b_smem + stage * Cfg::B_BYTES;
            if (p.b_kmajor) {
              // B stored N x K: one box of BN rows (n) x 64 k, K-major like A.
              tma_load_2d(bdst, &tmap_b, &full_bar[stage], k0, n0);
            } else {
#pragma unroll
              for (int j = 0; j < Cfg::BN / 64; ++j)
                tma_load_2d(bdst + j * Cfg::B_CHUNK_BYTES, &tmap_b, &full_bar[stage], n0 + j * 64, k0);
            }
            last_parity[stage] = static_cast<int>(phase);
            if (++stage == Cfg::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        // Every load issued has landed before the CTA may exit (a no-op on
        // the normal path, where the MMA warp consumed them all).
#pragma unroll 1
        for (int s = 0; s < Cfg::STAGES; ++s) {
          if (last_parity[s] >= 0) {
            volatile int no_abort = 0;
            mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 2);
          }
        }
      }
    } else {
      const int ptid = threadIdx.x;  // 0 .. PRODUCER_THREADS - 1
      constexpr int kThreads = Cfg::PRODUCER_WARPS * 32;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const int64_t lda = p.lda, ldb = p.ldb;
      const __half* a_end = p.A + static_cast<int64_t>(p.M - 1) * lda + p.K;
      const __half* b_end = p.B + static_cast<int64_t>(p.K - 1) * ldb + p.N;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(p, t, m_blk, n_blk);
        const int m0 = m_blk * Cfg::BM;
        const int n0 = n_blk * Cfg::BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const bool free_slot = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 3);
          if (!__all_sync(0xffffffffu, free_slot)) {
            ok = false;
            break;
          }
          const int k0 = kb * Cfg::BK;
          // Each producer thread stages 4 chunks of the A tile (128 rows x 8
          // chunks, 8 consecutive threads per row) and 8 of the B tile (64
          // k-rows x 32 chunks, one warp per k-row), in batches whose loads
          // are all in flight before any is used.
          constexpr int kA = (Cfg::BM * 8) / kThreads;
          constexpr int kB = (Cfg::BK * 32) / kThreads;
          constexpr int kBatch = 6;
          static_assert((kA + kB) % kBatch == 0, "batching");
#pragma unroll
          for (int b0 = 0; b0 < kA + kB; b0 += kBatch) {
            EdgeChunk plan[kBatch];
            uint32_t dst_off[kBatch];
            int row_of[kBatch], col_of[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int j = b0 + u;
              if (j < kA) {
                const int c = ptid + j * kThreads;
                const int r = c >> 3, kc = c & 7;
                row_of[u] = m0 + r;
                col_of[u] = k0 + kc * 8;
                dst_off[u] = static_cast<uint32_t>(stage * Cfg::A_BYTES) + sw128_offset(r, kc);
                plan[u] = edge_chunk_plan(p.A, a_end, lda, row_of[u], p.M, col_of[u], p.K);
              } else {
                const int c = ptid + (j - kA) * kThreads;
                const int kr = c >> 5, nc = c & 31;
                row_of[u] = k0 + kr;
                col_of[u] = n0 + nc * 8;
                dst_off[u] = static_cast<uint32_t>(stage * Cfg::B_BYTES + (nc >> 3) * Cfg::B_CHUNK_BYTES) +
                             sw128_offset(kr, nc & 7);
                plan[u] = edge_chunk_plan(p.B, b_end, ldb, row_of[u], p.K, col_of[u], p.N);
              }
            }
            uint4 lo[kBatch], hi[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              lo[u] = make_uint4(0u, 0u, 0u, 0u);
              hi[u] = lo[u];
              ld_nc_v4_pred(lo[u], plan[u].src, plan[u].fast);
              ld_nc_v4_pred(hi[u], plan[u].src + 1, plan[u].fast);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int j = b0 + u;
              uint4 v;
              if (plan[u].fast) {
                v = edge_realign(lo[u], hi[u], plan[u].shift);
              } else if (j < kA) {
                v = load_chunk_pred(p.A, lda, row_of[u], p.M, col_of[u], p.K);
              } else {
                v = load_chunk_pred(p.B, ldb, row_of[u], p.K, col_of[u], p.N);
              }
              *reinterpret_cast<uint4*>((j < kA ? a_smem : b_smem) + dst_off[u]) = v;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&full_bar[stage]);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------------
    // MMA issuer: one thread drives the tensor core.
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc_f16_f32(Cfg::BM, Cfg::BN, p.a_mnmajor != 0, p.b_kmajor == 0);
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&acc_empty_bar[acc], acc_phase ^ 1u, abort_flag, p.wait_budget_ns, 4)) break;
        tcgen05_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * Cfg::BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 5)) {
            ok = false;
            break;
          }
          tcgen05_fence_after_sync();
          const uint32_t a_addr = smem_u32(a_smem + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(b_smem + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < Cfg::BK / 16; ++k) {
            // A as M x K: advance 16 elements (32 bytes) inside the swizzled
            // row.  A as K x M: MN-major, two 64-row panels 8 KiB apart.
            const uint64_t adesc = p.a_mnmajor ? make_sw128_desc(a_addr + k * 2048, Cfg::B_CHUNK_BYTES, 1024)
                                               : make_sw128_desc(a_addr + k * 32, 16, 1024);
            // B as K x N: advance 16 k-rows (2048 bytes); 64-column panels 8 KiB
            // apart.  B as N x K: K-major like A.
            const uint64_t bdesc = p.b_kmajor ? make_sw128_desc(b_addr + k * 32, 16, 1024)
                                              : make_sw128_desc(b_addr + k * 2048, Cfg::B_CHUNK_BYTES, 1024);
            umma_f16_ss(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);  // frees the stage when these MMAs finish
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full_bar[acc]);  // accumulator ready for the epilogue
      }
      // All MMAs issued by this thread are complete before TMEM is released.
      umma_commit(mma_done_bar);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 6);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------
    // Epilogue: TMEM -> registers -> ReLU -> fp16 -> C.
    // ------------------------------------------------------------------
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      int m_blk, n_blk;
      tile_coords(p, t, m_blk, n_blk);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      // The TMEM loads below are warp-collective: leave only as a whole warp.
      const bool ready = mbar_wait(&acc_full_bar[acc], acc_phase, abort_flag, p.wait_budget_ns, 7);
      if (!__all_sync(0xffffffffu, ready)) break;
      tcgen05_fence_after_sync();
      const int row = m_blk * Cfg::BM + quad * 32 + lane;
      const bool row_ok = row < p.M;
      __half* crow = p.C + static_cast<int64_t>(row) * p.ldc;
#pragma unroll 1
      for (int c = 0; c < Cfg::BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * Cfg::BN + c * 32, r);
        tmem_ld_wait();
        const int col0 = n_blk * Cfg::BN + c * 32;
        if (col0 < p.N) {
          float b0[16], b1[16];
          load_bias16(p.bias, col0, p.N, b0);
          load_bias16(p.bias, col0 + 16, p.N, b1);
          uint32_t h[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) h[e] = relu_pack_f16x2_bias(r[2 * e], r[2 * e + 1], b0[2 * e], b0[2 * e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            h[8 + e] = relu_pack_f16x2_bias(r[16 + 2 * e], r[16 + 2 * e + 1], b1[2 * e], b1[2 * e + 1]);
          if (row_ok) store_row_chunk(crow, col0, p.N, h, p.c_aligned != 0, false);
        }
      }
      tcgen05_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty_bar[acc]);
    }
  }

  tcgen05_fence_before_sync();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    tcgen05_fence_after_sync();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace tg
