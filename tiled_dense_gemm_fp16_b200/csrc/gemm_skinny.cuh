// gemm_skinny.cuh -- small-M path of C = ReLU(A . B): swap-AB split-K on
// tcgen05 with a cluster-wide reduction through distributed shared memory.
//
// For small M the work is bound by streaming B (K x N) from HBM once.  The
// kernel computes the transposed product C^T (N x M) = B^T (N x K) . A^T
// (K x M), so that N fills the 128-row MMA dimension and M (padded to a
// multiple of 16, at most 256) is the MMA's N:
//   * the grid is (S, P): P = ceil(N / 128) panels of 128 columns of C, each
//     handled by a cluster of S CTAs that split the K loop (S <= 8);
//   * each CTA streams its K slice of the B panel (two 64-column TMA boxes per
//     64-deep k-block, 128-byte swizzle, read as an MN-major operand) and of A
//     (one box of M_pad rows, K-major) through an mbarrier ring, and one
//     thread issues 128 x M_pad x 16 UMMAs into a TMEM accumulator;
//   * the four epilogue warps copy the fp32 partial (row n of the panel, all
//     M_pad columns) from TMEM into the CTA's shared memory as [m][n];
//   * after a cluster barrier each CTA sums a share of the panel's outputs
//     over the S partials in rank order 0..S-1 (deterministic), applies ReLU
//     on fp32, rounds to fp16 and stores C; a second cluster barrier keeps
//     every CTA's shared memory alive until its peers have read it.
// Nothing outside A, B and C is touched: no workspace, no atomics.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace tg {

struct SkinnyParams {
  __half* C;
  const __half* bias;     // optional fp16[N] added before ReLU; nullptr = none
  int64_t ldc;            // row stride of C (elements)
  int b_kmajor;           // 1: B stored N x K, so the MMA's A operand is K-major
  int M, N, K;
  int m_pad;              // MMA N: M rounded up to a multiple of 16 (16..256)
  int k_blocks;           // ceil(K / 64)
  int splits;             // S: CTAs per cluster along K
  int stages;
  uint32_t a_stage_bytes; // m_pad * 128
  uint32_t tmem_cols;     // power of two >= max(32, m_pad)
  uint32_t idesc;
  int prefetch_kb;        // > 0: also prefetch into L2 the B boxes this many k-blocks ahead
  int c_aligned;          // 1: rows of C start on 8-byte boundaries (4-value stores)
  uint64_t wait_budget_ns;
};

struct SkinnyCfg {
  static constexpr int BK = 64;
  static constexpr int PANEL = 128;                   // MMA M (columns of C per cluster)
  static constexpr int B_STAGE_BYTES = PANEL * BK * 2; // 16 KiB: two 64 x 64 boxes
  static constexpr int B_BOX_BYTES = 64 * BK * 2;      // 8 KiB
  static constexpr int THREADS = 192;                  // producer, MMA, 4 epilogue warps
  static constexpr int EPI_WARP0 = 2;
  static constexpr int BAR_BYTES = 256;

  static int stage_bytes(int m_pad) { return B_STAGE_BYTES + m_pad * 128; }
  static int smem_bytes(int m_pad, int stages) { return 1024 + stages * stage_bytes(m_pad) + BAR_BYTES; }
};

__global__ void __launch_bounds__(SkinnyCfg::THREADS, 1)
    gemm_relu_skinny_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                            const SkinnyParams p) {
  using Cfg = SkinnyCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* b_smem = smem;                                          // stages x 16 KiB
  uint8_t* a_smem = smem + p.stages * Cfg::B_STAGE_BYTES;          // stages x a_stage_bytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.stages * (Cfg::B_STAGE_BYTES + p.a_stage_bytes));
  uint64_t* full_bar = bars;            // [stages]
  uint64_t* empty_bar = bars + 8;       // [stages], stages <= 8
  uint64_t* acc_full_bar = bars + 16;
  uint64_t* mma_done_bar = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* partial = reinterpret_cast<float*>(smem);                 // [m_pad][128], reuses the ring

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int panel = blockIdx.y;
  const int n0 = panel * Cfg::PANEL;
  // This CTA's k-blocks: [kb_lo, kb_hi).
  const int kb_lo = static_cast<int>((static_cast<int64_t>(p.k_blocks) * rank) / p.splits);
  const int kb_hi = static_cast<int>((static_cast<int64_t>(p.k_blocks) * (rank + 1)) / p.splits);
  const int my_blocks = kb_hi - kb_lo;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
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

  if (warp == 0) {
    // Producer: one thread issues the TMA loads of this CTA's K slice.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) last_parity[s] = -1;
      const uint32_t tx = Cfg::B_STAGE_BYTES + p.a_stage_bytes;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 0x21)) break;
        mbar_arrive_expect_tx(&full_bar[stage], tx);
        const int k0 = kb * Cfg::BK;
        uint8_t* bdst = b_smem + stage * Cfg::B_STAGE_BYTES;
        if (p.b_kmajor) {
          tma_load_2d(bdst, &tmap_b, &full_bar[stage], k0, n0);  // 128 n-rows x 64 k, K-major
        } else {
          tma_load_2d(bdst, &tmap_b, &full_bar[stage], n0, k0);
          tma_load_2d(bdst + Cfg::B_BOX_BYTES, &tmap_b, &full_bar[stage], n0 + 64, k0);
        }
        tma_load_2d(a_smem + stage * p.a_stage_bytes, &tmap_a, &full_bar[stage], k0, 0);
        if (p.prefetch_kb > 0 && kb + p.prefetch_kb < kb_hi) {
          const int kp = (kb + p.prefetch_kb) * Cfg::BK;
          tma_prefetch_l2_2d(&tmap_b, n0, kp);
          tma_prefetch_l2_2d(&tmap_b, n0 + 64, kp);
        }
        last_parity[stage] = static_cast<int>(phase);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < p.stages; ++s) {
        if (last_parity[s] >= 0) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 0x22);
        }
      }
    }
  } else if (warp == 1) {
    // MMA issuer.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < my_blocks; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 0x23)) {
          ok = false;
          break;
        }
        tcgen05_fence_after_sync();
        const uint32_t b_addr = smem_u32(b_smem + stage * Cfg::B_STAGE_BYTES);
        const uint32_t a_addr = smem_u32(a_smem + stage * p.a_stage_bytes);
#pragma unroll
        for (int k = 0; k < Cfg::BK / 16; ++k) {
          // MMA A operand = B^T panel.  B as K x N: MN-major, 64-column boxes
          // 8 KiB apart, 16 k-rows (2 KiB) per step.  B as N x K: K-major.
          const uint64_t adesc = p.b_kmajor ? make_sw128_desc(b_addr + k * 32, 16, 1024)
                                            : make_sw128_desc(b_addr + k * 2048, Cfg::B_BOX_BYTES, 1024);
          // MMA B operand = A^T: K-major rows of A, 32 bytes per 16-deep step.
          const uint64_t bdesc = make_sw128_desc(a_addr + k * 32, 16, 1024);
          umma_f16_ss(tmem_base, adesc, bdesc, p.idesc, (i | k) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && my_blocks > 0) umma_commit(acc_full_bar);
      umma_commit(mma_done_bar);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 0x24);
    }
    __syncwarp();
  } else {
    // Epilogue warps: TMEM partial -> shared memory [m][n] (fp32).
    const int quad = warp & 3;
    const int n_local = quad * 32 + lane;
    bool ready = true;
    if (my_blocks > 0) ready = mbar_wait(acc_full_bar, 0, abort_flag, p.wait_budget_ns, 0x25);
    ready = __all_sync(0xffffffffu, ready);
    if (ready) {
      tcgen05_fence_after_sync();
      for (int c = 0; c < p.m_pad / 16; ++c) {
        uint32_t r[16];
        if (my_blocks > 0) {
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c * 16, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = 0u;  // empty K slice: the partial is zero
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) partial[(c * 16 + e) * Cfg::PANEL + n_local] = __uint_as_float(r[e]);
      }
    }
    tcgen05_fence_before_sync();
  }

  __syncthreads();
  cluster_sync();  // every partial of the cluster is in shared memory

  if (warp >= Cfg::EPI_WARP0 && !*abort_flag) {
    // Reduction: items are (m, 4-column group); consecutive threads take
    // consecutive column groups of one row of C.
    const int e = threadIdx.x - Cfg::EPI_WARP0 * 32;  // 0..127
    const int items = p.M * (Cfg::PANEL / 4);
    const int lo = static_cast<int>((static_cast<int64_t>(items) * rank) / p.splits);
    const int hi = static_cast<int>((static_cast<int64_t>(items) * (rank + 1)) / p.splits);
    const uint32_t part_addr = smem_u32(partial);
    for (int it = lo + e; it < hi; it += 128) {
      const int m = it / (Cfg::PANEL / 4);
      const int j = it - m * (Cfg::PANEL / 4);
      const int n = n0 + 4 * j;
      if (n >= p.N) continue;  // with aligned rows (N % 8 == 0) a group is wholly inside or outside
      const uint32_t off = static_cast<uint32_t>((m * Cfg::PANEL + 4 * j) * 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < p.splits; ++q) {
        const float4 v = ld_shared_cluster_f4(mapa_shared(part_addr + off, static_cast<uint32_t>(q)));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      if (p.bias != nullptr) {
        const unsigned short* b16 = reinterpret_cast<const unsigned short*>(p.bias) + n;
        float bb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) bb[e] = (n + e < p.N) ? __half2float(__ushort_as_half(__ldg(b16 + e))) : 0.0f;
        acc.x += bb[0];
        acc.y += bb[1];
        acc.z += bb[2];
        acc.w += bb[3];
      }
      const __half2 h01 = __floats2half2_rn(acc.x > 0.f ? acc.x : 0.f, acc.y > 0.f ? acc.y : 0.f);
      const __half2 h23 = __floats2half2_rn(acc.z > 0.f ? acc.z : 0.f, acc.w > 0.f ? acc.w : 0.f);
      uint2 packed;
      packed.x = *reinterpret_cast<const uint32_t*>(&h01);
      packed.y = *reinterpret_cast<const uint32_t*>(&h23);
      __half* dst = p.C + static_cast<int64_t>(m) * p.ldc + n;
      if (p.c_aligned) {
        *reinterpret_cast<uint2*>(dst) = packed;
      } else {
        // Unaligned rows of C: 2-byte stores, only of columns inside C.
        unsigned short* d16 = reinterpret_cast<unsigned short*>(dst);
        const uint32_t w[2] = {packed.x, packed.y};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (n + e < p.N) d16[e] = static_cast<unsigned short>(w[e >> 1] >> ((e & 1) * 16));
      }
    }
  }

  cluster_sync();  // peers are done reading this CTA's partial
  if (warp == 1) {
    tcgen05_fence_after_sync();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace tg
