// gemm_mx_pair.cuh -- block-scaled grouped GEMMs (MXFP8 and NVF4) on CTA
// pairs: tcgen05 cta_group::2 MMAs of 256 x 256 per k-step.
//
// Same operation, layouts and roles as gemm_blockscaled_grouped_kernel
// (gemm_mx.cuh); what changes on a pair of SMs (a 2-CTA cluster):
//   * a pair tile is 256 rows of one group x 256 columns.  CTA r loads its
//     own 128 rows of A and rows [128 r, 128 r + 128) of the tile's 256 rows
//     of the (N x K) weight, so each SM stages half of the B tile and the
//     shared-memory traffic per MMA drops by a third;
//   * groups start on multiples of 128 rows, so a group's 128-row tiles are
//     paired in order; with an odd count its last pair tile has a second
//     half beyond the group, computed against the group's weight and never
//     stored;
//   * every CTA stages its own A scales and all 256 columns' B scales into
//     its own TMEM (the pair MMA reads both CTAs' TMEM at the same address);
//     the stager warps of both CTAs and the A/B loads of both CTAs signal the
//     even CTA, whose single thread issues the MMAs and commits to both CTAs'
//     barriers;
//   * each CTA drains its own 128 rows of the accumulator.
#pragma once

#include "gemm_mx.cuh"

namespace tg {

template <int KIND>
struct MxPairCfg {
  static constexpr int BM = 128;       // rows per CTA
  static constexpr int PAIR_M = 256;
  static constexpr int BN = 256;       // columns of the pair tile
  static constexpr int B_ROWS = 128;   // weight rows staged per CTA
  static constexpr int BK = 128;       // bytes of a row per k-stage
  static constexpr int STAGES = KIND == kKindNvf4 ? 5 : 6;
  static constexpr int ATOMS = KIND == kKindNvf4 ? 4 : 1;
  static constexpr int MMA_WARP = 1;
  static constexpr int SF_WARP0 = 2;
  static constexpr int SF_WARPS = 4;
  static constexpr int EPI_WARP0 = SF_WARP0 + SF_WARPS;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
  static constexpr int A_BYTES = BM * BK;      // 16 KiB
  static constexpr int B_BYTES = B_ROWS * BK;  // 16 KiB
  static constexpr int SFA_BYTES = 512 * ATOMS;
  static constexpr int SFB_BYTES = 1024 * ATOMS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 256;
  static constexpr int SF_STAGE_COLS = 12 * ATOMS <= 16 ? 16 : 12 * ATOMS;
  static constexpr int SFB_OFF = 4 * ATOMS;
  static constexpr int BAR_BYTES = 256;  // 4 x STAGES + 3 barriers, the TMEM slot and the abort flag
  static constexpr int SMEM_BYTES = 1024 + STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + BAR_BYTES;
  static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);
  static_assert(SF_COL0 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "scale buffers exceed the TMEM allocation");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA exceeded");
  static_assert((4 * STAGES + 3) * 8 + 8 <= BAR_BYTES, "barrier area");
};

__device__ __forceinline__ void mx_pair_coords(const MxParams& p, int t, int& pm, int& n_blk) {
  const int group_tiles = p.group_m * p.n_tiles;
  const int g = t / group_tiles;
  const int first_m = g * p.group_m;
  const int gm = min(p.pair_tiles - first_m, p.group_m);
  const int local = t - g * group_tiles;
  pm = first_m + local % gm;
  n_blk = local / gm;
}

// Group of pair tile pm and this CTA's stacked 128-row tile in it.
__device__ __forceinline__ int mx_pair_group(const MxParams& p, int pm, uint32_t rank, int& m_blk) {
  int lo = 0, hi = p.groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.pair_start[mid] <= pm)
      lo = mid;
    else
      hi = mid - 1;
  }
  m_blk = p.tile_start[lo] + 2 * (pm - p.pair_start[lo]) + static_cast<int>(rank);
  return lo;
}

template <int KIND>
__global__ void __launch_bounds__(MxPairCfg<KIND>::THREADS, 1)
    gemm_blockscaled_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                                 const __grid_constant__ MxParams p) {
  using Cfg = MxPairCfg<KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = a_smem + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* sfa_smem = b_smem + Cfg::STAGES * Cfg::B_BYTES;
  uint8_t* sfb_smem = sfa_smem + Cfg::STAGES * Cfg::SFA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sfb_smem + Cfg::STAGES * Cfg::SFB_BYTES);
  uint64_t* full_bar = bars;                       // even CTA: both CTAs' A/B bytes
  uint64_t* empty_bar = bars + Cfg::STAGES;        // per CTA
  uint64_t* sf_load_bar = bars + 2 * Cfg::STAGES;  // per CTA: its own scale copies
  uint64_t* sf_full_bar = bars + 3 * Cfg::STAGES;  // even CTA: both CTAs' stager warps
  uint64_t* acc_full_bar = bars + 4 * Cfg::STAGES; // per CTA
  uint64_t* acc_empty_bar = acc_full_bar + 1;      // even CTA: both CTAs' epilogue warps
  uint64_t* mma_done_bar = acc_empty_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_load_bar[s], 1);
      mbar_init(&sf_full_bar[s], 2 * Cfg::SF_WARPS);
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(acc_empty_bar, 2 * Cfg::EPI_WARPS);
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    if (p.k_stages > 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
    }
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_alloc_permit_pair();
  }
  tcgen05_fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tcgen05_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------
    // Producer (both CTAs): this CTA's A rows and weight rows, and its scales
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[Cfg::STAGES];
#pragma unroll
      for (int s = 0; s < Cfg::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      const uint64_t pol_b = l2_policy_evict_last();
      const uint64_t pol_a = l2_policy_evict_normal();
      for (int t = cluster_id; t < p.num_tiles && ok; t += num_clusters) {
        int pm, n_blk, m_blk;
        mx_pair_coords(p, t, pm, n_blk);
        const int g = mx_pair_group(p, pm, rank, m_blk);
        const bool a_rows_exist = m_blk < p.m_tiles;  // a half pair at the very end has no rows
        const int n0 = n_blk * Cfg::BN;
        const int b_row0 = g * p.N + n0 + static_cast<int>(rank) * Cfg::B_ROWS;
        const int band_b = g * p.n_atoms + n0 / 128;
        const bool second_b = n0 / 128 + 1 < p.n_atoms;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 51)) {
            ok = false;
            break;
          }
          const uint32_t full_even = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * (Cfg::A_BYTES + Cfg::B_BYTES));
          const int k0 = ks * Cfg::BK;
          tma_load_2d_pair_hint(a_smem + stage * Cfg::A_BYTES, &tmap_a, full_even, k0, m_blk * Cfg::BM, pol_a);
          tma_load_2d_pair_hint(b_smem + stage * Cfg::B_BYTES, &tmap_b, full_even, k0, b_row0, pol_b);
          const int atom0 = ks * Cfg::ATOMS;
          const int natoms = min(Cfg::ATOMS, p.atoms_k - atom0);
          const uint32_t span = static_cast<uint32_t>(natoms) * 512u;
          mbar_arrive_expect_tx(&sf_load_bar[stage], span * ((a_rows_exist ? 1u : 0u) + (second_b ? 2u : 1u)));
          if (a_rows_exist)
            bulk_load_g2s(sfa_smem + stage * Cfg::SFA_BYTES,
                          p.SFA + (static_cast<int64_t>(m_blk) * p.atoms_k + atom0) * 512, span, &sf_load_bar[stage]);
          bulk_load_g2s(sfb_smem + stage * Cfg::SFB_BYTES,
                        p.SFB + (static_cast<int64_t>(band_b) * p.atoms_k + atom0) * 512, span, &sf_load_bar[stage]);
          if (second_b)
            bulk_load_g2s(sfb_smem + stage * Cfg::SFB_BYTES + Cfg::SFB_BYTES / 2,
                          p.SFB + (static_cast<int64_t>(band_b + 1) * p.atoms_k + atom0) * 512, span,
                          &sf_load_bar[stage]);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every copy issued has landed before the CTA may exit: this CTA's
      // scale copies on its own barriers, both CTAs' A/B loads on the even
      // CTA's (the closing cluster barrier keeps the odd CTA until then).
#pragma unroll 1
      for (int s = 0; s < Cfg::STAGES; ++s) {
        if (last_parity[s] >= 0) {
          volatile int no_abort = 0;
          mbar_wait(&sf_load_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 52);
          if (leader) mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 52);
        }
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------------
    // MMA issuer (even CTA only)
    // ------------------------------------------------------------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = cluster_id; t < p.num_tiles && ok; t += num_clusters, ++local) {
        if (!mbar_wait_cluster(acc_empty_bar, (local & 1) ^ 1u, abort_flag, p.wait_budget_ns, 53)) break;
        tcgen05_fence_after_sync();
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 54) ||
              !mbar_wait_cluster(&sf_full_bar[stage], phase, abort_flag, p.wait_budget_ns, 55)) {
            ok = false;
            break;
          }
          tcgen05_fence_after_sync();
          const uint32_t sfa_tmem = tmem_base + Cfg::SF_COL0 + stage * Cfg::SF_STAGE_COLS;
          const uint32_t sfb_tmem = sfa_tmem + Cfg::SFB_OFF;
          const uint32_t a_addr = smem_u32(a_smem + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(b_smem + stage * Cfg::B_BYTES);
          const int nk = min(4, p.k_mmas - ks * 4);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k < nk) {
              const uint64_t adesc = make_sw128_desc(a_addr + k * 32, 16, 1024);
              const uint64_t bdesc = make_sw128_desc(b_addr + k * 32, 16, 1024);
              const uint32_t accumulate = (ks | k) != 0 ? 1u : 0u;
              if (KIND == kKindMxf8) {
                const uint32_t sel = static_cast<uint32_t>(k);
                umma_mxf8_ss_pair(tmem_base, adesc, bdesc, p.idesc | (sel << 29) | (sel << 4), sfa_tmem | (sel << 30),
                                  sfb_tmem | (sel << 30), accumulate);
              } else {
                umma_nvf4_ss_pair(tmem_base, adesc, bdesc, p.idesc, sfa_tmem + 4 * k, sfb_tmem + 8 * k, accumulate);
              }
            }
          }
          umma_commit_pair_mc(&empty_bar[stage], 0x3);  // both CTAs may refill this stage
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(acc_full_bar, 0x3);
      }
      umma_commit_pair_mc(mma_done_bar, 0x1);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 56);
    }
    __syncwarp();
  } else if (warp < Cfg::EPI_WARP0) {
    // ------------------------------------------------------------------
    // Scale stagers (both CTAs): this CTA's shared memory -> its TMEM quarter
    // ------------------------------------------------------------------
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = cluster_id; t < p.num_tiles && ok; t += num_clusters) {
      // Bands that were not loaded (no A rows past the last group, no second
      // band of B's scales past N) stage zero scales instead of stale memory.
      int pm, n_blk, m_blk;
      mx_pair_coords(p, t, pm, n_blk);
      (void)mx_pair_group(p, pm, rank, m_blk);
      const bool a_rows_exist = m_blk < p.m_tiles;
      const bool second_b = n_blk * 2 + 1 < p.n_atoms;
      for (int ks = 0; ks < p.k_stages; ++ks) {
        const bool ready = mbar_wait(&sf_load_bar[stage], phase, abort_flag, p.wait_budget_ns, 57);
        if (!__all_sync(0xffffffffu, ready)) {
          ok = false;
          break;
        }
        const int natoms = min(Cfg::ATOMS, p.atoms_k - ks * Cfg::ATOMS);
        const uint32_t sfa_tmem = tmem_base + lane_base + Cfg::SF_COL0 + stage * Cfg::SF_STAGE_COLS;
        const uint32_t sfb_tmem = sfa_tmem + Cfg::SFB_OFF;
        const uint4* sa = reinterpret_cast<const uint4*>(sfa_smem + stage * Cfg::SFA_BYTES) + lane;
        const uint4* sb = reinterpret_cast<const uint4*>(sfb_smem + stage * Cfg::SFB_BYTES) + lane;
        const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int a = 0; a < Cfg::ATOMS; ++a) {
          if (a < natoms) {
            const uint4 va = a_rows_exist ? sa[a * 32] : zero;
            const uint4 vb0 = sb[a * 32];
            const uint4 vb1 = second_b ? sb[Cfg::SFB_BYTES / 32 + a * 32] : zero;
            tmem_st_32x32b_x4(sfa_tmem + 4 * a, va);
            tmem_st_32x32b_x4(sfb_tmem + 8 * a, vb0);
            tmem_st_32x32b_x4(sfb_tmem + 8 * a + 4, vb1);
          }
        }
        tmem_st_wait();  // the stores are complete before the signal
        tcgen05_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&sf_full_bar[stage]), 0));
        if (++stage == Cfg::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Epilogue (both CTAs): this CTA's 128 rows of the pair tile
    // ------------------------------------------------------------------
    const int e = warp - Cfg::EPI_WARP0;
    const int quad = warp & 3;
    const int half = e >> 2;
    const bool relu = p.relu != 0;
    const bool have_k = p.k_mmas > 0;
    const float alpha = p.alpha;
    int local = 0;
    for (int t = cluster_id; t < p.num_tiles; t += num_clusters, ++local) {
      int pm, n_blk, m_blk;
      mx_pair_coords(p, t, pm, n_blk);
      const int g = mx_pair_group(p, pm, rank, m_blk);
      const bool ready = mbar_wait(acc_full_bar, local & 1, abort_flag, p.wait_budget_ns, 58);
      if (!__all_sync(0xffffffffu, ready)) break;
      tcgen05_fence_after_sync();
      uint32_t h[Cfg::EPI_COLS / 2];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + half * Cfg::EPI_COLS;
#pragma unroll
      for (int c = 0; c < Cfg::EPI_COLS / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + c * 16, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          h[c * 8 + q] = have_k ? pack_bf16x2(alpha * __uint_as_float(r[2 * q]),
                                              alpha * __uint_as_float(r[2 * q + 1]), relu)
                                : 0u;
      }
      tcgen05_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(acc_empty_bar), 0));
      const int local_row = (m_blk - p.tile_start[g]) * Cfg::BM + quad * 32 + lane;
      if (local_row < p.m_size[g]) {
        const int row = m_blk * Cfg::BM + quad * 32 + lane;
        const int col0 = n_blk * Cfg::BN + half * Cfg::EPI_COLS;
        uint4* dst = reinterpret_cast<uint4*>(p.C + static_cast<int64_t>(row) * p.N + col0);
#pragma unroll
        for (int q = 0; q < Cfg::EPI_COLS / 8; ++q)
          if (col0 + q * 8 < p.N) dst[q] = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
      }
    }
  }

  tcgen05_fence_before_sync();
  __syncthreads();
  cluster_sync();  // the pair is done with each other's shared memory and barriers
  if (warp == Cfg::MMA_WARP) {
    tcgen05_fence_after_sync();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace tg
