// gemm_mx.cuh -- block-scaled grouped GEMMs (MXFP8 and NVF4) on sm_100a
// tensor cores.
//
// The Blackwell MXFP8 grouped GEMM with block scaling and a transposed B
// ("Key Technical Milestones", zhichai.net TileLang topic page), with the
// number formats of the OCP Microscaling (MX) definitions:
//   C[r, j] = bf16( [relu]( sum_k a(r,k) sa(r, k/32) * b_g(j,k) sb_g(j, k/32) ) )
// for the rows r of group g.  A holds the groups' rows stacked, each group
// starting on a multiple of 128 rows; B holds one N x K weight per group
// (rows of length K: the transposed layout); all fp8 operands are K-major.
//
// Per CTA (persistent, one per SM): 128 x 256 output tiles, k-stages of 128
// fp8 elements (one 128-byte swizzled row), 4 stages.  Roles:
//   warp 0      TMA producer: A box 128 x 128 B, B box 256 x 128 B, plus the
//               stage's scale factors (512 B for A's 128 rows, 2 x 512 B for
//               B's 256 rows) with untiled bulk copies;
//   warp 1      TMEM owner and MMA issuer: per stage, four K = 32 MMAs of
//               kind::mxf8f6f4 with block_scale, each reading one scale byte;
//   warps 2-5   scale stagers, one per TMEM lane quarter: per stage they read
//               the scale atoms from shared memory and write them into that
//               stage's TMEM scale buffer with tcgen05.st, every quarter
//               holding the same 32 lines (the layout the MMA reads);
//   warps 6-13  epilogue: two warps per TMEM lane quarter, 128 columns each.
// Staging the scales with tcgen05.st keeps them off the tensor pipe, where
// tcgen05.cp copies would run in order with the MMAs.
// Scale factors are stored in the 128 x 4 blocked layout that the tensor
// core reads (512-byte atoms: 32 lines of 16 bytes, line l holding rows
// l, l+32, l+64, l+96 with four consecutive k-blocks each), so a stage's
// scales are a contiguous 512 bytes per 128 rows.  The accumulator is single-
// buffered (256 of 512 TMEM columns; the scale factors use one small buffer
// per pipeline stage in the rest): the
// epilogue drains it into registers, frees it, then stores, so the next
// tile's MMAs overlap the stores.
//
// The NVF4 variant (the NVF4 block-scaled MMA path of the tilelang-ai project
// page, "Three backends under one language dialect", read as NVIDIA's NVFP4)
// runs the same pipeline with kind::mxf4nvf4: E2M1 elements packed two per
// byte, so a 128-byte k-stage holds 256 elements; one UE4M3 scale per 16
// elements, so each K = 64 MMA reads a whole 4-byte scale word per row and a
// stage carries four 512-byte atoms per 128 rows; an fp32 alpha multiplies
// the accumulator in the epilogue.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace tg {

constexpr int kMxMaxGroups = 256;

enum { kKindMxf8 = 0, kKindNvf4 = 1 };

struct MxParams {
  const uint8_t* SFA;  // blocked scales of A's stacked rows
  const uint8_t* SFB;  // blocked scales of B's rows, groups padded to 128 rows
  __nv_bfloat16* C;    // stacked rows x N
  int N, K;
  int k_stages;        // k-stages of 128 bytes per row
  int k_mmas;          // MMAs along K: K / 32 (MXFP8) or K / 64 (NVF4)
  int atoms_k;         // 512-byte scale atoms per 128 rows along K
  float alpha;         // multiplies the accumulator (1 for MXFP8)
  int n_tiles, m_tiles, num_tiles, group_m;
  int groups;
  int n_atoms;         // ceil(N / 128): 128-row scale atoms per group of B
  int relu;
  uint32_t idesc;      // formats, shape and scale type; the sf bytes are or-ed in per MMA
  uint64_t wait_budget_ns;
  int tile_start[kMxMaxGroups + 1];  // first stacked 128-row tile of each group; [groups] = m_tiles
  int m_size[kMxMaxGroups];          // rows of each group
};

template <int KIND>
struct MxCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 256;
  static constexpr int BK = 128;  // bytes of a row per k-stage: 128 fp8 or 256 fp4 elements
  static constexpr int STAGES = 4;
  static constexpr int ATOMS = KIND == kKindNvf4 ? 4 : 1;  // scale atoms per 128 rows per stage
  static constexpr int MMA_WARP = 1;
  static constexpr int SF_WARP0 = 2;
  static constexpr int SF_WARPS = 4;
  static constexpr int EPI_WARP0 = SF_WARP0 + SF_WARPS;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
  static constexpr int A_BYTES = BM * BK;   // 16 KiB
  static constexpr int B_BYTES = BN * BK;   // 32 KiB
  static constexpr int SFA_BYTES = 512 * ATOMS;
  static constexpr int SFB_BYTES = 1024 * ATOMS;
  static constexpr int TMEM_COLS = 512;
  // Scale factors in TMEM, one buffer per pipeline stage so that a stage's
  // copies do not overwrite scales that earlier MMAs may still be reading:
  // per stage 4 columns of A scales and 8 of B scales per atom.
  static constexpr int SF_COL0 = 256;
  static constexpr int SF_STAGE_COLS = 12 * ATOMS <= 16 ? 16 : 12 * ATOMS;
  static constexpr int SFB_OFF = 4 * ATOMS;
  static constexpr int BAR_BYTES = 256;  // 3 x STAGES + 3 barriers, the TMEM slot and the abort flag
  static constexpr int SMEM_BYTES = 1024 + STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + BAR_BYTES;
  static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);  // 128 columns per epilogue warp
  static_assert(SF_COL0 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "scale buffers exceed the TMEM allocation");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA exceeded");
};

__device__ __forceinline__ void mx_tile_coords(const MxParams& p, int t, int& m_blk, int& n_blk) {
  const int group_tiles = p.group_m * p.n_tiles;
  const int g = t / group_tiles;
  const int first_m = g * p.group_m;
  const int gm = min(p.m_tiles - first_m, p.group_m);
  const int local = t - g * group_tiles;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

// Group that owns stacked tile row m_blk: the last g with tile_start[g] <= m_blk.
__device__ __forceinline__ int mx_group_of(const MxParams& p, int m_blk) {
  int lo = 0, hi = p.groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.tile_start[mid] <= m_blk)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float x0, float x1, bool relu) {
  if (relu) {
    x0 = x0 > 0.0f ? x0 : 0.0f;
    x1 = x1 > 0.0f ? x1 : 0.0f;
  }
  const __nv_bfloat162 v = __floats2bfloat162_rn(x0, x1);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int KIND>
__global__ void __launch_bounds__(MxCfg<KIND>::THREADS, 1)
    gemm_blockscaled_grouped_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                    const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ MxParams p) {
  using Cfg = MxCfg<KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = a_smem + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* sfa_smem = b_smem + Cfg::STAGES * Cfg::B_BYTES;
  uint8_t* sfb_smem = sfa_smem + Cfg::STAGES * Cfg::SFA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sfb_smem + Cfg::STAGES * Cfg::SFB_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + Cfg::STAGES;
  uint64_t* sf_full_bar = bars + 2 * Cfg::STAGES;
  uint64_t* acc_full_bar = bars + 3 * Cfg::STAGES;
  uint64_t* acc_empty_bar = acc_full_bar + 1;
  uint64_t* mma_done_bar = acc_empty_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_full_bar[s], Cfg::SF_WARPS);
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(acc_empty_bar, Cfg::EPI_WARPS);
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    if (p.k_stages > 0) {  // with K = 0 the tensor maps are not encoded
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
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------
    // Producer
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[Cfg::STAGES];
#pragma unroll
      for (int s = 0; s < Cfg::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      const uint64_t pol_b = l2_policy_evict_last();
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int m_blk, n_blk;
        mx_tile_coords(p, t, m_blk, n_blk);
        const int g = mx_group_of(p, m_blk);
        const int n0 = n_blk * Cfg::BN;
        const int b_row0 = g * p.N + n0;
        const int band_b = g * p.n_atoms + n0 / 128;  // first 128-row scale band of this B tile
        const bool second_b = n0 / 128 + 1 < p.n_atoms;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 41)) {
            ok = false;
            break;
          }
          const int atom0 = ks * Cfg::ATOMS;
          const int natoms = min(Cfg::ATOMS, p.atoms_k - atom0);
          const uint32_t sf_bytes = static_cast<uint32_t>(natoms) * 512u * (second_b ? 3u : 2u);
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::A_BYTES + Cfg::B_BYTES + sf_bytes);
          const int k0 = ks * Cfg::BK;
          tma_load_2d(a_smem + stage * Cfg::A_BYTES, &tmap_a, &full_bar[stage], k0, m_blk * Cfg::BM);
          tma_load_2d_hint(b_smem + stage * Cfg::B_BYTES, &tmap_b, &full_bar[stage], k0, b_row0, pol_b);
          // A stage's atoms of one 128-row band are contiguous in the blocked layout.
          const uint32_t span = static_cast<uint32_t>(natoms) * 512u;
          bulk_load_g2s(sfa_smem + stage * Cfg::SFA_BYTES,
                        p.SFA + (static_cast<int64_t>(m_blk) * p.atoms_k + atom0) * 512, span, &full_bar[stage]);
          bulk_load_g2s(sfb_smem + stage * Cfg::SFB_BYTES,
                        p.SFB + (static_cast<int64_t>(band_b) * p.atoms_k + atom0) * 512, span, &full_bar[stage]);
          if (second_b)
            bulk_load_g2s(sfb_smem + stage * Cfg::SFB_BYTES + Cfg::SFB_BYTES / 2,
                          p.SFB + (static_cast<int64_t>(band_b + 1) * p.atoms_k + atom0) * 512, span,
                          &full_bar[stage]);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every copy issued has landed before the CTA may exit.
#pragma unroll 1
      for (int s = 0; s < Cfg::STAGES; ++s) {
        if (last_parity[s] >= 0) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 42);
        }
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------------
    // Scale-factor copies and MMAs
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        if (!mbar_wait(acc_empty_bar, (local & 1) ^ 1u, abort_flag, p.wait_budget_ns, 43)) break;
        tcgen05_fence_after_sync();
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 44)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&sf_full_bar[stage], phase, abort_flag, p.wait_budget_ns, 47)) {
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
              // Each MMA consumes 32 bytes of every row (32 fp8 or 64 fp4 elements).
              const uint64_t adesc = make_sw128_desc(a_addr + k * 32, 16, 1024);
              const uint64_t bdesc = make_sw128_desc(b_addr + k * 32, 16, 1024);
              const uint32_t accumulate = (ks | k) != 0 ? 1u : 0u;
              if (KIND == kKindMxf8) {
                // One scale per 32 elements: MMA k reads byte k of the stage's atom.
                const uint32_t sel = static_cast<uint32_t>(k);
                umma_mxf8_ss(tmem_base, adesc, bdesc, p.idesc | (sel << 29) | (sel << 4), sfa_tmem | (sel << 30),
                             sfb_tmem | (sel << 30), accumulate);
              } else {
                // Four scales per 64 elements: MMA k reads the whole words of atom k.
                umma_nvf4_ss(tmem_base, adesc, bdesc, p.idesc, sfa_tmem + 4 * k, sfb_tmem + 8 * k, accumulate);
              }
            }
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(acc_full_bar);
      }
      umma_commit(mma_done_bar);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 45);
    }
    __syncwarp();
  } else if (warp < Cfg::EPI_WARP0) {
    // ------------------------------------------------------------------
    // Scale stagers: shared memory -> this warp's TMEM lane quarter
    // ------------------------------------------------------------------
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      // The second 128-row band of B's scales is not loaded for a tile that
      // ends within the first band: its columns are never stored, and zero
      // scales stand in for the stale shared memory.
      int m_blk, n_blk;
      mx_tile_coords(p, t, m_blk, n_blk);
      const bool second_b = n_blk * 2 + 1 < p.n_atoms;
      for (int ks = 0; ks < p.k_stages; ++ks) {
        const bool ready = mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 48);
        if (!__all_sync(0xffffffffu, ready)) {
          ok = false;
          break;
        }
        const int natoms = min(Cfg::ATOMS, p.atoms_k - ks * Cfg::ATOMS);
        const uint32_t sfa_tmem = tmem_base + lane_base + Cfg::SF_COL0 + stage * Cfg::SF_STAGE_COLS;
        const uint32_t sfb_tmem = sfa_tmem + Cfg::SFB_OFF;
        const uint4* sa = reinterpret_cast<const uint4*>(sfa_smem + stage * Cfg::SFA_BYTES) + lane;
        const uint4* sb = reinterpret_cast<const uint4*>(sfb_smem + stage * Cfg::SFB_BYTES) + lane;
#pragma unroll
        for (int a = 0; a < Cfg::ATOMS; ++a) {
          if (a < natoms) {
            // Line `lane` of each 512-byte atom: 16 bytes = 4 TMEM columns.
            const uint4 va = sa[a * 32];
            const uint4 vb0 = sb[a * 32];
            const uint4 vb1 = second_b ? sb[Cfg::SFB_BYTES / 32 + a * 32] : make_uint4(0, 0, 0, 0);
            tmem_st_32x32b_x4(sfa_tmem + 4 * a, va);
            tmem_st_32x32b_x4(sfb_tmem + 8 * a, vb0);
            tmem_st_32x32b_x4(sfb_tmem + 8 * a + 4, vb1);
          }
        }
        tmem_st_wait();
        tcgen05_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full_bar[stage]);
        if (++stage == Cfg::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Epilogue: TMEM -> registers (ReLU, bf16) -> free the accumulator -> C
    // ------------------------------------------------------------------
    const int e = warp - Cfg::EPI_WARP0;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
    const int half = e >> 2;                 // column half of the tile
    const bool relu = p.relu != 0;
    const bool have_k = p.k_mmas > 0;
    const float alpha = p.alpha;
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      int m_blk, n_blk;
      mx_tile_coords(p, t, m_blk, n_blk);
      const int g = mx_group_of(p, m_blk);
      const bool ready = mbar_wait(acc_full_bar, local & 1, abort_flag, p.wait_budget_ns, 46);
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
      if (lane == 0) mbar_arrive(acc_empty_bar);
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
  if (warp == Cfg::MMA_WARP) {
    tcgen05_fence_after_sync();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace tg
