// gemm_tc_pair.cuh -- the persistent tcgen05 GEMM + ReLU kernel on CTA pairs
// (cta_group::2): 256 x BN output tiles (BN = 256 or 512), each computed by
// the two SMs of a 2-CTA cluster.
//
// Same tile model as gemm_tc.cuh (the matmul_relu quick-start kernel: tiles
// staged through a pipelined K loop, cleared fp32 accumulator, tile MMAs,
// max(acc, 0), fp16 output), with the MMA spread over an SM pair:
//   * CTA r of the pair (r = 0, 1) loads rows [128 r, 128 r + 128) of the
//     A tile and, of every 256-column slab of the B tile, the columns
//     [128 r, 128 r + 128) into its own shared memory (TMA, 128-byte swizzle,
//     no multicast): 32 KiB per stage and 6 stages for BN = 256, 48 KiB per
//     stage and 4 stages for BN = 512;
//   * both CTAs' loads count their bytes on the even CTA's "full" barrier;
//     the even CTA's single MMA thread issues BN / 256 pair MMAs of
//     256 x 256 x 16 per k-step that read both CTAs' shared memory and write
//     both CTAs' TMEM (rows [128 r, 128 r + 128) of the tile land in CTA r);
//     BN = 256 double-buffers the accumulator (2 x 256 columns), BN = 512
//     uses all 512 columns for one accumulator;
//   * the MMA commits multicast to both CTAs' "empty" barriers (each CTA then
//     refills its own stage) and, per tile, to both CTAs' "accumulator full"
//     barriers; the eight epilogue warps of the pair release the accumulator
//     on the even CTA's "accumulator empty" barrier;
//   * per SM, each 64-deep k-block moves 32 KiB from L2 for 128 x 256 x 64
//     MACs at BN = 256 (two thirds of what the single-CTA 128 x 256 tile
//     needs) and 48 KiB for 128 x 512 x 64 MACs at BN = 512 (one half);
//   * BN = 512 drains the accumulator 32 columns per TMEM round trip into
//     registers as packed fp16, frees it, then stages C through shared
//     memory in 32 x 32 boxes that TMA writes out (rows of C 16-byte
//     aligned), so each warp's stores leave as whole 64-byte row pieces
//     instead of one 16-byte piece per row and store instruction.
// Every wait is bounded; a cluster barrier brackets the kernel so that no
// CTA exits while its peer may still touch its shared memory or barriers.
#pragma once

#include <cuda_fp16.h>

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace tg {

template <int STAGES_, int BN_>
struct TcPairCfg {
  static constexpr int BM = 128;        // rows per CTA (the pair tile is 256)
  static constexpr int PAIR_M = 256;
  static constexpr int BN = BN_;        // columns per pair tile: 256 or 512
  static constexpr int SLABS = BN / 256;          // pair MMAs per k-step
  static constexpr int BN_HALF = BN / 2;          // columns of B each CTA loads
  static constexpr int BK = 64;
  static constexpr int STAGES = STAGES_;
  static constexpr int MMA_WARP = 1;
  static constexpr int EPI_WARP0 = 2;
  // Epilogue warps: 4 per 256-column slab, each taking the slab's columns
  // for one TMEM lane quadrant (with the single accumulator of BN = 512 a
  // thread holds its 256 values in registers and releases TMEM before it
  // stores).
  static constexpr int EPI_WARPS = 4 * SLABS;
  static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);  // accumulator columns per epilogue warp
  static constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
  static constexpr int A_BYTES = BM * BK * 2;        // 16 KiB
  static constexpr int B_BYTES = BK * BN_HALF * 2;   // 16 or 32 KiB
  static constexpr int B_CHUNK_BYTES = BK * 64 * 2;  // 8 KiB panel of 64 columns
  static constexpr int B_SLAB_BYTES = 2 * B_CHUNK_BYTES;  // this CTA's 128 columns of one slab
  static constexpr int NUM_ACC = (BN == 256) ? 2 : 1;
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = 256;
  // C staging of the epilogue: per epilogue warp two 2 KiB buffers, each one
  // 32-row x 32-column fp16 box of C with the 64-byte swizzle, written by the
  // warp and stored by TMA while the warp fills the other.
  static constexpr int C_BOX_COLS = 32;
  static constexpr int C_BUF_BYTES = 32 * C_BOX_COLS * 2;
  static constexpr int C_STAGE_BYTES = EPI_WARPS * 2 * C_BUF_BYTES;
  static constexpr int SMEM_BYTES = 1024 + STAGES * (A_BYTES + B_BYTES) + C_STAGE_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA");
  static_assert(BN == 256 || BN == 512, "pair tile width");
  static_assert(NUM_ACC * BN <= TMEM_COLS, "TMEM columns");
};

// One 16-byte shared-memory store.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// tma_store_2d with an L2 cache policy for the written lines.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* smem_src, int x, int y,
                                                  uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

template <int STAGES, int BN>
__global__ void __launch_bounds__(TcPairCfg<STAGES, BN>::THREADS, 1)
    gemm_relu_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                             const __grid_constant__ CUtensorMap tmap_c, const TcParams p) {
  using Cfg = TcPairCfg<STAGES, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* c_stage = smem + Cfg::STAGES * (Cfg::A_BYTES + Cfg::B_BYTES);  // 1 KiB aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(c_stage + Cfg::C_STAGE_BYTES);
  uint64_t* full_bar = bars;                         // used in the even CTA
  uint64_t* empty_bar = bars + Cfg::STAGES;          // per CTA
  uint64_t* acc_full_bar = bars + 2 * Cfg::STAGES;   // per CTA
  uint64_t* acc_empty_bar = acc_full_bar + Cfg::NUM_ACC;  // used in the even CTA
  uint64_t* mma_done_bar = acc_empty_bar + Cfg::NUM_ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = even CTA (issues the MMAs), 1 = odd CTA
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < Cfg::NUM_ACC; ++b) {
      mbar_init(&acc_full_bar[b], 1);
      mbar_init(&acc_empty_bar[b], 2 * Cfg::EPI_WARPS);
    }
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if (Cfg::C_STAGE_BYTES > 0 && p.c_aligned) tma_prefetch_desc(&tmap_c);
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
  // Everything above touched only shared memory, TMEM and kernel parameters;
  // global memory is used only after the previous grid on the stream is done.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------
    // Producer (both CTAs): this CTA's half of the A and B tiles.
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[Cfg::STAGES];
#pragma unroll
      for (int s = 0; s < Cfg::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      const uint64_t pol_a = (p.l2_hints & 1) ? l2_policy_evict_last() : l2_policy_evict_normal();
      const uint64_t pol_b = (p.l2_hints & 2)   ? l2_policy_evict_last()
                             : (p.l2_hints & 4) ? l2_policy_evict_first()
                                                : l2_policy_evict_normal();
      for (int t = cluster_id; t < p.num_tiles && ok; t += num_clusters) {
        int m_blk, n_blk;
        tile_coords(p, t, m_blk, n_blk);
        const int m0 = m_blk * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM;
        // This CTA's 128 columns of slab j start at n0 + 256 j + 128 r.
        const int nb = n_blk * Cfg::BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 0x41)) {
            ok = false;
            break;
          }
          const uint32_t full_even = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * (Cfg::A_BYTES + Cfg::B_BYTES));
          const int k0 = kb * Cfg::BK;
          uint8_t* bdst = b_smem + stage * Cfg::B_BYTES;
          if (p.a_mnmajor) {
            // A stored K x M: this CTA's 128 m-rows as two 64 m x 64 k boxes.
            tma_load_2d_pair_hint(a_smem + stage * Cfg::A_BYTES, &tmap_a, full_even, m0, k0, pol_a);
            tma_load_2d_pair_hint(a_smem + stage * Cfg::A_BYTES + Cfg::B_CHUNK_BYTES, &tmap_a, full_even, m0 + 64,
                                  k0, pol_a);
          } else {
            tma_load_2d_pair_hint(a_smem + stage * Cfg::A_BYTES, &tmap_a, full_even, k0, m0, pol_a);
          }
#pragma unroll
          for (int j = 0; j < Cfg::SLABS; ++j) {
            if (p.b_kmajor) {
              // B stored N x K: this CTA's 128 n-rows x 64 k of slab j, K-major.
              tma_load_2d_pair_hint(bdst + j * Cfg::B_SLAB_BYTES, &tmap_b, full_even, k0, nb + 256 * j, pol_b);
            } else {
              tma_load_2d_pair_hint(bdst + j * Cfg::B_SLAB_BYTES, &tmap_b, full_even, nb + 256 * j, k0, pol_b);
              tma_load_2d_pair_hint(bdst + j * Cfg::B_SLAB_BYTES + Cfg::B_CHUNK_BYTES, &tmap_b, full_even,
                                    nb + 256 * j + 64, k0, pol_b);
            }
          }
          if (p.prefetch_kb > 0 && kb + p.prefetch_kb < p.k_blocks) {
            // Warm L2 with the boxes a few k-blocks ahead, so the ring's
            // loads find them there instead of waiting on HBM.
            const int kp = (kb + p.prefetch_kb) * Cfg::BK;
            if (p.a_mnmajor) {
              tma_prefetch_l2_2d(&tmap_a, m0, kp);
              tma_prefetch_l2_2d(&tmap_a, m0 + 64, kp);
            } else {
              tma_prefetch_l2_2d(&tmap_a, kp, m0);
            }
#pragma unroll
            for (int j = 0; j < Cfg::SLABS; ++j) {
              if (p.b_kmajor) {
                tma_prefetch_l2_2d(&tmap_b, kp, nb + 256 * j);
              } else {
                tma_prefetch_l2_2d(&tmap_b, nb + 256 * j, kp);
                tma_prefetch_l2_2d(&tmap_b, nb + 256 * j + 64, kp);
              }
            }
          }
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The even CTA's full barriers count both CTAs' bytes: once they have
      // completed, every load of the pair has landed.
      if (leader) {
#pragma unroll 1
        for (int s = 0; s < Cfg::STAGES; ++s) {
          if (last_parity[s] >= 0) {
            volatile int no_abort = 0;
            mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 0x42);
          }
        }
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------------
    // MMA issuer (even CTA only).
    // ------------------------------------------------------------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc_f16_f32(Cfg::PAIR_M, 256, p.a_mnmajor != 0, p.b_kmajor == 0);
      for (int t = cluster_id; t < p.num_tiles && ok; t += num_clusters, ++local) {
        const int acc = local % Cfg::NUM_ACC;
        const uint32_t acc_phase = (local / Cfg::NUM_ACC) & 1;
        if (!mbar_wait(&acc_empty_bar[acc], acc_phase ^ 1u, abort_flag, p.wait_budget_ns, 0x43)) break;
        tcgen05_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * Cfg::BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 0x44)) {
            ok = false;
            break;
          }
          tcgen05_fence_after_sync();
          const uint32_t a_addr = smem_u32(a_smem + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(b_smem + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < Cfg::BK / 16; ++k) {
            const uint64_t adesc = p.a_mnmajor ? make_sw128_desc(a_addr + k * 2048, Cfg::B_CHUNK_BYTES, 1024)
                                               : make_sw128_desc(a_addr + k * 32, 16, 1024);
#pragma unroll
            for (int j = 0; j < Cfg::SLABS; ++j) {
              // Slab j: as K x N, this CTA's two 64-column panels, 8 KiB apart;
              // as N x K, 128 K-major rows like A.
              const uint32_t slab_addr = b_addr + j * Cfg::B_SLAB_BYTES;
              const uint64_t bdesc = p.b_kmajor ? make_sw128_desc(slab_addr + k * 32, 16, 1024)
                                                : make_sw128_desc(slab_addr + k * 2048, Cfg::B_CHUNK_BYTES, 1024);
              umma_f16_ss_pair(d_tmem + 256 * j, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair_mc(&empty_bar[stage], 0x3);  // both CTAs may refill this stage
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(&acc_full_bar[acc], 0x3);  // both halves of the accumulator are ready
      }
      umma_commit_pair_mc(mma_done_bar, 0x1);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 0x45);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------
    // Epilogue (both CTAs): this CTA's 128 rows of the 256 x BN tile; warp
    // w reads TMEM lanes 32 (w mod 4) .. + 31, columns
    // [EPI_COLS * ((w - 2) / 4), + EPI_COLS) of the accumulator.
    // ------------------------------------------------------------------
    const int quad = warp & 3;
    const int col_base = ((warp - Cfg::EPI_WARP0) >> 2) * Cfg::EPI_COLS;
    int local = 0;
    for (int t = cluster_id; t < p.num_tiles; t += num_clusters, ++local) {
      int m_blk, n_blk;
      tile_coords(p, t, m_blk, n_blk);
      const int acc = local % Cfg::NUM_ACC;
      const uint32_t acc_phase = (local / Cfg::NUM_ACC) & 1;
      const bool ready = mbar_wait(&acc_full_bar[acc], acc_phase, abort_flag, p.wait_budget_ns, 0x46);
      if (!__all_sync(0xffffffffu, ready)) break;
      tcgen05_fence_after_sync();
      const int row = m_blk * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM + quad * 32 + lane;
      const bool row_ok = row < p.M;
      __half* crow = p.C + static_cast<int64_t>(row) * p.ldc;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * Cfg::BN + col_base;
      if (Cfg::NUM_ACC == 1) {
        // Single accumulator: read this thread's EPI_COLS columns into
        // registers as ReLU'd fp16 pairs, release the accumulator to the MMA
        // warp, and only then store, so the stores overlap the next tile's MMAs.
        uint32_t h[Cfg::EPI_COLS / 2];
#pragma unroll
        for (int c = 0; c < Cfg::EPI_COLS / 32; ++c) {
          uint32_t r[32];  // 32 columns per TMEM round trip
          tmem_ld_32x32b_x32(taddr + c * 32, r);
          tmem_ld_wait();
          if (p.bias != nullptr) {
#pragma unroll
            for (int part = 0; part < 4; ++part) {
              float bv[8];
              load_bias8(p.bias, n_blk * Cfg::BN + col_base + c * 32 + part * 8, p.N, bv);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                h[c * 16 + part * 4 + e] =
                    relu_pack_f16x2_bias(r[part * 8 + 2 * e], r[part * 8 + 2 * e + 1], bv[2 * e], bv[2 * e + 1]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) h[c * 16 + e] = relu_pack_f16x2(r[2 * e], r[2 * e + 1]);
          }
        }
        tcgen05_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty_bar[acc]), 0));
        if (p.c_aligned) {
          // Rows of C start on 16-byte boundaries: stage 32 x 32 boxes (lane
          // = row, 64 bytes each, 16-byte chunks swizzled by bits 1..2 of the
          // row) and let TMA write them; rows and columns past C are clipped
          // by the tensor map.  Each buffer is refilled only once the store
          // issued two boxes earlier has read it.
          const int y0 = m_blk * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM + quad * 32;
          uint8_t* wbuf = c_stage + (warp - Cfg::EPI_WARP0) * 2 * Cfg::C_BUF_BYTES;
          const uint64_t pol = p.store_streaming ? l2_policy_evict_first() : l2_policy_evict_normal();
          if (y0 < p.M) {
#pragma unroll
            for (int c = 0; c < Cfg::EPI_COLS / Cfg::C_BOX_COLS; ++c) {
              const int col0 = n_blk * Cfg::BN + col_base + c * Cfg::C_BOX_COLS;
              if (col0 >= p.N) break;
              uint8_t* buf = wbuf + (c & 1) * Cfg::C_BUF_BYTES;
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              const uint32_t row_addr = smem_u32(buf) + lane * 64;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                st_shared_v4(row_addr + ((q ^ ((lane >> 1) & 3)) << 4), h[c * 16 + 4 * q], h[c * 16 + 4 * q + 1],
                             h[c * 16 + 4 * q + 2], h[c * 16 + 4 * q + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d_hint(&tmap_c, buf, col0, y0, pol);
                bulk_commit_group();
              }
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < Cfg::EPI_COLS / 32; ++c) {
            const int col0 = n_blk * Cfg::BN + col_base + c * 32;
            uint32_t hc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) hc[e] = h[c * 16 + e];
            if (row_ok && col0 < p.N) store_row_chunk(crow, col0, p.N, hc, false, p.store_streaming != 0);
          }
        }
      } else {
        // Double-buffered accumulator: the next tile's MMAs already run in
        // the other buffer; drain 32 columns at a time.  With 16-byte aligned
        // rows of C each 32 x 32 piece goes out through a swizzled staging
        // box and a TMA store, as in the single-accumulator epilogue.
        const int y0 = m_blk * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM + quad * 32;
        uint8_t* wbuf = c_stage + (warp - Cfg::EPI_WARP0) * 2 * Cfg::C_BUF_BYTES;
        const uint64_t pol = p.store_streaming ? l2_policy_evict_first() : l2_policy_evict_normal();
#pragma unroll 1
        for (int c = 0; c < Cfg::EPI_COLS / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + c * 32, r);
          tmem_ld_wait();
          const int col0 = n_blk * Cfg::BN + col_base + c * 32;
          if (p.c_aligned) {
            if (y0 < p.M && col0 < p.N) {
              float b0[16], b1[16];
              load_bias16(p.bias, col0, p.N, b0);
              load_bias16(p.bias, col0 + 16, p.N, b1);
              uint32_t hc[16];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                hc[e] = relu_pack_f16x2_bias(r[2 * e], r[2 * e + 1], b0[2 * e], b0[2 * e + 1]);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                hc[8 + e] = relu_pack_f16x2_bias(r[16 + 2 * e], r[16 + 2 * e + 1], b1[2 * e], b1[2 * e + 1]);
              uint8_t* buf = wbuf + (c & 1) * Cfg::C_BUF_BYTES;
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              const uint32_t row_addr = smem_u32(buf) + lane * 64;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                st_shared_v4(row_addr + ((q ^ ((lane >> 1) & 3)) << 4), hc[4 * q], hc[4 * q + 1], hc[4 * q + 2],
                             hc[4 * q + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d_hint(&tmap_c, buf, col0, y0, pol);
                bulk_commit_group();
              }
            }
          } else if (row_ok && col0 < p.N) {
            float b0[16], b1[16];
            load_bias16(p.bias, col0, p.N, b0);
            load_bias16(p.bias, col0 + 16, p.N, b1);
            uint32_t hc[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) hc[e] = relu_pack_f16x2_bias(r[2 * e], r[2 * e + 1], b0[2 * e], b0[2 * e + 1]);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              hc[8 + e] = relu_pack_f16x2_bias(r[16 + 2 * e], r[16 + 2 * e + 1], b1[2 * e], b1[2 * e + 1]);
            store_row_chunk(crow, col0, p.N, hc, false, p.store_streaming != 0);
          }
        }
        tcgen05_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty_bar[acc]), 0));
      }
    }
  }

  if (warp >= Cfg::EPI_WARP0 && lane == 0) bulk_wait_group<0>();  // C is written
  tcgen05_fence_before_sync();
  __syncthreads();
  cluster_sync();  // the pair is done with each other's shared memory and barriers
  if (warp == Cfg::MMA_WARP) {
    tcgen05_fence_after_sync();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace tg
