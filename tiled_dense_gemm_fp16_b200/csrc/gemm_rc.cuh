// gemm_rc.cuh -- C = ReLU(A . B) when TMA cannot describe A (or B) as they
// are: row strides that are not a multiple of 16 bytes, or bases that are not
// 16-byte aligned.  No scratch memory: every operand is read in place.
//
// The tile model is the quick-start kernel's ("TileLang" wiki page,
// "Programming model": a ceildiv grid of output tiles, A and B tiles staged
// in shared memory through a pipelined K loop, a cleared fp32 accumulator,
// tile MMAs, max(acc, 0), fp16 output).  What changes is how the tiles are
// staged when the rows are misaligned.
//
// Residue classes of A's rows.  With A's row stride lda (elements), the rows
// r and r + 8 start 16*lda bytes apart, a multiple of 16.  So the rows of one
// class {r : r mod 8 = s} form a matrix with a 16-byte row stride whose rows
// all start e_s elements (0..7) past a 16-byte boundary.  One tensor map per
// class (base rounded down to 16 bytes, inner extent K + e_s) then loads a
// class's rows with 128-byte swizzle straight into the MMA's K-major layout,
// each row shifted by the same e_s elements: map column x holds A[r][x - e_s].
// Every output tile takes its rows (128, or 256 in split mode) from one
// class, and the k-block kb
// loads map columns [64 kb, 64 kb + 64), that is A[r][64 kb - e_s + j].  The
// shift is undone on the other operand: the B tile of the same k-block holds
// the k-rows 64 kb - e_s + j, which is a row offset of B, and TMA takes any
// row offset (negative rows read as zero).  The first k-block's A columns
// with k < 0 (the previous row's tail, or bytes just before A) are cleared in
// shared memory before its MMAs; columns k >= K read as zero.  Output row
// 8 q + s of C is row q of class s (lda a multiple of 8: one class).
//
// B as it is, when TMA can describe it: 64-column boxes with 128-byte
// swizzle at row offset 64 kb - e_s (the MN-major operand).  Otherwise eight
// realigning warps read B's k-rows in place: one coalesced 16-byte load per
// lane and row, the neighbouring block from the next lane by a shuffle, a
// funnel shift by the row's offset (the same across the warp), and a store
// into the swizzled operand tile that keeps each shared-memory phase free of
// bank conflicts.  The next k-block's rows are loaded into registers while
// this one's are shifted.
//
// C is written with aligned 16-byte stores: each epilogue thread owns one row
// of the tile and shifts its values into the 16-byte blocks of that row
// (RowWriter); only the partial blocks at the two ends of a row's piece are
// written element by element.
//
// Shapes with few tiles (one narrow column of tiles, N <= 240 say) split K
// over a cluster of CTAs, one tile per CTA; when a class spans more than one
// 128-row tile, a tile takes 2 x 128 of its rows (two accumulators sharing
// each B stage).  After a cluster barrier each CTA pushes its fp32 partial
// rows from TMEM into the shared memory of the rank that owns them, and each
// owner sums its rows over the cluster's partials in rank order: the small-M
// path's reduction turned on its side.  Every wait is bounded.
#pragma once

#include <cuda_fp16.h>

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace tg {

constexpr int kRcClasses = 8;

// Tensor maps of one call: A per residue class of rows, and B as a whole
// (direct mode only).
struct RcMaps {
  CUtensorMap a[kRcClasses];
  CUtensorMap b;
};

struct RcParams {
  __half* C;
  const __half* B;         // realigning mode: B read in place by the realigning warps
  const __half* bias;      // optional fp16[N] added before ReLU; nullptr = none
  int64_t ldb;             // row stride of B (elements)
  int64_t ldc;             // row stride of C (elements)
  int M, N, K;
  int a_classes;           // 8, or 1 when A's row stride is a multiple of 8 elements
  int a_shift[kRcClasses]; // e_s: elements between the class map's column 0 and A[r][0]
  int rows_in_class[kRcClasses];
  int tile_start[kRcClasses + 1];  // first tile of each class; [a_classes] = m_tiles
  int m_tiles, n_tiles, num_tiles, group_m;
  int bn;                  // tile width: 256, or N rounded up to 16 when N <= 240
  int panels;              // 64-column panels of the B tile: ceil(bn / 64)
  int ring_stages;
  int msub;                // 128-row sub-tiles per tile: 1, or 2 in split mode (one tile per CTA,
                           // two accumulators sharing each B stage)
  int ring_stage_bytes;    // msub x 16 KiB of A + panels x 8 KiB of B
  int splits;              // CTAs per cluster along K (split mode)
  uint32_t idesc;
  uint64_t wait_budget_ns;
};

template <bool REALIGN_B>
struct RcCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;   // 16 KiB
  static constexpr int PANEL_BYTES = BK * 64 * 2;  // 8 KiB: 64 k-rows x 64 columns
  static constexpr int MMA_WARP = 1;
  static constexpr int EPI_WARP0 = 2;
  static constexpr int EPI_WARPS = 4;
  static constexpr int REAL_WARP0 = EPI_WARP0 + EPI_WARPS;
  static constexpr int REAL_WARPS = REALIGN_B ? 8 : 0;  // realigning warps (B read in place)
  static constexpr int THREADS = (REAL_WARP0 + REAL_WARPS) * 32;
  static constexpr int MAX_RING = 8;
  static constexpr int BAR_BYTES = 512;
};

// Writes one piece of a row of C, columns [c0, c0 + count), from values that
// arrive 32 at a time as 16 packed fp16 pairs in column order (the first
// chunk starting at c0).  The row piece starts g elements (0..7) past a
// 16-byte boundary; block b covers the elements [8 b - g, 8 b - g + 8) of the
// piece.  Blocks wholly inside the piece leave as one 16-byte store; the
// partial blocks at either end are written element by element, so nothing
// outside the piece is touched.
struct RowWriter {
  unsigned short* blk0;  // 16-byte aligned: element 0 of block 0
  int lo, hi;            // element indices (from blk0) inside the piece: [g, g + count)
  uint32_t g;
  int next;              // next block to write
  uint4 carry;           // the previous chunk's last 8 values
};

__device__ __forceinline__ void rw_init(RowWriter& w, __half* piece, int count) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(piece);
  w.g = static_cast<uint32_t>((a >> 1) & 7u);
  w.blk0 = reinterpret_cast<unsigned short*>(a - 2u * w.g);
  w.lo = static_cast<int>(w.g);
  w.hi = static_cast<int>(w.g) + count;
  w.next = 0;
  w.carry = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void rw_emit(RowWriter& w, const uint4& v) {
  const int s = 8 * w.next;
  ++w.next;
  if (s >= w.hi || s + 8 <= w.lo) return;
  if (s >= w.lo && s + 8 <= w.hi) {
    __stcs(reinterpret_cast<int4*>(w.blk0 + s), *reinterpret_cast<const int4*>(&v));
    return;
  }
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int idx = s + e;
    if (idx >= w.lo && idx < w.hi) w.blk0[idx] = static_cast<unsigned short>(words[e >> 1] >> ((e & 1) * 16));
  }
}

__device__ __forceinline__ void rw_push(RowWriter& w, const uint32_t (&h)[16]) {
  const uint4 q0 = make_uint4(h[0], h[1], h[2], h[3]);
  const uint4 q1 = make_uint4(h[4], h[5], h[6], h[7]);
  const uint4 q2 = make_uint4(h[8], h[9], h[10], h[11]);
  const uint4 q3 = make_uint4(h[12], h[13], h[14], h[15]);
  if (w.g == 0) {
    rw_emit(w, q0);
    rw_emit(w, q1);
    rw_emit(w, q2);
    rw_emit(w, q3);
    return;
  }
  // Block b starts (8 - g) elements into the pair (previous 8 values, next 8).
  const uint32_t sh = 16u - 2u * w.g;
  rw_emit(w, edge_realign(w.carry, q0, sh));
  rw_emit(w, edge_realign(q0, q1, sh));
  rw_emit(w, edge_realign(q1, q2, sh));
  rw_emit(w, edge_realign(q2, q3, sh));
  w.carry = q3;
}

// As rw_push for 16 values (8 packed pairs).
__device__ __forceinline__ void rw_push8(RowWriter& w, const uint32_t (&h)[8]) {
  const uint4 q0 = make_uint4(h[0], h[1], h[2], h[3]);
  const uint4 q1 = make_uint4(h[4], h[5], h[6], h[7]);
  if (w.g == 0) {
    rw_emit(w, q0);
    rw_emit(w, q1);
    return;
  }
  const uint32_t sh = 16u - 2u * w.g;
  rw_emit(w, edge_realign(w.carry, q0, sh));
  rw_emit(w, edge_realign(q0, q1, sh));
  w.carry = q1;
}

// The block holding the piece's last g values (nothing when g == 0).
__device__ __forceinline__ void rw_finish(RowWriter& w) {
  if (w.g != 0) rw_emit(w, edge_realign(w.carry, make_uint4(0u, 0u, 0u, 0u), 16u - 2u * w.g));
}

__device__ __forceinline__ void st_shared_u4_pred(uint32_t addr, const uint4& v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "@p st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n\t}" ::"r"(addr),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

// 16-byte store to a shared::cluster address (this CTA's or a peer's).
__device__ __forceinline__ void st_shared_cluster_u4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint4& v) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
}

__device__ __forceinline__ void st_shared_u4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Realigning step for 8 k-rows whose pieces start WO words plus bits / 16
// elements past their first aligned block: lane l holds block l of each row
// (lane 31 also block 32, in ext), takes block l + 1 from lane l + 1, and
// stores output chunk l at dst + 1024 m (row 8 m of the panel layout).
template <int WO, int R>
__device__ __forceinline__ void rc_shift_rows(const uint4 (&cur)[R], const uint4 (&ext)[R], uint32_t bits, uint32_t dst,
                                              bool stores, bool last_lane) {
#pragma unroll
  for (int m = 0; m < R; ++m) {
    uint32_t w[8] = {cur[m].x, cur[m].y, cur[m].z, cur[m].w, 0u, 0u, 0u, 0u};
    const uint32_t e[4] = {ext[m].x, ext[m].y, ext[m].z, ext[m].w};
#pragma unroll
    for (int i = 0; i <= WO; ++i) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, w[i], 1);
      w[4 + i] = last_lane ? e[i] : v;
    }
    const uint4 out = make_uint4(__funnelshift_r(w[WO], w[WO + 1], bits), __funnelshift_r(w[WO + 1], w[WO + 2], bits),
                                 __funnelshift_r(w[WO + 2], w[WO + 3], bits), __funnelshift_r(w[WO + 3], w[WO + 4], bits));
    st_shared_u4_pred(dst + 1024u * m, out, stores);
  }
}

// One output tile: class s, rows q0 .. q0 + 127 of the class, columns
// n0 .. n0 + bn - 1, and this CTA's k-blocks [kb_lo, kb_hi) of the class's
// ceil((K + e) / 64).
struct RcTile {
  int s, q0, n0, e, kb_lo, kb_hi;
};

__device__ __forceinline__ RcTile rc_tile(const RcParams& p, int t, int rank, int splits) {
  const int group_tiles = p.group_m * p.n_tiles;
  const int g = t / group_tiles;
  const int first = g * p.group_m;
  const int gm = min(p.m_tiles - first, p.group_m);
  const int local = t - g * group_tiles;
  const int mt = first + local % gm;
  RcTile r;
  r.n0 = (local / gm) * p.bn;
  int s = 0;
#pragma unroll
  for (int c = 1; c < kRcClasses; ++c)
    if (c < p.a_classes && p.tile_start[c] <= mt) s = c;
  r.s = s;
  r.q0 = (mt - p.tile_start[s]) * 128 * p.msub;
  r.e = p.a_shift[s];
  const int kb_total = (p.K + r.e + 63) / 64;
  r.kb_lo = static_cast<int>((static_cast<int64_t>(kb_total) * rank) / splits);
  r.kb_hi = static_cast<int>((static_cast<int64_t>(kb_total) * (rank + 1)) / splits);
  return r;
}

// B_DEEP (realigning mode, tiles narrower than 256 columns): the realigning
// warps keep two k-blocks of B in flight instead of one.
template <bool REALIGN_B, bool SPLIT, bool B_DEEP = false>
__global__ void __launch_bounds__(RcCfg<REALIGN_B>::THREADS, 1)
    gemm_relu_rc_kernel(const __grid_constant__ RcMaps maps, const RcParams p) {
  using Cfg = RcCfg<REALIGN_B>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.ring_stages * p.ring_stage_bytes);
  uint64_t* full_bar = bars;                       // [ring] TMA bytes landed
  uint64_t* empty_bar = bars + Cfg::MAX_RING;      // [ring] MMAs done with the slot
  uint64_t* bfull_bar = bars + 2 * Cfg::MAX_RING;  // [ring] realigned B written (realigning mode)
  uint64_t* acc_full = bars + 3 * Cfg::MAX_RING;   // [2]
  uint64_t* acc_empty = acc_full + 2;              // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = SPLIT ? static_cast<int>(cluster_ctarank()) : 0;
  const int splits = SPLIT ? p.splits : 1;
  const int t_first = SPLIT ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
  const int t_step = SPLIT ? p.num_tiles : static_cast<int>(gridDim.x);
  constexpr uint32_t kTmemCols = 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring_stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&bfull_bar[s], Cfg::REAL_WARPS > 0 ? Cfg::REAL_WARPS : 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], Cfg::EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(tmem_slot, kTmemCols);
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
    // Producer: A's class boxes into the ring, and B's boxes too in direct
    // mode (otherwise the realigning warps bring B).
    // ------------------------------------------------------------------
    if (lane == 0) {
      int r = 0;
      uint32_t rph = 0;
      int last_full[Cfg::MAX_RING];
      for (int i = 0; i < Cfg::MAX_RING; ++i) last_full[i] = -1;
      bool ok = true;
      for (int t = t_first; t < p.num_tiles && ok; t += t_step) {
        const RcTile T = rc_tile(p, t, rank, splits);
        for (int kb = T.kb_lo; kb < T.kb_hi; ++kb) {
          if (!mbar_wait(&empty_bar[r], rph ^ 1u, abort_flag, p.wait_budget_ns, 0x61)) {
            ok = false;
            break;
          }
          uint8_t* slot = ring + r * p.ring_stage_bytes;
          const int k_lo = kb * 64 - T.e;  // B's first k-row of this block
          const int a_bytes = p.msub * Cfg::A_BYTES;
          mbar_arrive_expect_tx(&full_bar[r], REALIGN_B ? a_bytes : a_bytes + p.panels * Cfg::PANEL_BYTES);
          tma_load_2d(slot, &maps.a[T.s], &full_bar[r], kb * 64, T.q0);
          if (!REALIGN_B) {
            for (int c = 0; c < p.panels; ++c)
              tma_load_2d(slot + a_bytes + c * Cfg::PANEL_BYTES, &maps.b, &full_bar[r], T.n0 + 64 * c, k_lo);
          }
          last_full[r] = static_cast<int>(rph);
          if (++r == p.ring_stages) {
            r = 0;
            rph ^= 1u;
          }
        }
      }
      // Every load issued has landed before the CTA may exit.
      volatile int no_abort = 0;
      for (int i = 0; i < p.ring_stages; ++i)
        if (last_full[i] >= 0)
          mbar_wait(&full_bar[i], static_cast<uint32_t>(last_full[i]), &no_abort, p.wait_budget_ns, 0x64);
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------------
    // MMA issuer (lane 0), with the whole warp clearing the first k-block's
    // A columns that lie before k = 0.
    // ------------------------------------------------------------------
    int r = 0, local = 0;
    uint32_t rph = 0;
    bool ok = true;
    for (int t = t_first; t < p.num_tiles && ok; t += t_step, ++local) {
      const RcTile T = rc_tile(p, t, rank, splits);
      const int acc = SPLIT ? 0 : (local & 1);
      const uint32_t acc_phase = SPLIT ? 0u : static_cast<uint32_t>((local >> 1) & 1);
      if (!SPLIT) {
        const bool free_acc = mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.wait_budget_ns, 0x65);
        if (!__all_sync(0xffffffffu, free_acc)) break;
      }
      tcgen05_fence_after_sync();
      const uint32_t d_tmem = tmem_base + acc * 256;
      for (int kb = T.kb_lo; kb < T.kb_hi; ++kb) {
        bool landed = mbar_wait(&full_bar[r], rph, abort_flag, p.wait_budget_ns, 0x66);
        if (REALIGN_B) landed = landed && mbar_wait(&bfull_bar[r], rph, abort_flag, p.wait_budget_ns, 0x6C);
        if (!__all_sync(0xffffffffu, landed)) {
          ok = false;
          break;
        }
        tcgen05_fence_after_sync();
        uint8_t* slot = ring + r * p.ring_stage_bytes;
        if (kb == 0 && T.e > 0) {
          // Columns j < e of k-block 0 are k < 0: clear them (chunk 0 of
          // each swizzled 128-byte row sits at (row & 7) * 16).
          const uint32_t keep_from = static_cast<uint32_t>(T.e);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int row = lane + 32 * i;
            if (i < 4 * p.msub) {
              const uint32_t addr = smem_u32(slot) + row * 128 + ((row & 7) << 4);
              uint4 v;
              ld_shared_v4(addr, v);
              uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (static_cast<uint32_t>(e) < keep_from) w[e >> 1] &= (e & 1) ? 0x0000ffffu : 0xffff0000u;
              st_shared_u4(addr, make_uint4(w[0], w[1], w[2], w[3]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(slot);
          const uint32_t b_addr = a_addr + p.msub * Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = make_sw128_desc(b_addr + k * 2048, Cfg::PANEL_BYTES, 1024);
            for (int u = 0; u < p.msub; ++u) {
              const uint64_t adesc = make_sw128_desc(a_addr + u * Cfg::A_BYTES + k * 32, 16, 1024);
              umma_f16_ss(d_tmem + u * 256, adesc, bdesc, p.idesc, (kb != T.kb_lo || k != 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty_bar[r]);
        }
        __syncwarp();
        if (++r == p.ring_stages) {
          r = 0;
          rph ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0 && T.kb_hi > T.kb_lo) umma_commit(&acc_full[acc]);
      __syncwarp();
    }
    if (lane == 0) {
      umma_commit(mma_done);
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, p.wait_budget_ns, 0x67);
    }
    __syncwarp();
  } else if (warp < Cfg::REAL_WARP0) {
    // ------------------------------------------------------------------
    // Epilogue: TMEM -> registers -> (bias) ReLU -> fp16 -> C rows, or, in
    // split mode, the fp32 partial into shared memory.
    // ------------------------------------------------------------------
    const int quad = warp & 3;
    const int i = quad * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    if (!SPLIT) {
      int local = 0;
      for (int t = t_first; t < p.num_tiles; t += t_step, ++local) {
        const RcTile T = rc_tile(p, t, rank, splits);
        const int acc = local & 1;
        const uint32_t acc_phase = static_cast<uint32_t>((local >> 1) & 1);
        const bool ready = mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.wait_budget_ns, 0x68);
        if (!__all_sync(0xffffffffu, ready)) break;
        tcgen05_fence_after_sync();
        const int qrow = T.q0 + i;
        const bool valid = qrow < p.rows_in_class[T.s];
        const int64_t row = static_cast<int64_t>(qrow) * p.a_classes + T.s;
        const int ncols = min(p.bn, p.N - T.n0);
        RowWriter w;
        if (valid) rw_init(w, p.C + row * p.ldc + T.n0, ncols);
        for (int c = 0; c * 32 < ncols; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + acc * 256 + c * 32, v);
          tmem_ld_wait();
          const int col0 = T.n0 + c * 32;
          float b0[16], b1[16];
          load_bias16(p.bias, col0, p.N, b0);
          load_bias16(p.bias, col0 + 16, p.N, b1);
          uint32_t h[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) h[e] = relu_pack_f16x2_bias(v[2 * e], v[2 * e + 1], b0[2 * e], b0[2 * e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            h[8 + e] = relu_pack_f16x2_bias(v[16 + 2 * e], v[17 + 2 * e], b1[2 * e], b1[2 * e + 1]);
          if (valid) rw_push(w, h);
        }
        if (valid) rw_finish(w);
        tcgen05_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
    } else {
      // The partial stays in TMEM until every CTA of the cluster is done
      // with its ring (below).  A failed wait has set the abort flag.
      const RcTile T = rc_tile(p, t_first, rank, splits);
      if (T.kb_hi > T.kb_lo) mbar_wait(&acc_full[0], 0, abort_flag, p.wait_budget_ns, 0x69);
      __syncwarp();
      tcgen05_fence_before_sync();
    }
  } else if (REALIGN_B) {
    // ------------------------------------------------------------------
    // Realigning warps: B's k-rows straight from global memory into the
    // swizzled MN-major operand tile, no staging buffer.  Warp w owns the
    // k-rows j = 8 m + w of a block.  For one row, lane l loads the 16-byte
    // aligned block l of the row piece (one coalesced load per row; lane 31
    // also loads block 32), takes block l + 1 from lane l + 1 by a shuffle,
    // shifts the pair by the piece's offset f and stores output chunk l to
    // panel l / 8, position (l mod 8) xor (j mod 8): the 8 lanes of a
    // shared-memory phase hit 8 different bank groups.  Rows 8 apart start
    // 16 ldb bytes apart, so a warp's eight rows share f for the whole tile:
    // one uniform branch per k-block picks the word offset and the rows'
    // steps interleave.  The next k-block's rows are loaded into registers
    // while this block's are shifted.  Blocks that start past a row's end are
    // not loaded; a block that ends past it reads at most 14 bytes beyond, in
    // the same 16-byte block (never another page), and those values reach
    // only output columns that are not stored.  Rows outside [0, K) are
    // written as zeros.
    // ------------------------------------------------------------------
    static_assert(!REALIGN_B || Cfg::REAL_WARPS == 8, "k-rows j = 8 m + warp: row j mod 8 is the warp's");
    constexpr int kRows = 8;
    const int rw = warp - Cfg::REAL_WARP0;
    const uintptr_t bbytes = reinterpret_cast<uintptr_t>(p.B);
    const uintptr_t n_bytes = 2u * static_cast<uintptr_t>(p.N);
    const uintptr_t stride = 16u * static_cast<uintptr_t>(p.ldb);  // 8 k-rows, in bytes
    const int chunks = p.bn >> 3;  // 16-byte chunks per operand row, <= 32
    // Chunk `lane` of row j = 8 m + rw sits in panel lane / 8 at row j,
    // position (lane mod 8) xor (j mod 8), and j mod 8 = rw.
    const uint32_t dst_off = static_cast<uint32_t>((lane >> 3) * Cfg::PANEL_BYTES + rw * 128 +
                                                   (((lane & 7) ^ (rw & 7)) << 4));
    const bool stores = lane < chunks;
    if constexpr (B_DEEP) {
      // Two k-blocks in flight: two register sets of 8 rows.  Tiles are
      // narrower than 256 columns (at most 31 chunks per row), so no lane
      // needs a 33rd block and the registers that hold it in the one-block
      // loop below hold the second set here.
      uint4 rows[2][kRows];
      uint32_t f_row[2] = {};  // the rows' offset past their first aligned block
      // The k-blocks this CTA walks, in the order every role walks them: `ld`
      // is the next one to load, `pr` the next one to realign.
      struct Walk {
        int t, kb;
        RcTile T;
        bool valid;
      };
      Walk ld{t_first, 0, RcTile{}, false};
      for (; ld.t < p.num_tiles; ld.t += t_step) {
        ld.T = rc_tile(p, ld.t, rank, splits);
        if (ld.T.kb_hi > ld.T.kb_lo) {
          ld.kb = ld.T.kb_lo;
          ld.valid = true;
          break;
        }
      }
      auto advance = [&](Walk& w) {
        ++w.kb;
        while (w.kb >= w.T.kb_hi) {
          w.t += t_step;
          if (w.t >= p.num_tiles) {
            w.valid = false;
            return;
          }
          w.T = rc_tile(p, w.t, rank, splits);
          w.kb = w.T.kb_lo;
        }
      };
      Walk pr = ld;
      // Rows k0 + 8 m: their pieces start at the same offset f past a 16-byte
      // boundary (8 rows are 16 ldb bytes apart), so one address and one
      // bounds test serve all eight.
      auto load_rows = [&](uint4 (&cur)[kRows], uint32_t& f) {
        const int k0 = ld.kb * 64 - ld.T.e + rw;
        const uintptr_t row0 = bbytes + 2u * static_cast<uintptr_t>(static_cast<int64_t>(k0) * p.ldb);
        const uintptr_t start = row0 + 2u * static_cast<uintptr_t>(ld.T.n0);
        const uintptr_t a0 = start & ~uintptr_t(15);
        const uintptr_t blk = a0 + 16u * static_cast<uintptr_t>(lane);
        const bool lane_ok = lane <= chunks && blk < row0 + n_bytes;
        f = static_cast<uint32_t>((start >> 1) & 7u);
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
          const bool in = static_cast<unsigned>(k0 + 8 * m) < static_cast<unsigned>(p.K);
          cur[m] = make_uint4(0u, 0u, 0u, 0u);
          ld_nc_v4_pred(cur[m], reinterpret_cast<const void*>(blk + m * stride), in && lane_ok);
        }
        advance(ld);
      };
      if (ld.valid) load_rows(rows[0], f_row[0]);
      if (ld.valid) load_rows(rows[1], f_row[1]);
      int r = 0;
      uint32_t rph = 0;
      bool ok = true;
      // Realign k-block `pr` from one register set, then refill that set with
      // the next k-block still to load.  Lane 31's output chunk is never
      // stored (chunks <= 31), so its shuffle partner may be any value: the
      // set itself stands in for the 33rd block.
      auto step = [&](uint4 (&cur)[kRows], uint32_t& f) {
        if (!mbar_wait(&empty_bar[r], rph ^ 1u, abort_flag, p.wait_budget_ns, 0x6B)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          return;
        }
        // Rows outside [0, K) were loaded as zeros and shift to zeros.
        const uint32_t dst = smem_u32(ring + r * p.ring_stage_bytes) + p.msub * Cfg::A_BYTES + dst_off;
        const uint32_t bits = (f & 1u) * 16u;
        switch (f >> 1) {
          case 0: rc_shift_rows<0>(cur, cur, bits, dst, stores, false); break;
          case 1: rc_shift_rows<1>(cur, cur, bits, dst, stores, false); break;
          case 2: rc_shift_rows<2>(cur, cur, bits, dst, stores, false); break;
          default: rc_shift_rows<3>(cur, cur, bits, dst, stores, false); break;
        }
        if (ld.valid) load_rows(cur, f);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull_bar[r]);
        if (++r == p.ring_stages) {
          r = 0;
          rph ^= 1u;
        }
        advance(pr);
      };
      while (pr.valid && ok) {
        step(rows[0], f_row[0]);
        if (pr.valid && ok) step(rows[1], f_row[1]);
      }
    } else {
      const bool extra = lane == 31 && chunks == 32;  // block 32 of the piece
      uint4 cur[kRows], ext[kRows];
      uint32_t f_cur = 0, f_next = 0;  // the rows' offset past their first aligned block
      // The k-blocks this CTA walks, in the order every role walks them.
      int t = t_first, kb = 0;
      RcTile T{};
      bool valid = false;
      for (; t < p.num_tiles; t += t_step) {
        T = rc_tile(p, t, rank, splits);
        if (T.kb_hi > T.kb_lo) {
          kb = T.kb_lo;
          valid = true;
          break;
        }
      }
      // Rows k0 + 8 m: their pieces start at the same offset f past a 16-byte
      // boundary (8 rows are 16 ldb bytes apart), so one address and one
      // bounds test serve all eight.
      auto load_rows = [&](const RcTile& U, int kbu) {
        const int k0 = kbu * 64 - U.e + rw;
        const uintptr_t row0 = bbytes + 2u * static_cast<uintptr_t>(static_cast<int64_t>(k0) * p.ldb);
        const uintptr_t start = row0 + 2u * static_cast<uintptr_t>(U.n0);
        const uintptr_t a0 = start & ~uintptr_t(15);
        const uintptr_t blk = a0 + 16u * static_cast<uintptr_t>(lane);
        const bool lane_ok = lane <= chunks && blk < row0 + n_bytes;
        const bool ext_ok = extra && a0 + 512u < row0 + n_bytes;
        f_next = static_cast<uint32_t>((start >> 1) & 7u);
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
          const bool in = static_cast<unsigned>(k0 + 8 * m) < static_cast<unsigned>(p.K);
          cur[m] = make_uint4(0u, 0u, 0u, 0u);
          ext[m] = make_uint4(0u, 0u, 0u, 0u);
          ld_nc_v4_pred(cur[m], reinterpret_cast<const void*>(blk + m * stride), in && lane_ok);
          ld_nc_v4_pred(ext[m], reinterpret_cast<const void*>(a0 + 512u + m * stride), in && ext_ok);
        }
      };
      if (valid) load_rows(T, kb);
      int r = 0;
      uint32_t rph = 0;
      while (valid) {
        // The next k-block in the walk.
        int t2 = t, kb2 = kb + 1;
        RcTile T2 = T;
        bool valid2 = true;
        while (kb2 >= T2.kb_hi) {
          t2 += t_step;
          if (t2 >= p.num_tiles) {
            valid2 = false;
            break;
          }
          T2 = rc_tile(p, t2, rank, splits);
          kb2 = T2.kb_lo;
        }
        f_cur = f_next;
        const bool got = mbar_wait(&empty_bar[r], rph ^ 1u, abort_flag, p.wait_budget_ns, 0x6B);
        if (!__all_sync(0xffffffffu, got)) break;
        // Rows outside [0, K) were loaded as zeros and shift to zeros.
        const uint32_t dst = smem_u32(ring + r * p.ring_stage_bytes) + p.msub * Cfg::A_BYTES + dst_off;
        const uint32_t bits = (f_cur & 1u) * 16u;
        switch (f_cur >> 1) {
          case 0: rc_shift_rows<0>(cur, ext, bits, dst, stores, lane == 31); break;
          case 1: rc_shift_rows<1>(cur, ext, bits, dst, stores, lane == 31); break;
          case 2: rc_shift_rows<2>(cur, ext, bits, dst, stores, lane == 31); break;
          default: rc_shift_rows<3>(cur, ext, bits, dst, stores, lane == 31); break;
        }
        if (valid2) load_rows(T2, kb2);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull_bar[r]);
        if (++r == p.ring_stages) {
          r = 0;
          rph ^= 1u;
        }
        t = t2;
        kb = kb2;
        T = T2;
        valid = valid2;
      }
    }
  }

  if (SPLIT) {
    // The tile has R = 128 msub rows; rank q owns rows [R q / S, R (q + 1) / S).
    // Once every CTA of the cluster is done with its ring, each epilogue
    // thread pushes its row of the fp32 partial into the owner's shared
    // memory, slot `rank` (remote stores, nothing waits on a round trip).  A
    // slot is laid out by 16-byte column chunk, then row (chunk c4 of slot
    // row il at (c4 rpo + il) x 16 bytes), so a warp's 32 rows store one
    // contiguous 512-byte block.  After a second cluster barrier each owner
    // sums its rows over the slots in rank order, from its own shared
    // memory, and writes them to C.
    const RcTile T = rc_tile(p, t_first, rank, splits);
    const int R = 128 * p.msub;
    const int rpo = (R + splits - 1) / splits;  // slot rows
    const uint32_t slot_bytes = static_cast<uint32_t>(rpo * p.bn * 4);
    const uint32_t part = smem_u32(ring);
    tcgen05_fence_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp >= Cfg::EPI_WARP0 && warp < Cfg::EPI_WARP0 + Cfg::EPI_WARPS && !*abort_flag) {
      tcgen05_fence_after_sync();
      const int quad = warp & 3;
      const int i = quad * 32 + lane;  // row of the tile = TMEM lane
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      const bool has_k = T.kb_hi > T.kb_lo;
      for (int u = 0; u < p.msub; ++u) {
        const int row = u * 128 + i;  // sub-tile u sits in TMEM columns [256 u, 256 u + bn)
        int q = (row * splits) / R;
        if ((R * (q + 1)) / splits <= row) ++q;
        const int il = row - (R * q) / splits;
        const uint32_t dst = mapa_shared(part + rank * slot_bytes + static_cast<uint32_t>(il * 16), static_cast<uint32_t>(q));
        for (int c = 0; c * 16 < p.bn; ++c) {
          uint32_t v[16];
          if (has_k) {
            tmem_ld_32x32b_x16(lane_base + u * 256 + c * 16, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;  // empty K share: the partial is zero
          }
#pragma unroll
          for (int e = 0; e < 4; ++e)
            st_shared_cluster_u4(dst + static_cast<uint32_t>((4 * c + e) * rpo * 16),
                                 make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]));
        }
      }
    }
    cluster_sync();
    if (!*abort_flag) {
      const int r_lo = (R * rank) / splits, r_hi = (R * (rank + 1)) / splits;
      const int nrows = r_hi - r_lo;
      const int ncols = min(p.bn, p.N - T.n0);
      const int segs = (ncols + 63) / 64;
      for (int it = threadIdx.x; it < nrows * segs; it += Cfg::THREADS) {
        const int il = it % nrows;
        const int seg = it / nrows;
        const int qrow = T.q0 + r_lo + il;
        if (qrow >= p.rows_in_class[T.s]) continue;
        const int64_t row = static_cast<int64_t>(qrow) * p.a_classes + T.s;
        const int c0 = 64 * seg, c1 = min(c0 + 64, ncols);
        RowWriter w;
        rw_init(w, p.C + row * p.ldc + T.n0 + c0, c1 - c0);
        for (int cc = c0; cc < c1; cc += 16) {
          float acc[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
          for (int qr = 0; qr < splits; ++qr) {
            const uint32_t off = part + qr * slot_bytes + static_cast<uint32_t>(((cc >> 2) * rpo + il) * 16);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 x;
              ld_shared_v4(off + static_cast<uint32_t>(v4 * rpo * 16), x);
              acc[4 * v4] += __uint_as_float(x.x);
              acc[4 * v4 + 1] += __uint_as_float(x.y);
              acc[4 * v4 + 2] += __uint_as_float(x.z);
              acc[4 * v4 + 3] += __uint_as_float(x.w);
            }
          }
          float b0[16];
          load_bias16(p.bias, T.n0 + cc, p.N, b0);
          uint32_t h[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            h[e] = relu_pack_f16x2_bias(__float_as_uint(acc[2 * e]), __float_as_uint(acc[2 * e + 1]), b0[2 * e],
                                        b0[2 * e + 1]);
          rw_push8(w, h);
        }
        rw_finish(w);
      }
    }
  }

  tcgen05_fence_before_sync();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    tcgen05_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace tg
