// gemm_w4a16.cuh -- 4-bit weight-only GEMM: C = ReLU(A . W^T) with fp16 A
// (M x K), W (N x K) stored as 4-bit codes with one fp16 scale per group of
// K elements, w = fp16((q - 8) * s); fp32 accumulation, fp16 C (M x N).
//
// The dequantize_gemm workload of the TileLang pages ("TileLang" wiki page,
// opening paragraph), read as the common W4A16 scheme.  Two kernels:
//   * dequant_w4_kernel: W -> fp16 (N x K) in HBM, bandwidth-bound; a large-M
//     call dequantizes into the caller's workspace and then runs the fp16
//     tensor-core GEMM with the weight in the N x K layout;
//   * gemm_relu_w4a16_skinny_kernel: for M <= 256, one kernel that streams
//     the packed weight once.  It is the small-M kernel's swap-AB split-K
//     scheme (C^T = W . A^T, the weight's 128-row panel is the MMA's M side,
//     a cluster of S CTAs splits K and reduces through distributed shared
//     memory) with a dequantization stage in front of the MMA:
//       - warp 0 loads, per 64-deep k-block, the panel's packed codes (128
//         rows x 32 bytes), a 16-byte box of each row's scales (8 groups
//         around the k-block) and the activations (m_pad rows x 64) into a
//         deep ring, so no scale load sits on the dequantization's path;
//       - warps 6-13 turn each packed tile into the fp16 tile the MMA reads
//         (128-byte swizzled, K-major) in a small second ring: a nibble is
//         masked into the mantissa of 1024.0 or of 64.0 (where its bits have
//         unit weight), 1032 or 72 is subtracted (exact: q - 8), and the fp16
//         multiply by the group's scale rounds once to nearest even;
//       - warp 1 issues 128 x m_pad x 16 MMAs; warps 2-5 move the fp32
//         partial to shared memory for the cluster reduction.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace tg {

// ---------------------------------------------------------------------------
// Stand-alone dequantization
// ---------------------------------------------------------------------------

struct DequantParams {
  const uint8_t* Wq;  // N x K/2 bytes
  const __half* S;    // N x K/group scales
  __half* W;          // N x K output
  int64_t N, K;
  int group;
  int64_t chunks;     // N * K / 8: 8 codes (4 bytes) -> 8 fp16 (16 bytes) each
};

// Eight 4-bit codes (a 32-bit word, element 2i in the low nibble of byte i)
// as eight fp16 values (q - 8) * s, in the pairs the arithmetic yields:
// v[i] = (e_i, e_{i+4}), low half first.  Masking the word (or the word
// shifted by 8) with 0x000F000F puts elements i and i + 4 in the low mantissa
// bits of 1024.0 (1024 + q, 1032 subtracted exactly); masking with 0x00F000F0
// puts the odd elements in mantissa bits 4..7, which have unit weight in
// 64.0 (64 + q, 72 subtracted exactly).  One mask per pair, one shift per
// word; the multiply by the scale then rounds once to nearest even.
__device__ __forceinline__ void dequant8_pairs(uint32_t w, __half2 s2, uint32_t (&v)[4]) {
  const uint32_t w8 = w >> 8;
  v[0] = (w & 0x000F000Fu) | 0x64006400u;   // 1024 + q
  v[1] = (w & 0x00F000F0u) | 0x54005400u;   // 64 + q
  v[2] = (w8 & 0x000F000Fu) | 0x64006400u;
  v[3] = (w8 & 0x00F000F0u) | 0x54005400u;
  const __half2 even_bias = __floats2half2_rn(1032.0f, 1032.0f), odd_bias = __floats2half2_rn(72.0f, 72.0f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 x = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&v[i]), (i & 1) ? odd_bias : even_bias), s2);
    v[i] = *reinterpret_cast<const uint32_t*>(&x);
  }
}

// The same eight values in element order, packed two per word.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __half2 s2) {
  uint32_t v[4];
  dequant8_pairs(w, s2, v);
  return make_uint4(__byte_perm(v[0], v[1], 0x5410), __byte_perm(v[2], v[3], 0x5410),
                    __byte_perm(v[0], v[1], 0x7632), __byte_perm(v[2], v[3], 0x7632));
}

// Index: the type of the chunk arithmetic, 32-bit below 2^31 chunks (a
// 64-bit division is a long software routine on the GPU).  Four chunks per
// thread and round, their code and scale loads issued before any store, so
// that enough bytes are in flight to cover the memory latency.
template <typename Index>
__device__ __forceinline__ void dequant_w4_body(const DequantParams& p) {
  constexpr int kUnroll = 4;
  const Index per_row = static_cast<Index>(p.K / 8);
  const Index chunks = static_cast<Index>(p.chunks);
  const Index stride = static_cast<Index>(gridDim.x) * blockDim.x;
  const int gshift = __ffs(p.group) - 1;  // the group is a power of two
  const int64_t groups_per_row = p.K >> gshift;
  for (Index base = static_cast<Index>(blockIdx.x) * blockDim.x + threadIdx.x; base < chunks;
       base += stride * kUnroll) {
    uint32_t w[kUnroll];
    __half sc[kUnroll];
    int64_t n[kUnroll], k[kUnroll];
    bool live[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const Index c = base + u * stride;
      live[u] = c < chunks;
      const Index nr = live[u] ? c / per_row : 0;
      n[u] = static_cast<int64_t>(nr);
      k[u] = static_cast<int64_t>(c - nr * per_row) * 8;
      w[u] = 0u;
      sc[u] = __float2half(0.0f);
      if (live[u]) {
        w[u] = __ldg(reinterpret_cast<const uint32_t*>(p.Wq + n[u] * (p.K / 2) + k[u] / 2));
        sc[u] = p.S[n[u] * groups_per_row + (k[u] >> gshift)];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (live[u]) reinterpret_cast<uint4*>(p.W + n[u] * p.K)[k[u] / 8] = dequant8(w[u], __halves2half2(sc[u], sc[u]));
  }
}

__global__ void __launch_bounds__(256) dequant_w4_kernel(const DequantParams p) {
  grid_dependency_wait();
  grid_launch_dependents();
  if (p.chunks < (int64_t(1) << 31))
    dequant_w4_body<uint32_t>(p);
  else
    dequant_w4_body<int64_t>(p);
}

// ---------------------------------------------------------------------------
// Fused small-M kernel
// ---------------------------------------------------------------------------

struct W4Params {
  __half* C;
  const __half* S;        // N x K/group scales
  int M, N, K;
  int group;
  int m_pad;              // MMA N: M rounded up to a multiple of 16 (16..256)
  int k_blocks;           // K / 64
  int splits;             // CTAs per cluster along K
  int stages;             // depth of the packed ring (<= 16)
  uint32_t a_stage_bytes; // m_pad * 128
  uint32_t tmem_cols;
  uint32_t idesc;
  int c_aligned;          // rows of C start on 8-byte boundaries
  int wdq_slots;          // fp16 tiles in flight (<= MAX_WDQ_SLOTS)
  int scale_tma;          // 1: scales arrive with the ring (rows of K/group fp16 are 16-byte multiples)
  uint64_t wait_budget_ns;
};

struct W4Cfg {
  static constexpr int BK = 64;
  static constexpr int PANEL = 128;
  static constexpr int PACKED_BYTES = PANEL * BK / 2;  // 4 KiB of codes per k-block
  static constexpr int WDQ_BYTES = PANEL * BK * 2;     // 16 KiB fp16 tile
  static constexpr int MAX_WDQ_SLOTS = 6;
  static constexpr int SCALE_BYTES = PANEL * 16;        // 128 rows x 8 scales
  static constexpr int EPI_WARP0 = 2;
  static constexpr int DQ_WARP0 = 6;
  static constexpr int DQ_WARPS = 8;
  static constexpr int THREADS = (DQ_WARP0 + DQ_WARPS) * 32;
  static constexpr int MAX_STAGES = 16;
  static constexpr int BAR_BYTES = 512;

  static int ring_stage_bytes(int m_pad) { return PACKED_BYTES + SCALE_BYTES + m_pad * 128; }
  static int smem_bytes(int m_pad, int stages, int wdq_slots) {
    return 1024 + wdq_slots * WDQ_BYTES + stages * ring_stage_bytes(m_pad) + BAR_BYTES;
  }
};

__global__ void __launch_bounds__(W4Cfg::THREADS, 2)
    gemm_relu_w4a16_skinny_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                                  const __grid_constant__ CUtensorMap tmap_s, const W4Params p) {
  using Cfg = W4Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wdq_smem = smem;                                               // wdq_slots x 16 KiB (1024-aligned)
  uint8_t* a_smem = wdq_smem + p.wdq_slots * Cfg::WDQ_BYTES;              // stages x a_stage_bytes (1024-aligned)
  uint8_t* packed_smem = a_smem + p.stages * p.a_stage_bytes;             // stages x 4 KiB
  uint8_t* scale_smem = packed_smem + p.stages * Cfg::PACKED_BYTES;       // stages x 2 KiB
  uint64_t* bars = reinterpret_cast<uint64_t*>(scale_smem + p.stages * Cfg::SCALE_BYTES);
  uint64_t* full_bar = bars;                                // [MAX_STAGES]: codes + activations landed
  uint64_t* empty_bar = bars + Cfg::MAX_STAGES;             // [MAX_STAGES]: the MMAs read the activations
  uint64_t* wdq_full_bar = bars + 2 * Cfg::MAX_STAGES;          // [MAX_WDQ_SLOTS]: fp16 tile written
  uint64_t* wdq_empty_bar = wdq_full_bar + Cfg::MAX_WDQ_SLOTS;  // [MAX_WDQ_SLOTS]: the MMAs read the fp16 tile
  uint64_t* acc_full_bar = wdq_empty_bar + Cfg::MAX_WDQ_SLOTS;
  uint64_t* mma_done_bar = acc_full_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* partial = reinterpret_cast<float*>(smem);          // [m_pad][128], reuses the rings

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int n0 = blockIdx.y * Cfg::PANEL;
  const int kb_lo = static_cast<int>((static_cast<int64_t>(p.k_blocks) * rank) / p.splits);
  const int kb_hi = static_cast<int>((static_cast<int64_t>(p.k_blocks) * (rank + 1)) / p.splits);
  const int my_blocks = kb_hi - kb_lo;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < p.wdq_slots; ++s) {
      mbar_init(&wdq_full_bar[s], Cfg::DQ_WARPS);
      mbar_init(&wdq_empty_bar[s], 1);
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_w);
    if (p.scale_tma) tma_prefetch_desc(&tmap_s);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish_alloc_permit();
  }
  tcgen05_fence_before_sync();
  __syncthreads();
  tcgen05_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // Producer: packed codes of the panel and the activations, per k-block.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[Cfg::MAX_STAGES];
#pragma unroll
      for (int s = 0; s < Cfg::MAX_STAGES; ++s) last_parity[s] = -1;
      const uint32_t tx = Cfg::PACKED_BYTES + p.a_stage_bytes + (p.scale_tma ? Cfg::SCALE_BYTES : 0u);
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_budget_ns, 0x61)) break;
        mbar_arrive_expect_tx(&full_bar[stage], tx);
        tma_load_2d(packed_smem + stage * Cfg::PACKED_BYTES, &tmap_w, &full_bar[stage], kb * (Cfg::BK / 2), n0);
        if (p.scale_tma)  // the 8 groups that start at the k-block's group rounded down to a multiple of 8
          tma_load_2d(scale_smem + stage * Cfg::SCALE_BYTES, &tmap_s, &full_bar[stage],
                      (kb * Cfg::BK / p.group) & ~7, n0);
        tma_load_2d(a_smem + stage * p.a_stage_bytes, &tmap_a, &full_bar[stage], kb * Cfg::BK, 0);
        last_parity[stage] = static_cast<int>(phase);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < p.stages; ++s) {
        if (last_parity[s] >= 0) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], static_cast<uint32_t>(last_parity[s]), &no_abort, p.wait_budget_ns, 0x62);
        }
      }
    }
  } else if (warp == 1) {
    // MMA issuer: dequantized weight (K-major, MMA A) x activations (K-major, MMA B).
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < my_blocks; ++i) {
        const int slot = i % p.wdq_slots;
        const uint32_t slot_phase = static_cast<uint32_t>((i / p.wdq_slots) & 1);
        if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 0x63) ||
            !mbar_wait(&wdq_full_bar[slot], slot_phase, abort_flag, p.wait_budget_ns, 0x64)) {
          ok = false;
          break;
        }
        tcgen05_fence_after_sync();
        const uint32_t w_addr = smem_u32(wdq_smem + slot * Cfg::WDQ_BYTES);
        const uint32_t a_addr = smem_u32(a_smem + stage * p.a_stage_bytes);
#pragma unroll
        for (int k = 0; k < Cfg::BK / 16; ++k) {
          const uint64_t adesc = make_sw128_desc(w_addr + k * 32, 16, 1024);
          const uint64_t bdesc = make_sw128_desc(a_addr + k * 32, 16, 1024);
          umma_f16_ss(tmem_base, adesc, bdesc, p.idesc, (i | k) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
        umma_commit(&wdq_empty_bar[slot]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && my_blocks > 0) umma_commit(acc_full_bar);
      umma_commit(mma_done_bar);
      volatile int no_abort = 0;
      mbar_wait(mma_done_bar, 0, &no_abort, p.wait_budget_ns, 0x65);
    }
    __syncwarp();
  } else if (warp >= Cfg::DQ_WARP0) {
    // Dequantization: thread t owns row t/2 of the panel and 32 of its 64
    // codes per k-block (4 chunks of 8).
    const int t = threadIdx.x - Cfg::DQ_WARP0 * 32;  // 0..255
    const int r = t >> 1;
    const int half = t & 1;
    const bool row_ok = n0 + r < p.N;
    const int groups_per_row = p.K / p.group;
    const __half* srow = p.S + static_cast<int64_t>(row_ok ? n0 + r : 0) * groups_per_row;
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < my_blocks; ++i) {
      const int kb = kb_lo + i;
      const int slot = i % p.wdq_slots;
      const uint32_t slot_phase = static_cast<uint32_t>((i / p.wdq_slots) & 1);
      const bool ready = mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_budget_ns, 0x66) &&
                         mbar_wait(&wdq_empty_bar[slot], slot_phase ^ 1u, abort_flag, p.wait_budget_ns, 0x67);
      if (!__all_sync(0xffffffffu, ready)) break;
      // Rows past N were zero-filled by TMA; a zero scale keeps them finite.
      const int g = (kb * Cfg::BK + half * 32) / p.group;
      __half s = __float2half(0.0f);
      if (row_ok) {
        s = p.scale_tma ? reinterpret_cast<const __half*>(scale_smem + stage * Cfg::SCALE_BYTES + r * 16)[g & 7]
                        : srow[g];
      }
      const __half2 s2 = __halves2half2(s, s);
      const uint4 codes = *reinterpret_cast<const uint4*>(packed_smem + stage * Cfg::PACKED_BYTES + r * 32 + half * 16);
      uint8_t* dst = wdq_smem + slot * Cfg::WDQ_BYTES + r * 128;
      const uint32_t words[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int chunk = half * 4 + j;  // 8 fp16 values = 16 bytes
        *reinterpret_cast<uint4*>(dst + ((chunk ^ (r & 7)) << 4)) = dequant8(words[j], s2);
      }
      fence_proxy_async_smem();  // the generic-proxy writes become visible to the MMA's reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&wdq_full_bar[slot]);
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else {
    // Epilogue warps: TMEM partial -> shared memory [m][n] (fp32).
    const int quad = warp & 3;
    const int n_local = quad * 32 + lane;
    bool ready = true;
    if (my_blocks > 0) ready = mbar_wait(acc_full_bar, 0, abort_flag, p.wait_budget_ns, 0x68);
    ready = __all_sync(0xffffffffu, ready);
    if (ready) {
      tcgen05_fence_after_sync();
      for (int c = 0; c < p.m_pad / 16; ++c) {
        uint32_t rr[16];
        if (my_blocks > 0) {
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c * 16, rr);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) rr[e] = 0u;
        }
        // The rings are free once the last MMA has completed (acc_full).
#pragma unroll
        for (int e = 0; e < 16; ++e) partial[(c * 16 + e) * Cfg::PANEL + n_local] = __uint_as_float(rr[e]);
      }
    }
    tcgen05_fence_before_sync();
  }

  __syncthreads();
  cluster_sync();  // every partial of the cluster is in shared memory

  if (warp >= Cfg::EPI_WARP0 && warp < Cfg::DQ_WARP0 && !*abort_flag) {
    // Reduction over the S partials in rank order; items are (m, 4-column group).
    const int e = threadIdx.x - Cfg::EPI_WARP0 * 32;  // 0..127
    const int items = p.M * (Cfg::PANEL / 4);
    const int lo = static_cast<int>((static_cast<int64_t>(items) * rank) / p.splits);
    const int hi = static_cast<int>((static_cast<int64_t>(items) * (rank + 1)) / p.splits);
    const uint32_t part_addr = smem_u32(partial);
    for (int it = lo + e; it < hi; it += 128) {
      const int m = it / (Cfg::PANEL / 4);
      const int j = it - m * (Cfg::PANEL / 4);
      const int n = n0 + 4 * j;
      if (n >= p.N) continue;
      const uint32_t off = static_cast<uint32_t>((m * Cfg::PANEL + 4 * j) * 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < p.splits; ++q) {
        const float4 v = ld_shared_cluster_f4(mapa_shared(part_addr + off, static_cast<uint32_t>(q)));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const __half2 h01 = __floats2half2_rn(acc.x > 0.f ? acc.x : 0.f, acc.y > 0.f ? acc.y : 0.f);
      const __half2 h23 = __floats2half2_rn(acc.z > 0.f ? acc.z : 0.f, acc.w > 0.f ? acc.w : 0.f);
      uint2 packed;
      packed.x = *reinterpret_cast<const uint32_t*>(&h01);
      packed.y = *reinterpret_cast<const uint32_t*>(&h23);
      __half* dst = p.C + static_cast<int64_t>(m) * p.N + n;
      if (p.c_aligned) {
        *reinterpret_cast<uint2*>(dst) = packed;
      } else {
        unsigned short* d16 = reinterpret_cast<unsigned short*>(dst);
        const uint32_t w[2] = {packed.x, packed.y};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (n + q < p.N) d16[q] = static_cast<unsigned short>(w[q >> 1] >> ((q & 1) * 16));
      }
    }
  }

  cluster_sync();  // peers are done reading this CTA's partial
  if (warp == 1) {
    tcgen05_fence_after_sync();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// Decode kernel (M <= 16): dequantization in registers, warp-level MMAs
// ---------------------------------------------------------------------------
// A decode step is bound by streaming the packed weight from HBM, so this
// kernel keeps every step of a warp's work in its own registers: no shared
// memory round trip for the dequantized weight and no hand-off to an MMA
// thread.  A warp owns 32 weight rows (4 groups of 8, the n side of
// mma.sync.m16n8k16); per 256-deep step of K the 4 lanes that share a row
// load its 128 bytes (256 codes) as two 64-byte halves, 16 bytes per lane
// per half, so every load instruction reads whole 32-byte sectors.  The codes are dequantized with the arithmetic of dequant8_pairs and
// fed straight into the MMA (fp16 operands, fp32 accumulation) as the B
// fragment.  The pairs come out as (e_i, e_{i+4}); instead of reordering
// them, the k order of the MMA is permuted the same way on the activation
// side, where byte permutes build the A fragments from the CTA's slice of
// the activations (rows 0..15, zero past M), copied once into shared memory
// by cp.async in row order with the 16-byte chunks of each 128-byte line
// XOR-swizzled so that the fragment reads are conflict-free.  A sum over k
// is the same sum in any order, so only the fp32 rounding order changes.
//
// Grid (S, N/128): a cluster of S CTAs along K shares a 128-column panel;
// each CTA (4 warps) streams its K/S slice with two steps of codes and
// scales in flight per warp, then the cluster adds its S fp32 partials
// through distributed shared memory in rank order (deterministic) and
// writes ReLU(sum) rounded to fp16.
struct W4DecodeParams {
  const __half* A;    // M x K
  const uint8_t* Wq;  // N x K/2
  const __half* S;    // N x K/group
  __half* C;          // M x N
  int M, N, K;
  int group_shift;    // log2(group)
  int k_split;        // K per CTA: a multiple of kW4DecodeStepK, at most kW4DecodeMaxSplit
};

constexpr int kW4DecodeThreads = 128;
constexpr int kW4DecodePanel = 128;      // columns per CTA: 4 warps x 32
constexpr int kW4DecodeStepK = 256;      // K per main-loop step: 128 bytes of each weight row
constexpr int kW4DecodeMaxSplit = 2048;  // K per CTA (its A fragments take k_split * 32 bytes)

__host__ __device__ constexpr int w4_decode_smem_bytes(int k_split) { return k_split * 32 + 16 * kW4DecodePanel * 4; }

// Byte offset of the 16-byte chunk kc (8 activations) of row r in the CTA's
// activation slice: rows of k_split * 2 bytes, and inside each 128-byte line
// the chunk position XOR (2 (line mod 2) + (r mod 2)).  The lanes of a
// quarter warp read rows g, g + 1 at chunks 4t + q (+ a multiple of 16):
// positions q and q + 4 of two consecutive lines, which the XOR spreads over
// the eight 16-byte bank groups.
__device__ __forceinline__ uint32_t w4_act_offset(int r, int kc, int k_split) {
  const int line = kc >> 3;
  const int pos = (kc & 7) ^ (((line & 1) << 1) | (r & 1));
  return static_cast<uint32_t>(r * k_split * 2 + line * 128 + pos * 16);
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void mma_m16n8k16_f16_f32(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// Codes and scales of one step for one lane: per row group, 8 words (64
// codes: k = 128 u + 32 t + 8 q + i of the step) and the scales of its
// halves u = 0, 1 (low and high half).
struct W4DecodeStep {
  uint4 w[4][2];
  __half2 s[4];
};

__global__ void __launch_bounds__(kW4DecodeThreads, 4) gemm_relu_w4a16_decode_kernel(const W4DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t act = smem_u32(smem);                            // [16][k_split] fp16, swizzled
  float* part = reinterpret_cast<float*>(smem + p.k_split * 32);  // [16][128] fp32
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t split = cluster_ctarank();
  const int splits = static_cast<int>(gridDim.x);
  const int k0 = static_cast<int>(blockIdx.x) * p.k_split;
  const int n_panel = static_cast<int>(blockIdx.y) * kW4DecodePanel;
  const int nsteps = p.k_split / kW4DecodeStepK;
  const int64_t row_bytes = p.K / 2;
  const int64_t scales_per_row = p.K >> p.group_shift;

  grid_dependency_wait();
  grid_launch_dependents();

  // The activation slice: every copy in flight at once, no registers held.
  {
    const int chunks = p.k_split / 8;
    for (int idx = threadIdx.x; idx < 16 * chunks; idx += kW4DecodeThreads) {
      const int r = idx / chunks, kc = idx - r * chunks;
      const __half* src = p.A + static_cast<int64_t>(r < p.M ? r : 0) * p.K + k0 + 8 * kc;
      cp_async_16(act + w4_act_offset(r, kc, p.k_split), src, r < p.M ? 16u : 0u);
    }
  }

  // This lane's weight rows (one per 8-column group; a row past N reads row
  // N - 1 instead, whose columns are never stored) and the byte where its
  // first 32 codes of step 0 start.
  const int n_lane = n_panel + warp * 32 + g;
  const uint8_t* wbase = p.Wq + k0 / 2 + 16 * t;
  auto row_of = [&](int gi) { return static_cast<int64_t>(min(n_lane + gi * 8, p.N - 1)); };
  // Step c's codes and scales (nothing is read past the slice).
  auto load = [&](int c, W4DecodeStep& d) {
    if (c >= nsteps) return;
    const int kq = k0 + kW4DecodeStepK * c + 32 * t;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const int64_t n = row_of(gi);
      const uint8_t* src = wbase + n * row_bytes + c * 128;
      d.w[gi][0] = __ldg(reinterpret_cast<const uint4*>(src));
      d.w[gi][1] = __ldg(reinterpret_cast<const uint4*>(src + 64));
      const __half* srow = p.S + n * scales_per_row;
      d.s[gi] = __halves2half2(__ldg(srow + (kq >> p.group_shift)), __ldg(srow + ((kq + 128) >> p.group_shift)));
    }
  };
  W4DecodeStep cur, nxt;
  load(0, cur);
  load(1, nxt);

  cp_async_commit_wait_all();
  __syncthreads();

  float acc[4][4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[gi][e] = 0.0f;

#pragma unroll 1
  for (int c = 0; c < nsteps; ++c) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // Word q of each group gives k-steps 2q ((e0,e4), (e1,e5)) and 2q + 1
        // ((e2,e6), (e3,e7)); the activations of rows g and g + 8 at the same
        // 8 k build the A fragments of both (words 0/2 from row g, 1/3 from
        // row g + 8).
        const int kc = 32 * c + 16 * u + 4 * t + q;
        const uint4 lo = lds128(act + w4_act_offset(g, kc, p.k_split));
        const uint4 hi = lds128(act + w4_act_offset(g + 8, kc, p.k_split));
        const uint4 af0 = make_uint4(__byte_perm(lo.x, lo.z, 0x5410), __byte_perm(hi.x, hi.z, 0x5410),
                                     __byte_perm(lo.x, lo.z, 0x7632), __byte_perm(hi.x, hi.z, 0x7632));
        const uint4 af1 = make_uint4(__byte_perm(lo.y, lo.w, 0x5410), __byte_perm(hi.y, hi.w, 0x5410),
                                     __byte_perm(lo.y, lo.w, 0x7632), __byte_perm(hi.y, hi.w, 0x7632));
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          const uint4& w = cur.w[gi][u];
          const uint32_t word = q == 0 ? w.x : q == 1 ? w.y : q == 2 ? w.z : w.w;
          uint32_t bv[4];
          dequant8_pairs(word, u == 0 ? __low2half2(cur.s[gi]) : __high2half2(cur.s[gi]), bv);
          mma_m16n8k16_f16_f32(acc[gi], af0, bv[0], bv[1]);
          mma_m16n8k16_f16_f32(acc[gi], af1, bv[2], bv[3]);
        }
      }
    }
    cur = nxt;
    load(c + 2, nxt);
  }

  // This CTA's fp32 partial: rows g and g + 8, columns 2t, 2t + 1 of each group.
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    const int col = warp * 32 + gi * 8 + 2 * t;
    *reinterpret_cast<float2*>(part + g * kW4DecodePanel + col) = make_float2(acc[gi][0], acc[gi][1]);
    *reinterpret_cast<float2*>(part + (g + 8) * kW4DecodePanel + col) = make_float2(acc[gi][2], acc[gi][3]);
  }
  cluster_sync();  // every partial of the cluster is written

  // CTA `split` finishes columns [split * 128 / S, +128 / S): four at a time,
  // the S partials added in rank order.
  const int cols = kW4DecodePanel / splits;
  const int quads = 16 * cols / 4;
  for (int i = threadIdx.x; i < quads; i += kW4DecodeThreads) {
    const int r = (i * 4) / cols;
    const int cl = static_cast<int>(split) * cols + (i * 4) % cols;
    if (r >= p.M) continue;
    const uint32_t local = smem_u32(part + r * kW4DecodePanel + cl);
    float4 v[8];  // all remote reads in flight before the adds (splits <= 8)
#pragma unroll
    for (int rk = 0; rk < 8; ++rk)
      if (rk < splits) v[rk] = ld_shared_cluster_f4(mapa_shared(local, static_cast<uint32_t>(rk)));
    float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int rk = 0; rk < 8; ++rk) {
      if (rk < splits) {
        sum.x += v[rk].x;
        sum.y += v[rk].y;
        sum.z += v[rk].z;
        sum.w += v[rk].w;
      }
    }
    const float o[4] = {sum.x, sum.y, sum.z, sum.w};
    __half* crow = p.C + static_cast<int64_t>(r) * p.N;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = n_panel + cl + e;
      if (n < p.N) crow[n] = __float2half_rn(o[e] > 0.0f ? o[e] : 0.0f);
    }
  }
  cluster_sync();  // no CTA leaves while a peer may still read its partial
}

}  // namespace tg
