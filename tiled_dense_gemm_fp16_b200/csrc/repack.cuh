// repack.cuh -- copy a row-major fp16 matrix whose rows are not 16-byte
// aligned into a row-major copy with rows padded to a multiple of 8 elements
// (16 bytes), zero in the padding, so that TMA can describe it; and the
// reverse copy for C (unpad_rows_kernel below).
//
// Used by the workspace path of C = ReLU(A . B) for operands whose leading
// dimension (K for A, N for B) is not a multiple of 8 or whose base address
// is not 16-byte aligned.  Zero padding columns contribute nothing to the K
// sum (A) and produce output columns that are never stored (B).
//
// Bandwidth-bound: every thread writes whole 16-byte chunks of the padded
// copy; a chunk's 8 source values are read with two aligned 16-byte loads and
// shifted into place (the loads of several chunks are issued before any is
// used), with a scalar path at row ends and at the edges of the source.  No
// byte outside the source matrix is read.
#pragma once

#include <cuda_fp16.h>

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace tg {

struct RepackParams {
  const __half* src;
  __half* dst;
  int64_t src_ld;            // row stride of the source (elements, >= cols)
  int rows, cols, cols_pad;  // cols_pad = cols rounded up to a multiple of 8
  int64_t chunks;            // rows * cols_pad / 8
};

// Index: the type of the chunk arithmetic.  32-bit when the copy has fewer
// than 2^31 chunks (a 32-bit division per chunk instead of a 64-bit one,
// which is a long software routine on the GPU), else 64-bit.
template <typename Index>
__device__ __forceinline__ void pad_rows_body(const RepackParams& p) {
  constexpr int kUnroll = 4;
  const Index chunks_per_row = static_cast<Index>(p.cols_pad >> 3);
  const Index chunks = static_cast<Index>(p.chunks);
  const __half* src_end = p.src + static_cast<int64_t>(p.rows - 1) * p.src_ld + p.cols;
  const Index stride = static_cast<Index>(gridDim.x) * blockDim.x;
  for (Index base = static_cast<Index>(blockIdx.x) * blockDim.x + threadIdx.x; base < chunks;
       base += stride * kUnroll) {
    EdgeChunk plan[kUnroll];
    int row[kUnroll], col[kUnroll];
    bool live[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const Index c = base + u * stride;
      live[u] = c < chunks;
      row[u] = live[u] ? static_cast<int>(c / chunks_per_row) : 0;
      col[u] = live[u] ? static_cast<int>(c - static_cast<Index>(row[u]) * chunks_per_row) * 8 : 0;
      plan[u] = edge_chunk_plan(p.src, src_end, p.src_ld, live[u] ? row[u] : p.rows, p.rows, col[u], p.cols);
    }
    uint4 lo[kUnroll], hi[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      lo[u] = make_uint4(0u, 0u, 0u, 0u);
      hi[u] = lo[u];
      ld_nc_v4_pred(lo[u], plan[u].src, plan[u].fast);
      ld_nc_v4_pred(hi[u], plan[u].src + 1, plan[u].fast);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!live[u]) continue;
      const uint4 v = plan[u].fast ? edge_realign(lo[u], hi[u], plan[u].shift)
                                   : load_chunk_pred(p.src, p.src_ld, row[u], p.rows, col[u], p.cols);
      *reinterpret_cast<uint4*>(p.dst + static_cast<int64_t>(row[u]) * p.cols_pad + col[u]) = v;
    }
  }
}

__global__ void __launch_bounds__(256) pad_rows_kernel(const RepackParams p) {
  grid_dependency_wait();
  grid_launch_dependents();
  if (p.chunks < (int64_t(1) << 31))
    pad_rows_body<uint32_t>(p);
  else
    pad_rows_body<int64_t>(p);
}

// The reverse copy, for C: the GEMM writes a padded copy (rows of cols_pad
// elements, 16-byte aligned) and this kernel moves it into C, whose rows may
// start on any 2-byte boundary.  Each thread writes one 16-byte-aligned block
// of a destination row: its 8 values are read with two aligned 16-byte loads
// of the padded copy and shifted into place, so every interior store is a
// whole aligned 16 bytes; the partial blocks at either end of a row are
// written element by element.  Nothing outside [0, cols) of a row is written,
// and nothing outside the padded copy is read.
struct UnpadParams {
  const __half* src;  // rows x cols_pad, 16-byte aligned
  __half* dst;        // rows of `cols` elements, row stride dst_ld, 2-byte aligned
  int64_t dst_ld;
  int rows, cols, cols_pad;
  int blocks_per_row;  // cols / 8 + 2: enough 16-byte blocks for any alignment of a row
  int64_t blocks;      // rows * blocks_per_row
};

// Index as in pad_rows_body.
template <typename Index>
__device__ __forceinline__ void unpad_rows_body(const UnpadParams& p) {
  constexpr int kUnroll = 4;  // four blocks' loads in flight per thread before any store
  const uintptr_t src_end = reinterpret_cast<uintptr_t>(p.src + static_cast<int64_t>(p.rows) * p.cols_pad);
  const Index blocks = static_cast<Index>(p.blocks);
  const Index blocks_per_row = static_cast<Index>(p.blocks_per_row);
  const Index stride = static_cast<Index>(gridDim.x) * blockDim.x;
  for (Index base = static_cast<Index>(blockIdx.x) * blockDim.x + threadIdx.x; base < blocks;
       base += stride * kUnroll) {
    __half* drow[kUnroll];
    const __half* srow[kUnroll];
    int e0[kUnroll];
    uintptr_t s[kUnroll], s0[kUnroll];
    bool fast[kUnroll], live[kUnroll];
    uint4 lo[kUnroll], hi[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const Index i = base + u * stride;
      live[u] = i < blocks;
      const int r = live[u] ? static_cast<int>(i / blocks_per_row) : 0;
      const int j = live[u] ? static_cast<int>(i - static_cast<Index>(r) * blocks_per_row) : 0;
      drow[u] = p.dst + static_cast<int64_t>(r) * p.dst_ld;
      srow[u] = p.src + static_cast<int64_t>(r) * p.cols_pad;
      // Elements before the row's first aligned block, then block j's first element.
      const int a = static_cast<int>((reinterpret_cast<uintptr_t>(drow[u]) & 15u) >> 1);
      e0[u] = 8 * j - a;
      live[u] = live[u] && e0[u] < p.cols;
      s[u] = reinterpret_cast<uintptr_t>(srow[u] + e0[u]);
      s0[u] = s[u] & ~uintptr_t(15);
      fast[u] = live[u] && e0[u] >= 0 && e0[u] + 8 <= p.cols && (s0[u] + 32 <= src_end || s[u] == s0[u]);
      lo[u] = make_uint4(0u, 0u, 0u, 0u);
      hi[u] = lo[u];
      if (fast[u]) {
        lo[u] = __ldg(reinterpret_cast<const uint4*>(s0[u]));
        if (s[u] != s0[u]) hi[u] = __ldg(reinterpret_cast<const uint4*>(s0[u]) + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!live[u]) continue;
      if (fast[u]) {
        *reinterpret_cast<uint4*>(drow[u] + e0[u]) = edge_realign(lo[u], hi[u], static_cast<uint32_t>(s[u] - s0[u]));
      } else {
        for (int k = 0; k < 8; ++k) {
          const int e = e0[u] + k;
          if (e >= 0 && e < p.cols) drow[u][e] = srow[u][e];
        }
      }
    }
  }
}

__global__ void __launch_bounds__(256) unpad_rows_kernel(const UnpadParams p) {
  grid_dependency_wait();
  grid_launch_dependents();
  if (p.blocks < (int64_t(1) << 31))
    unpad_rows_body<uint32_t>(p);
  else
    unpad_rows_body<int64_t>(p);
}

}  // namespace tg

namespace tg {

// K == 0 with a bias: every row of C is ReLU(bias) rounded to fp16 (the sum
// over an empty K range is zero).
struct BiasRowsParams {
  __half* C;
  const __half* bias;
  int64_t ldc;
  int M, N;
};

__global__ void __launch_bounds__(256) bias_relu_rows_kernel(const BiasRowsParams p) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t total = static_cast<int64_t>(p.M) * p.N;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int m = static_cast<int>(i / p.N);
    const int n = static_cast<int>(i - static_cast<int64_t>(m) * p.N);
    const float b = __half2float(p.bias[n]);
    p.C[static_cast<int64_t>(m) * p.ldc + n] = __float2half_rn(b > 0.0f ? b : 0.0f);
  }
}

}  // namespace tg
