// Quadtree (Z) token order of a square token grid (LLSA GitHub README, token reordering
// example: reorder image tokens so that similar, nearby tokens get adjacent indices, which
// is what makes 16-token blocks and their 16x pooling spatially compact).
//
// Grid position (r, c) of a side x side grid (row-major index r * side + c) has Z index
// z = sum_b (2 r_b + c_b) 4^b.  to_z: dst[z(p)] = src[p]; from_z: dst[p] = src[z(p)].
// One thread per 16-byte piece of a destination row; consecutive threads cover a row, so
// the writes are coalesced and each read is a whole token row.  HBM streaming: each
// element is read once and written once.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

constexpr int kZThreads = 256;

// Even bits of x packed together (bits 0, 2, 4, ... -> 0, 1, 2, ...).
__device__ __forceinline__ uint32_t z_compact(uint32_t x) {
  x &= 0x55555555u;
  x = (x | (x >> 1)) & 0x33333333u;
  x = (x | (x >> 2)) & 0x0f0f0f0fu;
  x = (x | (x >> 4)) & 0x00ff00ffu;
  x = (x | (x >> 8)) & 0x0000ffffu;
  return x;
}

// Bits of x spread to the even positions (inverse of z_compact).
__device__ __forceinline__ uint32_t z_spread(uint32_t x) {
  x &= 0x0000ffffu;
  x = (x | (x << 8)) & 0x00ff00ffu;
  x = (x | (x << 4)) & 0x0f0f0f0fu;
  x = (x | (x << 2)) & 0x33333333u;
  x = (x | (x << 1)) & 0x55555555u;
  return x;
}

// rows = B*H*N token rows of `row_bytes` bytes (a multiple of 16); log_side = log2(side).
__global__ void __launch_bounds__(kZThreads) zorder_permute_kernel(const uint4* __restrict__ src,
                                                                   uint4* __restrict__ dst, long long rows, int N,
                                                                   int log_side, int pieces, int to_z) {
  pdl_enter();
  const long long t = (long long)blockIdx.x * kZThreads + threadIdx.x;
  if (t >= rows * pieces) return;
  const long long row = t / pieces;
  const int piece = (int)(t - row * pieces);
  const long long bh = row / N;
  const uint32_t i = (uint32_t)(row - bh * N);  // destination position within the (b, h) grid
  uint32_t j;
  if (to_z) {  // destination is Z index i: its grid position
    const uint32_t r = z_compact(i >> 1), c = z_compact(i);
    j = (r << log_side) | c;
  } else {  // destination is grid position i: its Z index
    const uint32_t r = i >> log_side, c = i & ((1u << log_side) - 1u);
    j = (z_spread(r) << 1) | z_spread(c);
  }
  dst[t] = __ldg(src + (bh * N + j) * pieces + piece);
}

}  // namespace llsa
