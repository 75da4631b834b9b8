// Step 1: the mean-pooled Q/K/V pyramid ("Trainable Log-linear Sparse Attention for
// Efficient Diffusion Transformers", abstract: block-wise compression of tokens; skill page
// "Log Linear Sparse Attention", Core Technique 1).
//
// Level l token j = (((0 + x_0) + x_1) + ... + x_15) * (1/16) over the 16 level-(l-1) tokens
// 16j..16j+15, each addition rounded to fp32 in that order (__fadd_rn keeps the compiler
// from re-associating or contracting), so results are bit-identical to any other
// implementation of the same order.
// A padded sequence (nv < N real tokens) changes only the tokens whose span reaches past nv
// (pooled_mean below): they average their c real tokens, level 1 as (sum of the real tokens
// in order) / c, level l >= 2 as (sum in order of c_child * child) / c, and empty ones are 0.
//
// Bound: HBM streaming.  Reads B*H*N*D input elements of each of q, k, v once and writes
// B*H*D*sum_l n_l fp32 values per tensor; levels 1 and 2 are produced by one kernel (the
// 16 level-1 rows that make a level-2 row stay in shared memory), levels >= 3 by a small
// kernel per level reading the L2-resident level below.  The level-1/2 kernel brings its
// input span (ROWS * 16 contiguous token rows, 64 KB) into shared memory with one bulk copy
// completing on an mbarrier, so a CTA has its whole span in flight at once.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

template <typename T>
struct Vec16 {};

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&out)[8]) {  // shared memory
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // bf16 -> fp32 widening is exact: the bf16 bits become the top half of the float.
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

template <>
struct Vec16<float> {
  static constexpr int kElems = 4;
  __device__ __forceinline__ static void load(const float* p, float (&out)[4]) {  // shared memory
    const float4 u = *reinterpret_cast<const float4*>(p);
    out[0] = u.x;
    out[1] = u.y;
    out[2] = u.z;
    out[3] = u.w;
  }
};

constexpr int kPyrThreads = 256;

// Mean of a token from its in-order fp32 sum and its count of real tokens: the exact
// power-of-two scaling for a full token (the unpadded pyramid), 0 for an empty one, a
// correctly rounded division otherwise.
__device__ __forceinline__ float pooled_mean(float sum, int count, int full) {
  if (count == full) return __fmul_rn(sum, 1.0f / (float)full);
  return count == 0 ? 0.0f : __fdiv_rn(sum, (float)count);
}

// Level-l token j (l >= 2) of level-(l-1) rows src[r * stride], r < 16: (sum of the 16
// rows) / 16 for a full token; the count-weighted form for a token a padded sequence cuts.
__device__ __forceinline__ float pool_up(const Geometry& g, int l, int j, const float (&x)[kBlock]) {
  const int c = pool_count(g, l, j);
  const int full = 1 << (4 * l);
  float acc = 0.0f;
  if (c == full) {
#pragma unroll
    for (int r = 0; r < kBlock; ++r) acc = __fadd_rn(acc, x[r]);
    return __fmul_rn(acc, 0.0625f);
  }
#pragma unroll
  for (int r = 0; r < kBlock; ++r) acc = __fadd_rn(acc, __fmul_rn((float)pool_count(g, l - 1, j * kBlock + r), x[r]));
  return c == 0 ? 0.0f : __fdiv_rn(acc, (float)c);
}

// Launch shape of pyramid_l12_kernel<T, D>: each thread owns VE consecutive channels of one
// level-1 output row; a CTA makes ROWS level-1 rows (at least 16, so whole level-2 rows)
// from its span of ROWS * 16 input rows.
template <typename T, int D>
struct PyrCfg {
  static constexpr int VE = Vec16<T>::kElems;
  static constexpr int TPR = D / VE;                                          // threads per row
  static constexpr int ROWS = kPyrThreads / TPR > kBlock ? kPyrThreads / TPR : kBlock;
  static constexpr int THREADS = ROWS * TPR;
  static constexpr int SPAN = ROWS * kBlock * D * (int)sizeof(T);             // dynamic smem bytes
};

// One unit of levels 1-2: ROWS level-1 rows (tile `tile` of head bh) of one tensor x, and
// the level-2 rows they make.  The CTA's input span (ROWS * 16 token rows) arrives by one
// bulk copy completing on `bar` with phase parity `parity`, or, under grid order, as ROWS/16
// 16 x 16 pixel patches (one level-2 token each) by TMA boxes of `pmap`; `span` and `s1` are
// the CTA's shared buffers.  Under grid order `zout` (if not null) also receives the span's
// tokens in quadtree order (the step's copies of q, k, v and dO), and `pyr` may be null for a
// tensor that is only copied.  Every thread of the CTA calls it; returns false (for the whole
// CTA) if the copy did not land within the bounded wait.
template <typename T, int D>
__device__ __forceinline__ bool pyramid_l12_unit(const Geometry& g, const T* __restrict__ x,
                                                 float* __restrict__ pyr, int bh, int tile, uint8_t* span,
                                                 float (*s1)[D], uint32_t bar, uint32_t parity,
                                                 const CUtensorMap* pmap, T* __restrict__ zout = nullptr) {
  using C = PyrCfg<T, D>;
  constexpr int VE = C::VE;
  constexpr int TPR = C::TPR;
  constexpr int ROWS = C::ROWS;
  const int n1 = g.n[1];
  const int t = threadIdx.x;
  const int o = t / TPR;
  const int c0 = (t % TPR) * VE;
  const int j1 = tile * ROWS + o;
  __syncthreads();  // the span and s1 of the previous unit are no longer read
  constexpr int OUT2 = ROWS / kBlock;  // level-2 rows per unit
  constexpr int PATCH = kBlock * kBlock * D * (int)sizeof(T);
  if (t == 0) {
    const uint32_t bytes = (uint32_t)(min(ROWS, n1 - tile * ROWS) * kBlock * D * (int)sizeof(T));
    mbar_expect_tx(bar, bytes);
    if (g.grid) {
      const int lg2 = g.log_g - 4;  // level-2 tokens per grid row: G / 16
      for (int o2 = 0; o2 < OUT2 && (tile * OUT2 + o2) * kBlock < n1; ++o2) {
        const int p = z_to_rowmajor(tile * OUT2 + o2, lg2);
        tma_load_4d(smem_u32(span) + o2 * PATCH, pmap, 0, 16 * (p & ((1 << lg2) - 1)), 16 * (p >> lg2), bh, bar);
      }
    } else {
      bulk_load(smem_u32(span), x + ((long long)bh * g.N + (long long)tile * ROWS * kBlock) * D, bytes, bar);
    }
  }
  if (!__syncthreads_and(mbar_wait(bar, parity))) {
    mbar_wait(bar, parity);  // recorded as LLSA_ERR_TIMEOUT; one more bounded wait for the copy
    return false;
  }
  if (j1 < n1) {
    float v[kBlock][VE];
    if (g.grid) {
      // level-1 token o is block o % 16 (quadtree order) of patch o / 16; its token r is
      // pixel (4 br + tr, 4 bc + tc) of the patch, rows of 16 pixels
      const T* patch = reinterpret_cast<const T*>(span + (o >> 4) * PATCH) + c0;
      const int b = o & 15;
      const int br = compact_even_bits(b >> 1), bc = compact_even_bits(b);
      if (zout) {  // the block's 16 tokens, in quadtree order, to the copy (16 bytes a thread)
        T* zrow = zout + ((long long)bh * g.N + (long long)j1 * kBlock) * D + c0;
#pragma unroll
        for (int r = 0; r < kBlock; ++r) {
          const int tr = compact_even_bits(r >> 1), tc = compact_even_bits(r);
          *reinterpret_cast<uint4*>(zrow + r * D) =
              *reinterpret_cast<const uint4*>(patch + ((4 * br + tr) * kBlock + 4 * bc + tc) * D);
        }
      }
      if (!pyr) return true;  // a tensor that is only copied (every thread of the CTA returns)
#pragma unroll
      for (int r = 0; r < kBlock; ++r) {
        const int tr = compact_even_bits(r >> 1), tc = compact_even_bits(r);
        Vec16<T>::load(patch + ((4 * br + tr) * kBlock + 4 * bc + tc) * D, v[r]);
      }
    } else {
      const T* src = reinterpret_cast<const T*>(span) + (o * kBlock) * D + c0;
#pragma unroll
      for (int r = 0; r < kBlock; ++r) Vec16<T>::load(src + r * D, v[r]);
    }
    float acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0f;
    const int c1 = pool_count(g, 1, j1);  // 16 unless the sequence is padded
#pragma unroll
    for (int r = 0; r < kBlock; ++r)
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = __fadd_rn(acc[e], r < c1 ? v[r][e] : 0.0f);
    float* dst = pyr + g.pyr_off[1] + ((long long)bh * n1 + j1) * D + c0;
#pragma unroll
    for (int e = 0; e < VE; ++e) {
      acc[e] = pooled_mean(acc[e], c1, kBlock);
      s1[o][c0 + e] = acc[e];
    }
    if constexpr (VE == 8) {
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
  }
  if (!pyr || g.L < 2) return true;
  __syncthreads();
  for (int i = t; i < OUT2 * D; i += blockDim.x) {
    const int o2 = i / D;
    const int d = i % D;
    const int j2 = tile * OUT2 + o2;
    if (j2 < g.n[2] && (j2 + 1) * kBlock <= n1) {
      float xr[kBlock];
#pragma unroll
      for (int r = 0; r < kBlock; ++r) xr[r] = s1[o2 * kBlock + r][d];
      pyr[g.pyr_off[2] + ((long long)bh * g.n[2] + j2) * D + d] = pool_up(g, 2, j2, xr);
    }
  }
  return true;
}

// Quadtree-ordered copies made by pyramid_l12_kernel under grid order (the step's q, k, v,
// dO copies; null pointers: none).  Slice 3 (dO) is copied, not pooled.
template <typename T>
struct ZOut {
  T* z[4];
  const T* x3;
};

// grid.x = B*H * ceil(n_1 / ROWS), grid.y = 3 (q, k, v), or 4 with dO copied under grid order.
// pm0..pm3: the grid-order patch maps of q, k, v, dO (unused in quadtree order).
template <typename T, int D>
__global__ void __launch_bounds__(PyrCfg<T, D>::THREADS) pyramid_l12_kernel(Geometry g, const T* __restrict__ x0,
                                                                            const T* __restrict__ x1,
                                                                            const T* __restrict__ x2,
                                                                            float* __restrict__ p0,
                                                                            float* __restrict__ p1,
                                                                            float* __restrict__ p2,
                                                                            const __grid_constant__ CUtensorMap pm0,
                                                                            const __grid_constant__ CUtensorMap pm1,
                                                                            const __grid_constant__ CUtensorMap pm2,
                                                                            const __grid_constant__ CUtensorMap pm3,
                                                                            ZOut<T> zo) {
  pdl_enter();
  using C = PyrCfg<T, D>;
  __shared__ float s1[C::ROWS][D];
  __shared__ __align__(8) uint64_t bar_storage;
  extern __shared__ __align__(128) uint8_t pyr_span[];  // ROWS * 16 input rows (C::SPAN bytes)
  const int tiles = (g.n[1] + C::ROWS - 1) / C::ROWS;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  const int y = blockIdx.y;
  const T* x = y == 0 ? x0 : (y == 1 ? x1 : (y == 2 ? x2 : zo.x3));
  float* pyr = y == 0 ? p0 : (y == 1 ? p1 : (y == 2 ? p2 : nullptr));
  const CUtensorMap* pm = y == 0 ? &pm0 : (y == 1 ? &pm1 : (y == 2 ? &pm2 : &pm3));
  const int bh = blockIdx.x / tiles;
  pyramid_l12_unit<T, D>(g, x, pyr, bh, blockIdx.x - bh * tiles, pyr_span, s1, bar, 0, pm, zo.z[y]);
}

// Level l >= 3 from level l-1 (fp32).  One thread per output value; grid.y = tensor.
template <int D>
__global__ void __launch_bounds__(kPyrThreads) pyramid_up_kernel(Geometry g, int level, float* __restrict__ p0,
                                                                 float* __restrict__ p1, float* __restrict__ p2) {
  pdl_enter();
  float* pyr = blockIdx.y == 0 ? p0 : (blockIdx.y == 1 ? p1 : p2);
  const long long total = (long long)g.BH * g.n[level] * D;
  const long long i = (long long)blockIdx.x * kPyrThreads + threadIdx.x;
  if (i >= total) return;
  const int d = (int)(i % D);
  const long long row = i / D;  // bh * n_l + j
  const int nl = g.n[level];
  const long long bh = row / nl;
  const int j = (int)(row - bh * nl);
  const float* src = pyr + g.pyr_off[level - 1] + (bh * g.n[level - 1] + (long long)j * kBlock) * D + d;
  float x[kBlock];
#pragma unroll
  for (int r = 0; r < kBlock; ++r) x[r] = src[r * D];
  pyr[g.pyr_off[level] + row * D + d] = pool_up(g, level, j, x);
}

}  // namespace llsa
