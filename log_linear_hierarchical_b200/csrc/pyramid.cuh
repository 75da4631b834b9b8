// Step 1: the mean-pooled Q/K/V pyramid ("Trainable Log-linear Sparse Attention for
// Efficient Diffusion Transformers", abstract: block-wise compression of tokens; skill page
// "Log Linear Sparse Attention", Core Technique 1).
//
// Level l token j = (((0 + x_0) + x_1) + ... + x_15) * (1/16) over the 16 level-(l-1) tokens
// 16j..16j+15, each addition rounded to fp32 in that order (__fadd_rn keeps the compiler
// from re-associating or contracting), so results are bit-identical to any other
// implementation of the same order.
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

// Dynamic shared memory of pyramid_l12_kernel<T>: its span of ROWS * 16 input rows.
template <typename T>
constexpr int pyramid_span_bytes() {
  return (kPyrThreads / (kD / (16 / (int)sizeof(T)))) * kBlock * kD * (int)sizeof(T);
}

// grid.x = B*H * ceil(n_1 / rows_per_cta), grid.y = 3 (q, k, v).
// Each thread owns kElems consecutive channels of one level-1 output row.
template <typename T>
__global__ void __launch_bounds__(kPyrThreads) pyramid_l12_kernel(Geometry g, const T* __restrict__ x0,
                                                                  const T* __restrict__ x1,
                                                                  const T* __restrict__ x2, float* __restrict__ p0,
                                                                  float* __restrict__ p1, float* __restrict__ p2) {
  pdl_enter();
  constexpr int VE = Vec16<T>::kElems;
  constexpr int TPR = kD / VE;                   // threads per row
  constexpr int ROWS = kPyrThreads / TPR;         // level-1 rows per CTA (32 for bf16, 16 for fp32)
  __shared__ float s1[ROWS][kD];
  __shared__ __align__(8) uint64_t bar_storage;
  extern __shared__ __align__(128) uint8_t pyr_span[];  // ROWS * 16 input rows (pyramid_span_bytes)

  const T* x = blockIdx.y == 0 ? x0 : (blockIdx.y == 1 ? x1 : x2);
  float* pyr = blockIdx.y == 0 ? p0 : (blockIdx.y == 1 ? p1 : p2);

  const int n1 = g.n[1];
  const int tiles = (n1 + ROWS - 1) / ROWS;
  const int bh = blockIdx.x / tiles;
  const int tile = blockIdx.x - bh * tiles;
  const int t = threadIdx.x;
  const int o = t / TPR;
  const int c0 = (t % TPR) * VE;
  const int j1 = tile * ROWS + o;

  const uint32_t bar = smem_u32(&bar_storage);
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (t == 0) {
    const uint32_t bytes = (uint32_t)(min(ROWS, n1 - tile * ROWS) * kBlock * kD * (int)sizeof(T));
    mbar_expect_tx(bar, bytes);
    bulk_load(smem_u32(pyr_span), x + ((long long)bh * g.N + (long long)tile * ROWS * kBlock) * kD, bytes, bar);
  }
  if (!mbar_wait(bar, 0)) {  // recorded as LLSA_ERR_TIMEOUT; give the copy one more bounded wait
    mbar_wait(bar, 0);
    return;
  }

  if (j1 < n1) {
    const T* src = reinterpret_cast<const T*>(pyr_span) + (o * kBlock) * kD + c0;
    float v[kBlock][VE];
#pragma unroll
    for (int r = 0; r < kBlock; ++r) Vec16<T>::load(src + r * kD, v[r]);
    float acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0f;
#pragma unroll
    for (int r = 0; r < kBlock; ++r)
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = __fadd_rn(acc[e], v[r][e]);
    float* dst = pyr + g.pyr_off[1] + ((long long)bh * n1 + j1) * kD + c0;
#pragma unroll
    for (int e = 0; e < VE; ++e) {
      acc[e] = __fmul_rn(acc[e], 0.0625f);
      s1[o][c0 + e] = acc[e];
    }
    if constexpr (VE == 8) {
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
  }
  if (g.L < 2) return;
  __syncthreads();
  constexpr int OUT2 = ROWS / kBlock;  // level-2 rows per CTA
  if (t < OUT2 * kD) {
    const int o2 = t / kD;
    const int d = t % kD;
    const int j2 = tile * OUT2 + o2;
    if (j2 < g.n[2] && (j2 + 1) * kBlock <= n1) {
      float acc = 0.0f;
#pragma unroll
      for (int r = 0; r < kBlock; ++r) acc = __fadd_rn(acc, s1[o2 * kBlock + r][d]);
      pyr[g.pyr_off[2] + ((long long)bh * g.n[2] + j2) * kD + d] = __fmul_rn(acc, 0.0625f);
    }
  }
}

// Level l >= 3 from level l-1 (fp32).  One thread per output value; grid.y = tensor.
__global__ void __launch_bounds__(kPyrThreads) pyramid_up_kernel(Geometry g, int level, float* __restrict__ p0,
                                                                 float* __restrict__ p1, float* __restrict__ p2) {
  pdl_enter();
  float* pyr = blockIdx.y == 0 ? p0 : (blockIdx.y == 1 ? p1 : p2);
  const long long total = (long long)g.BH * g.n[level] * kD;
  const long long i = (long long)blockIdx.x * kPyrThreads + threadIdx.x;
  if (i >= total) return;
  const int d = (int)(i % kD);
  const long long row = i / kD;  // bh * n_l + j
  const int nl = g.n[level];
  const long long bh = row / nl;
  const int j = (int)(row - bh * nl);
  const float* src = pyr + g.pyr_off[level - 1] + (bh * g.n[level - 1] + (long long)j * kBlock) * kD + d;
  float acc = 0.0f;
#pragma unroll
  for (int r = 0; r < kBlock; ++r) acc = __fadd_rn(acc, src[r * kD]);
  pyr[g.pyr_off[level] + row * kD + d] = __fmul_rn(acc, 0.0625f);
}

}  // namespace llsa
