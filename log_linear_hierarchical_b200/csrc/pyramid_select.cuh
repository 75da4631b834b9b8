// Steps 1 and 2 in one launch: the pyramid and the whole hierarchical selection (skill page
// "Log Linear Sparse Attention", Core Technique 1: the selection works on the compressed
// tokens, so it consumes the pyramid as soon as each level exists).
//
// A persistent cooperative kernel: every CTA takes the work units of one phase in turn
// (grid-stride), and the phases are separated by grid-wide barriers:
//   1. levels 1-2 of the q, k, v pyramids (pyramid_l12_unit: a span of input rows by one
//      bulk copy, level-1 rows kept in shared memory for level 2);
//   2. per (b, h): levels 3..L pooled and the coarsest Top-K (coarsest_small_unit);
//   3. per level l = L-1 .. 1: the sparse Top-K of every sibling group over the children of
//      its parent's picks (select_children_unit), one barrier after each level.
// The units are the bodies of the separate pyramid and selection kernels, so the results are
// bit-identical to theirs; only the launches between them are gone (4 launches at L = 3).
// Used for bf16 inputs when the coarsest level is small (n_L <= 64) and K is 2, 4, 8 or 16.
//
// Grid barrier: a monotonic arrival counter in global memory (zeroed before the launch);
// barrier b completes when b * gridDim.x CTAs have arrived.  The cooperative launch keeps
// every CTA resident, and every wait is bounded: a barrier that does not complete within the
// wait limit records LLSA_ERR_TIMEOUT, and the CTA skips the remaining work (still arriving
// at the later barriers, so no other CTA waits on it).
#pragma once

#include "select.cuh"

namespace llsa {

// Bytes of the shared buffer of pyramid_select_kernel: the largest of its phases' buffers.
template <int D, int CPT>
__host__ __device__ constexpr int pyramid_select_smem() {
  using C = PyrCfg<__nv_bfloat16, D>;
  constexpr int pyr = C::SPAN + C::ROWS * D * 4;
  constexpr int top = coarsest_small_smem<D>();
  constexpr int sel = (int)sizeof(float) * (kBlock * D + 32 * CPT * sel_row_stride<D>() + 32 * CPT);
  return pyr > top ? (pyr > sel ? pyr : sel) : (top > sel ? top : sel);
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Arrive at grid barrier number `phase` (1, 2, ...) and wait, bounded, for all CTAs.  The
// arrival follows a gpu-scope fence (release) and the wait polls with gpu-scope acquire
// loads, so the writes of every CTA before the barrier are visible to every CTA after it
// (through the coherent path: loads of such data here do not use the read-only cache).
__device__ __forceinline__ bool grid_barrier(unsigned* counter, unsigned phase) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's writes are visible before its arrival is
    atomicAdd(counter, 1u);
    const unsigned target = phase * gridDim.x;
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire_gpu(counter) < target) {
      if (*reinterpret_cast<volatile int*>(&g_llsa_status) == LLSA_ERR_TIMEOUT || clock64() - t0 > kWaitLimitCycles) {
        record_error(LLSA_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();  // the other CTAs' writes are read after the barrier
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

template <int D, int CPT>
__global__ void __launch_bounds__(kSelThreads) pyramid_select_kernel(Geometry g, const __nv_bfloat16* __restrict__ q,
                                                                     const __nv_bfloat16* __restrict__ k,
                                                                     const __nv_bfloat16* __restrict__ v,
                                                                     float* __restrict__ q_pyr,
                                                                     float* __restrict__ k_pyr,
                                                                     float* __restrict__ v_pyr, int* __restrict__ idx,
                                                                     unsigned* __restrict__ barrier,
                                                                     const __grid_constant__ CUtensorMap pm0,
                                                                     const __grid_constant__ CUtensorMap pm1,
                                                                     const __grid_constant__ CUtensorMap pm2) {
  using C = PyrCfg<__nv_bfloat16, D>;
  static_assert(C::THREADS == kSelThreads, "one block shape for every phase");
  extern __shared__ __align__(128) uint8_t ps_smem[];
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  bool ok = true;
  unsigned phase = 0;
  // 1. levels 1-2 of q, k, v
  {
    const int tiles = (g.n[1] + C::ROWS - 1) / C::ROWS;
    const int per_tensor = g.BH * tiles;
    uint32_t parity = 0;
    float(*s1)[D] = reinterpret_cast<float(*)[D]>(ps_smem + C::SPAN);
    for (int u = blockIdx.x; u < 3 * per_tensor && ok; u += gridDim.x) {
      const int t = u / per_tensor;
      const int rem = u - t * per_tensor;
      const int bh = rem / tiles;
      const __nv_bfloat16* x = t == 0 ? q : (t == 1 ? k : v);
      float* pyr = t == 0 ? q_pyr : (t == 1 ? k_pyr : v_pyr);
      const CUtensorMap* pm = t == 0 ? &pm0 : (t == 1 ? &pm1 : &pm2);
      ok = pyramid_l12_unit<__nv_bfloat16, D>(g, x, pyr, bh, rem - bh * tiles, ps_smem, s1, bar, parity, pm);
      parity ^= 1u;
    }
  }
  ok = grid_barrier(barrier, ++phase) && ok;
  // 2. levels 3..L and the coarsest selection, per (b, h)
  float* fs = reinterpret_cast<float*>(ps_smem);
  for (int u = blockIdx.x; u < g.BH && ok; u += gridDim.x) {
    if (g.L >= 3)
      coarsest_small_unit<D, true>(g, q_pyr, k_pyr, v_pyr, idx, u, fs);
    else
      coarsest_small_unit<D, false>(g, q_pyr, k_pyr, v_pyr, idx, u, fs);
  }
  // 3. the sparse levels, coarsest first
  for (int l = g.L - 1; l >= 1; --l) {
    ok = grid_barrier(barrier, ++phase) && ok;
    const int units = g.BH * (g.n[l] / kBlock);
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x)
      select_children_unit<D, CPT, false>(g, l, q_pyr + g.pyr_off[l], k_pyr + g.pyr_off[l],
                                          idx + g.idx_off[l + 1], idx + g.idx_off[l], u, fs);
  }
}

}  // namespace llsa
